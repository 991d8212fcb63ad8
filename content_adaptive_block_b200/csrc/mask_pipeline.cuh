// The whole mask stage in one launch: per-block gzip lengths -> literal
// flags -> per-class block lists.
//
// Gzip-guided Sparse Attention (daiwk.github.io), flowchart and section
// "核心公式": gzip level-1 per block, r_i > r̄ per sample, then the mask of
// each head class.  The flags of a sample need all of its lengths, so the
// launch is cooperative (every CTA resident at once) with two phases and one
// grid barrier between them:
//   1. lengths: the CTA's lengths warps take chunks of consecutive blocks,
//      one block per lane, exactly as the lengths kernel does
//      (deflate_lane.cuh);
//   2. lists: jobs (sample, class) spread over the CTAs, all of a CTA's
//      warps on one job (or, for short lists and many jobs, one job per
//      warp).  A job sums its sample's lengths, sets the flags
//      (len_i * nblk > Σ len) in shared memory — the sample's first job also
//      writes them out — and builds the class's lists.  The local class's
//      lists depend only on (nblk, w) (mask equation: |i - j| <= w
//      intersected with causality), so they are not built at all: the
//      attention kernels derive them.
// The barrier: each CTA adds one to a counter in caller-owned memory and
// waits (bounded by a time limit, after which it records an error code and
// leaves) until all have; each CTA adds one more as it leaves, and the last
// to leave sets the counter back to zero for the next call.
#pragma once

#include "deflate_lane.cuh"
#include "flags_csr.cuh"

namespace gsa {
namespace pipeline {

constexpr int kMaxBlocks = 1024;   // blocks per sample (the lists' scratch sits in the CTA's shared memory)

// A CTA of T warps, the first W of which compute lengths in phase 1 (each
// with its lanes' words in shared memory, which phase 2 reuses as the list
// jobs' scratch); all T build lists in phase 2.  Phase 1's shared memory caps
// the lengths warps per SM, phase 2 needs none of it, so the CTA carries
// more warps than phase 1 can use.
template <int MAXB, int W, int T>
struct Shape {
    static constexpr int kWarpBytes = deflate_lane::Layout<MAXB>::kWords * 128;
    static constexpr int kLengthsWarps = W;
    static constexpr int kWarps = T;
    static constexpr size_t kLengthsBytes = static_cast<size_t>(W) * kWarpBytes;
    static constexpr size_t kListBytes = ((kMaxBlocks + 15) & ~15) + 4 * (2 * kMaxBlocks + 2 * (kMaxBlocks + 1) + 64);
    static constexpr size_t kSmemBytes = kLengthsBytes > kListBytes ? kLengthsBytes : kListBytes;
    // a warp job's scratch (lists of at most kMaxWarpJobBlocks blocks), one per warp
    static constexpr int kMaxWarpJobBlocks = 64;
    static constexpr size_t kWarpJobBytes = (((kMaxWarpJobBlocks + 15) & ~15) + 4 * (2 * kMaxWarpJobBlocks + 2 * (kMaxWarpJobBlocks + 1) + 64) + 15) & ~size_t(15);
    static_assert(kSmemBytes <= 227 * 1024, "pipeline CTA above the shared-memory limit");
    static_assert(T * kWarpJobBytes <= kSmemBytes, "warp job scratch does not fit");
    static_assert(W <= T, "lengths warps are a subset of the CTA");
    // CTAs per SM that phase 1's shared memory allows: the register cap
    // below keeps them all resident
    static constexpr int kPerSm = 232448 / (static_cast<int>(kSmemBytes) + 1024) < 8
                                      ? 232448 / (static_cast<int>(kSmemBytes) + 1024) : 8;
};

// The two CTA shapes of each block size.  Wide: as many lengths warps as fit
// one CTA, and 32 warps in all (64 registers a thread), so a few list jobs,
// or long lists, each get many threads.
// Narrow: the fewest lengths warps that keep an SM's lengths warps at the
// shared-memory maximum, so many list jobs run side by side (one per CTA),
// plus list-only warps up to 64 registers a thread over the SM.
template <int MAXB>
struct Shapes {
    static constexpr int kWarpBytes = deflate_lane::Layout<MAXB>::kWords * 128;
    static constexpr int kWideW = 220 * 1024 / kWarpBytes < 16 ? 220 * 1024 / kWarpBytes : 16;
    static constexpr int kWideT = 32;
    static constexpr int kNarrowW = MAXB > 64 ? 1 : 3;
    static constexpr int kNarrowT = MAXB > 64 ? 8 : 6;
};

struct PipeArgs {
    const uint8_t* bytes;
    int b;
    int B;
    int nblk;
    int64_t total;        // B * nblk blocks
    int32_t* lengths;     // [B][nblk]
    uint8_t* flags;       // [B][nblk]
    mask::CsrArgs a;
    int* counter;         // the grid barrier's counter (zero between calls)
    int nper;             // classes built per sample (literal, hybrid: the local class is implicit)
    int per[3];           // ... and which
    int warp_jobs;        // 1: a list job per warp (each warp a scratch of its own), 0: a job per CTA
    int bpw;              // blocks per warp in the lengths phase (1 .. 32)
};

// All CTAs of the grid reach this point (thread 0 of each waits, bounded);
// false when the wait gave up.
__device__ __forceinline__ bool grid_barrier(int* counter, int target) {
    __shared__ int ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();   // this CTA's lengths before its arrival
        atomicAdd(counter, 1);
        ok = 1;
        const unsigned long long t0 = globaltimer_ns();
        for (uint32_t it = 0;; ++it) {
            int v;
            asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
            if (v >= target) break;
            __nanosleep(256);   // leave the SM's issue slots to the warps still computing lengths
            if ((it & 15u) == 15u && globaltimer_ns() - t0 > kWaitLimitNs) {
                record_error(kErrTimeoutOther);
                ok = 0;
                break;
            }
        }
        __threadfence();
    }
    __syncthreads();
    return ok != 0;
}

template <int MAXB, int W, int T>
__global__ void __launch_bounds__(32 * T, (Shape<MAXB, W, T>::kPerSm)) mask_pipeline_kernel(const PipeArgs P) {
    using S = Shape<MAXB, W, T>;
    extern __shared__ __align__(16) uint8_t dsmem[];
    __shared__ long long part[T];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- phase 1: lengths, chunks of bpw blocks per lengths warp (one per
    // lane); consecutive chunks go to consecutive CTAs, so a small batch
    // still spreads over the SMs
    if (warp < W) {
        uint32_t* region = reinterpret_cast<uint32_t*>(dsmem) +
                           static_cast<size_t>(warp) * deflate_lane::Layout<MAXB>::kWords * 32;
        const int64_t nchunks = (P.total + P.bpw - 1) / P.bpw;
        for (int64_t ch = static_cast<int64_t>(warp) * gridDim.x + blockIdx.x; ch < nchunks;
             ch += static_cast<int64_t>(gridDim.x) * W) {
            const int64_t task0 = ch * P.bpw;
            const int nb = P.total - task0 < P.bpw ? static_cast<int>(P.total - task0) : P.bpw;
            deflate_lane::warp_block_lengths<MAXB>(region, P.bytes, P.b, task0, nb, P.lengths, lane);
        }
    }
    if (!grid_barrier(P.counter, static_cast<int>(gridDim.x))) return;

    // ---- phase 2: (sample, class) jobs.  Per sample max(nper, 1) jobs (one
    // writes the flags even when no list is built).
    const int n = P.nblk;
    const int jobs_per = P.nper > 0 ? P.nper : 1;
    const int njobs = P.B * jobs_per;
    if (P.warp_jobs) {
        // one job per warp at a time, each warp with its own scratch: all the
        // jobs run side by side instead of a few per CTA in turn
        uint8_t* ws = dsmem + static_cast<size_t>(warp) * S::kWarpJobBytes;
        for (int j = blockIdx.x * T + warp; j < njobs; j += gridDim.x * T) {
            const int s = j / jobs_per;
            const int k = j % jobs_per;
            const int c = P.nper > 0 ? P.per[k] : -1;
            __syncwarp();
            const int32_t* row = P.lengths + static_cast<int64_t>(s) * n;
            long long acc = 0;
            for (int i = lane; i < n; i += 32) acc += __ldcg(row + i);
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            const bool write = k == 0;
            for (int i = lane; i < n; i += 32) {
                const uint8_t f = static_cast<long long>(__ldcg(row + i)) * n > acc ? 1 : 0;
                ws[i] = f;
                if (write) P.flags[static_cast<int64_t>(s) * n + i] = f;
            }
            if (c >= 0) mask::build_csr_sample(P.a, c, s, ws, true, mask::WarpGroup{});
        }
        __syncthreads();
        if (threadIdx.x == 0 && atomicAdd(P.counter, 1) == 2 * static_cast<int>(gridDim.x) - 1) *P.counter = 0;
        return;
    }
    uint8_t* fl = dsmem;   // the list builder's flag scratch: dsm[0 .. n)
    for (int j = blockIdx.x; j < njobs; j += gridDim.x) {
        const int s = j / jobs_per;
        const int k = j % jobs_per;
        const int c = P.nper > 0 ? P.per[k] : -1;
        __syncthreads();   // the previous job's scratch
        const int32_t* row = P.lengths + static_cast<int64_t>(s) * n;
        long long acc = 0;
        for (int i = threadIdx.x; i < n; i += blockDim.x) acc += __ldcg(row + i);
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) part[warp] = acc;
        __syncthreads();
        long long total = 0;
        for (int w = 0; w < T; ++w) total += part[w];
        const bool write = k == 0;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const uint8_t f = static_cast<long long>(__ldcg(row + i)) * n > total ? 1 : 0;
            fl[i] = f;
            if (write) P.flags[static_cast<int64_t>(s) * n + i] = f;
        }
        if (c >= 0) mask::build_csr_sample(P.a, c, s, dsmem, true);
    }

    // ---- leave: the last CTA out resets the counter for the next call
    __syncthreads();
    if (threadIdx.x == 0 && atomicAdd(P.counter, 1) == 2 * static_cast<int>(gridDim.x) - 1) *P.counter = 0;
}

}  // namespace pipeline
}  // namespace gsa
