// The whole mask stage in one launch: per-block gzip lengths -> literal
// flags -> per-class block lists.
//
// Gzip-guided Sparse Attention (daiwk.github.io), flowchart and section
// "核心公式": gzip level-1 per block, r_i > r̄ per sample, then the mask of
// each head class.  The flags of a sample need every one of its lengths, so
// the stages meet per sample: each CTA (four warps, one block each, as in the
// lengths kernel) adds the number of blocks it finished for each sample to a
// per-sample counter after a fence; the CTA whose addition completes a
// sample computes that sample's flags and its three classes' lists with all
// 128 threads, reusing the shared memory of the lengths phase, and resets the
// counter.  No CTA waits for another, so nothing can stall.
#pragma once

#include "deflate_len.cuh"
#include "flags_csr.cuh"

namespace gsa {
namespace pipeline {

constexpr int kMaxBlocks = 1024;   // block lists built in the lengths phase's shared memory
// the list scratch of build_csr_sample (csr_smem_bytes) fits in the lengths phase's
static_assert(sizeof(deflate::WarpSmem) * deflate::kWarps >=
                  ((kMaxBlocks + 15) & ~15) + 4 * (2 * kMaxBlocks + 2 * (kMaxBlocks + 1) + 64),
              "list scratch fits in the lengths scratch");

__global__ void __launch_bounds__(32 * deflate::kWarps)
mask_pipeline_kernel(const uint8_t* __restrict__ bytes, int64_t L, int b, int64_t nblocks_total,
                     int32_t* __restrict__ lengths, uint8_t* __restrict__ flags, mask::CsrArgs a,
                     int* __restrict__ counters) {
    extern __shared__ __align__(16) uint8_t dsmem[];
    __shared__ int fin[deflate::kWarps];
    __shared__ int nfin;
    __shared__ long long part[deflate::kWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nblk = L / b;
    const int64_t task0 = static_cast<int64_t>(blockIdx.x) * deflate::kWarps;
    const int64_t task = task0 + warp;
    if (task < nblocks_total) {
        deflate::WarpSmem& ws = reinterpret_cast<deflate::WarpSmem*>(dsmem)[warp];
        const int64_t s = task / nblk, i = task % nblk;
        const int len = deflate::block_length_warp(ws, bytes + s * L + i * b, b, lane);
        if (lane == 0) {
            lengths[task] = len;
            __threadfence();   // ordered before this CTA's counter update
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // this CTA's blocks, per sample (consecutive tasks: samples ascend)
        nfin = 0;
        int64_t t = task0;
        const int64_t tend = task0 + deflate::kWarps < nblocks_total ? task0 + deflate::kWarps : nblocks_total;
        while (t < tend) {
            const int64_t s = t / nblk;
            const int64_t send = (s + 1) * nblk < tend ? (s + 1) * nblk : tend;
            const int cnt = static_cast<int>(send - t);
            if (atomicAdd(&counters[s], cnt) + cnt == nblk) fin[nfin++] = static_cast<int>(s);
            t = send;
        }
    }
    __syncthreads();
    for (int f = 0; f < nfin; ++f) {
        const int s = fin[f];
        __threadfence();   // the other CTAs' lengths of this sample are visible
        const int32_t* row = lengths + static_cast<int64_t>(s) * nblk;
        long long acc = 0;
        for (int i = threadIdx.x; i < nblk; i += blockDim.x) acc += __ldcg(row + i);
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) part[warp] = acc;
        __syncthreads();
        long long total = 0;
        for (int k = 0; k < deflate::kWarps; ++k) total += part[k];
        uint8_t* frow = flags + static_cast<int64_t>(s) * nblk;
        for (int i = threadIdx.x; i < nblk; i += blockDim.x)
            frow[i] = static_cast<long long>(__ldcg(row + i)) * nblk > total ? 1 : 0;
        __syncthreads();
        for (int c = 0; c < 3; ++c) {
            mask::build_csr_sample(a, c, s, dsmem);
            __syncthreads();
        }
        if (threadIdx.x == 0) counters[s] = 0;   // ready for the next call
    }
}

}  // namespace pipeline
}  // namespace gsa
