// Block lists of the fixed comparison masks (Longformer, BigBird) in the same
// CSR / CSC / pairing-order layout the attention calls take.
//
// Gzip-guided Sparse Attention (daiwk.github.io), background paragraph of
// "核心公式", and the arXiv abstract: BigBird and Longformer are the fixed,
// content-blind masks the method is compared with.  At block granularity and
// causal, like the adaptive mask:
//   Longformer: live(i, j) = j <= i and (i - j <= w or j < g or i < g)
//   BigBird:    the same, or j in R_i = {u_ik mod (i + 1) : k < r}
// with w the window half-width in blocks, g the global blocks (the first g)
// and u_ik the caller's uniform 32-bit words (the random draws are inputs).
//
// One CTA per (class slot, sample); the three class slots receive the same
// lists, so any head-to-class map reads the fixed mask.  Rows are built a
// 32-bit word of key blocks at a time (window, global and random bits OR-ed,
// then cut causally; the random bits come from a per-warp row bitmap), so a
// row's entries come out ascending without a sort.  Columns are built by
// testing live(i, j) for i = j .. n-1 a warp-wide chunk at a time, with the
// random picks of every row held in shared memory.
#pragma once

#include "flags_csr.cuh"

namespace gsa {
namespace fixed {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxBlocks = 8192;
constexpr int kMaxRandom = 8;

struct FixedArgs {
    int kind;            // 0 Longformer, 1 BigBird
    int nblk, w, g, r;
    const uint32_t* rnd; // [B][nblk][r]
    int64_t cap;
    int32_t* row_ptr;
    int32_t* col_idx;
    int32_t* col_ptr;
    int32_t* row_idx;
    int32_t* q_order;
    int32_t* k_order;
};

// shared memory: picks [n][r] int16, rptr [n+1], cptr [n+1], scan scratch [64],
// per-warp row bitmaps [kWarps][n/32 rounded up]
inline size_t smem_bytes(int n, int r) {
    const size_t words = (static_cast<size_t>(n) + 31) / 32;
    return ((static_cast<size_t>(n) * r * 2 + 15) & ~static_cast<size_t>(15)) + 2 * (static_cast<size_t>(n) + 1) * 4 +
           64 * 4 + kWarps * words * 4;
}

// Bits of the key blocks [lo, hi] that fall in word wd (blocks 32 wd .. 32 wd + 31).
__device__ __forceinline__ uint32_t range_bits(int lo, int hi, int wd) {
    const int a = lo > 32 * wd ? lo - 32 * wd : 0;
    const int b = hi < 32 * wd + 31 ? hi - 32 * wd : 31;
    if (b < a) return 0u;
    const uint32_t upto_b = b == 31 ? 0xffffffffu : ((1u << (b + 1)) - 1u);
    return upto_b & ~((1u << a) - 1u);
}

__global__ void __launch_bounds__(kThreads) build_fixed_csr_kernel(FixedArgs a) {
    extern __shared__ __align__(16) uint8_t dsm[];
    const int n = a.nblk, r = a.r, w = a.w, g = a.g;
    const int nwords = (n + 31) >> 5;
    int16_t* picks = reinterpret_cast<int16_t*>(dsm);
    int* rptr = reinterpret_cast<int*>(dsm + ((static_cast<size_t>(n) * r * 2 + 15) & ~static_cast<size_t>(15)));
    int* cptr = rptr + n + 1;
    int* scratch = cptr + n + 1;
    uint32_t* rowbits_all = reinterpret_cast<uint32_t*>(scratch + 64);
    const int c = blockIdx.x, s = blockIdx.y;
    const int64_t gi = static_cast<int64_t>(s) * 3 + c;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t* rowbits = rowbits_all + warp * nwords;
    const bool bigbird = a.kind == 1 && r > 0;

    if (bigbird) {
        const uint32_t* src = a.rnd + static_cast<int64_t>(s) * n * r;
        for (int e = threadIdx.x; e < n * r; e += blockDim.x) {
            const int i = e / r;
            picks[e] = static_cast<int16_t>(src[e] % static_cast<uint32_t>(i + 1));
        }
    }
    __syncthreads();

    // the key-block word wd of row i (ascending bits), given the warp's random bitmap of row i
    auto row_word = [&](int i, int wd) {
        uint32_t v = range_bits(i - w < 0 ? 0 : i - w, i, wd) | range_bits(0, g - 1, wd);
        if (i < g) v |= range_bits(0, i, wd);
        if (bigbird) v |= rowbits[wd];
        return v & range_bits(0, i, wd);
    };
    auto load_rowbits = [&](int i) {
        if (!bigbird) return;
        for (int wd = lane; wd < nwords; wd += 32) rowbits[wd] = 0u;
        __syncwarp();
        if (lane < r) {
            const int j = picks[i * r + lane];
            atomicOr(&rowbits[j >> 5], 1u << (j & 31));
        }
        __syncwarp();
    };
    auto live_col = [&](int i, int j) {   // i >= j
        bool v = (i - j <= w) || (j < g) || (i < g);
        if (bigbird && !v) {
            for (int k = 0; k < r; ++k) v = v || picks[i * r + k] == j;
        }
        return v;
    };
    const int per = (nwords + 31) >> 5;   // words per lane in a row
    const int w0 = lane * per, w1 = w0 + per < nwords ? w0 + per : nwords;

    // ---- counts
    for (int i = warp; i < n; i += kWarps) {
        load_rowbits(i);
        int cnt = 0;
        for (int wd = w0; wd < w1; ++wd) cnt += __popc(row_word(i, wd));
        for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        if (lane == 0) rptr[i] = cnt;
        __syncwarp();   // the bitmap is rewritten for the next row
    }
    for (int j = warp; j < n; j += kWarps) {
        int cnt = 0;
        for (int i0 = j; i0 < n; i0 += 32) {
            const int i = i0 + lane;
            cnt += __popc(__ballot_sync(0xffffffffu, i < n && live_col(i, j)));
        }
        if (lane == 0) cptr[j] = cnt;
    }
    __syncthreads();

    // ---- pointers: exclusive scans over contiguous chunks of blocks
    const int chunk = (n + blockDim.x - 1) / blockDim.x;
    const int lo = threadIdx.x * chunk < n ? threadIdx.x * chunk : n;
    const int hi = lo + chunk < n ? lo + chunk : n;
    int rc = 0, cc = 0;
    for (int i = lo; i < hi; ++i) {
        rc += rptr[i];
        cc += cptr[i];
    }
    int rtot, ctot;
    int roff = mask::block_exclusive_scan(rc, scratch, &rtot);
    int coff = mask::block_exclusive_scan(cc, scratch, &ctot);
    for (int i = lo; i < hi; ++i) {
        const int rv = rptr[i], cv = cptr[i];
        rptr[i] = roff;
        roff += rv;
        cptr[i] = coff;
        coff += cv;
    }
    if (threadIdx.x == 0) {
        rptr[n] = rtot;
        cptr[n] = ctot;
    }
    __syncthreads();
    for (int i = threadIdx.x; i <= n; i += blockDim.x) {
        a.row_ptr[gi * (n + 1) + i] = rptr[i];
        a.col_ptr[gi * (n + 1) + i] = cptr[i];
    }
    // pairing orders: query blocks descending (later rows see more keys, so
    // heaviest first), key blocks ascending (earlier keys are seen by more rows)
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        a.q_order[gi * n + i] = n - 1 - i;
        a.k_order[gi * n + i] = i;
    }

    // ---- entries
    int32_t* cidx = a.col_idx + gi * a.cap;
    int32_t* ridx = a.row_idx + gi * a.cap;
    for (int i = warp; i < n; i += kWarps) {
        load_rowbits(i);
        int cnt = 0;
        for (int wd = w0; wd < w1; ++wd) cnt += __popc(row_word(i, wd));
        int incl = cnt;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int pos = rptr[i] + incl - cnt;
        for (int wd = w0; wd < w1; ++wd) {
            uint32_t u = row_word(i, wd);
            while (u) {
                const int bit = __ffs(u) - 1;
                u &= u - 1;
                cidx[pos++] = 32 * wd + bit;
            }
        }
        __syncwarp();
    }
    for (int j = warp; j < n; j += kWarps) {
        int pos = cptr[j];
        for (int i0 = j; i0 < n; i0 += 32) {
            const int i = i0 + lane;
            const bool v = i < n && live_col(i, j);
            const uint32_t bal = __ballot_sync(0xffffffffu, v);
            if (v) ridx[pos + __popc(bal & ((1u << lane) - 1u))] = i;
            pos += __popc(bal);
        }
    }
}

}  // namespace fixed
}  // namespace gsa
