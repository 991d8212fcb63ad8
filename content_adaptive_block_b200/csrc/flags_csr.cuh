// Literal flags and the per-class block lists of the adaptive mask.
//
// Flags — Gzip-guided Sparse Attention (daiwk.github.io), section "核心公式",
// l_i = 1[r_i > r̄] with r̄ the mean over the sample's blocks.  Multiplying
// both sides by b * nblk gives the integer test len_i * nblk > Σ_j len_j,
// evaluated in 64 bits: one CTA per sample, a block reduction, a compare.
//
// Lists — same section, mask equation M = M_lit ∪ M_local ∪ I ∩ causal, and
// "背景与主要改动" for the head classes.  For a sample with literal prefix
// counts P(i) = #{literal j <= i} and n_lit literals, the live key blocks of
// query block i, ascending, are:
//   local   : max(0, i-w) .. i
//   literal : every literal j <= i if l_i, else just i
//   hybrid  : the literal j < i-w (if l_i), then max(0, i-w) .. i
// and the query blocks that see key block j, ascending:
//   local   : j .. min(nblk-1, j+w)
//   literal : every literal i >= j if l_j, else just j
//   hybrid  : j .. min(nblk-1, j+w), then the literal i > j+w (if l_j)
// One CTA per (class, sample): a block scan of the flags gives P and the
// list of literal blocks; a scan of the row (column) counts gives the CSR
// (CSC) pointers; one warp per row (column) writes its entries, so the
// stores of a row are contiguous.
#pragma once

#include "common.cuh"

namespace gsa {
namespace mask {

constexpr int kThreads = 512;
constexpr int kMaxBlocksCsr = 8192;

__global__ void __launch_bounds__(256) literal_flags_kernel(const int32_t* __restrict__ lengths, int nblk,
                                                            uint8_t* __restrict__ flags) {
    __shared__ long long part[8];
    const int64_t s = blockIdx.x;
    const int32_t* row = lengths + s * nblk;
    long long acc = 0;
    for (int i = threadIdx.x; i < nblk; i += blockDim.x) acc += row[i];
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    long long total = 0;
    for (int k = 0; k < static_cast<int>(blockDim.x >> 5); ++k) total += part[k];
    for (int i = threadIdx.x; i < nblk; i += blockDim.x)
        flags[s * nblk + i] = static_cast<long long>(row[i]) * nblk > total ? 1 : 0;
}

// Exclusive scan over the CTA of one value per thread.  Returns the
// thread's exclusive prefix; *total receives the sum.
__device__ int block_exclusive_scan(int v, int* scratch, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < static_cast<int>(blockDim.x >> 5) ? scratch[lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        scratch[32 + lane] = w;   // inclusive warp totals
    }
    __syncthreads();
    const int before = warp > 0 ? scratch[32 + warp - 1] : 0;
    *total = scratch[32 + (blockDim.x >> 5) - 1];
    __syncthreads();
    return before + x - v;
}

struct CsrArgs {
    const uint8_t* flags;
    int nblk;
    int w;
    int64_t cap;
    int32_t* row_ptr;
    int32_t* col_idx;
    int32_t* col_ptr;
    int32_t* row_idx;
    int32_t* q_order;
    int32_t* k_order;
    int cls[3];   // the classes built: CTA column x of the list kernel builds class cls[x]
};

__device__ __forceinline__ int imin(int a, int b) { return a < b ? a : b; }
__device__ __forceinline__ int imax(int a, int b) { return a > b ? a : b; }

// The threads that build one (sample, class)'s lists together: the whole CTA
// (CtaGroup, any multiple of 32 threads up to 1024) or one warp (WarpGroup).
struct CtaGroup {
    __device__ __forceinline__ int rank() const { return threadIdx.x; }
    __device__ __forceinline__ int size() const { return blockDim.x; }
    __device__ __forceinline__ int warp() const { return threadIdx.x >> 5; }
    __device__ __forceinline__ int nwarps() const { return blockDim.x >> 5; }
    __device__ __forceinline__ void sync() const { __syncthreads(); }
    __device__ __forceinline__ int scan(int v, int* scratch, int* total) const {
        return block_exclusive_scan(v, scratch, total);
    }
};
struct WarpGroup {
    __device__ __forceinline__ int rank() const { return threadIdx.x & 31; }
    __device__ __forceinline__ int size() const { return 32; }
    __device__ __forceinline__ int warp() const { return 0; }
    __device__ __forceinline__ int nwarps() const { return 1; }
    __device__ __forceinline__ void sync() const { __syncwarp(); }
    __device__ __forceinline__ int scan(int v, int*, int* total) const {
        const int lane = threadIdx.x & 31;
        int x = v;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        *total = __shfl_sync(0xffffffffu, x, 31);
        return x - v;
    }
};

// Lists of class c for sample s, by the group G (every thread of it calls
// this); dsm holds csr_smem_bytes(nblk).  Reads the flags from a.flags (a
// group that wrote them must synchronise first), or, with flags_ready,
// finds them (0 / 1) already in dsm[0 .. nblk).
template <typename G>
__device__ void build_csr_sample(const CsrArgs& a, int c, int s, uint8_t* dsm, bool flags_ready, const G& grp) {
    const int n = a.nblk;
    uint8_t* fl = dsm;                                              // [n]
    int* pre = reinterpret_cast<int*>(dsm + ((n + 15) & ~15));      // [n] inclusive literal count
    int* lit = pre + n;                                             // [n] literal block list
    int* rptr = lit + n;                                            // [n + 1]
    int* cptr = rptr + n + 1;                                       // [n + 1]
    int* scratch = cptr + n + 1;                                    // [64]

    const int64_t g = static_cast<int64_t>(s) * 3 + c;
    const int w = a.w;
    if (!flags_ready)
        for (int i = grp.rank(); i < n; i += grp.size()) fl[i] = a.flags[static_cast<int64_t>(s) * n + i] ? 1 : 0;
    grp.sync();

    // literal prefix counts: each thread scans a contiguous chunk
    const int chunk = (n + grp.size() - 1) / grp.size();
    const int lo = imin(n, grp.rank() * chunk), hi = imin(n, lo + chunk);
    int cnt = 0;
    for (int i = lo; i < hi; ++i) cnt += fl[i];
    int nlit;
    int off = grp.scan(cnt, scratch, &nlit);
    for (int i = lo; i < hi; ++i) {
        if (fl[i]) lit[off++] = i;
        pre[i] = off;
    }
    grp.sync();

    // row and column counts
    auto lit_upto = [&](int i) { return i < 0 ? 0 : pre[i]; };   // literal j <= i
    auto row_count = [&](int i) {
        const int win = i - imax(0, i - w) + 1;
        if (c == 0) return win;
        if (c == 1) return fl[i] ? pre[i] : 1;
        return win + (fl[i] ? lit_upto(i - w - 1) : 0);
    };
    auto col_count = [&](int j) {
        const int win = imin(n - 1, j + w) - j + 1;
        if (c == 0) return win;
        if (c == 1) return fl[j] ? nlit - pre[j] + 1 : 1;
        return win + (fl[j] ? nlit - pre[imin(n - 1, j + w)] : 0);
    };
    int rc = 0, cc = 0;
    for (int i = lo; i < hi; ++i) { rc += row_count(i); cc += col_count(i); }
    int rtot, ctot;
    int roff = grp.scan(rc, scratch, &rtot);
    int coff = grp.scan(cc, scratch, &ctot);
    for (int i = lo; i < hi; ++i) {
        rptr[i] = roff;
        roff += row_count(i);
        cptr[i] = coff;
        coff += col_count(i);
    }
    if (grp.rank() == 0) {
        rptr[n] = rtot;
        cptr[n] = ctot;
    }
    grp.sync();
    for (int i = grp.rank(); i <= n; i += grp.size()) {
        a.row_ptr[g * (n + 1) + i] = rptr[i];
        a.col_ptr[g * (n + 1) + i] = cptr[i];
    }

    // tile orders: local classes keep block order; literal and hybrid
    // classes put literal blocks together (descending for query tiles,
    // heaviest first; ascending for key tiles, heaviest first)
    for (int i = grp.rank(); i < n; i += grp.size()) {
        int qpos, kpos;
        if (c == 0) {
            qpos = i;
            kpos = i;
        } else if (fl[i]) {
            qpos = nlit - pre[i];
            kpos = pre[i] - 1;
        } else {
            const int nonlit_upto = i + 1 - pre[i];   // non-literal j <= i
            qpos = nlit + (n - nlit) - nonlit_upto;
            kpos = nlit + nonlit_upto - 1;
        }
        a.q_order[g * n + qpos] = i;
        a.k_order[g * n + kpos] = i;
    }

    // entries: one warp per row / column, so the stores of a row are contiguous
    const int lane = grp.rank() & 31, warp = grp.warp(), nwarps = grp.nwarps();
    int32_t* cidx = a.col_idx + g * a.cap;
    int32_t* ridx = a.row_idx + g * a.cap;
    for (int i = warp; i < n; i += nwarps) {
        const int cntr = rptr[i + 1] - rptr[i];
        const int wlo = imax(0, i - w);
        const int nfar = (c == 2 && fl[i]) ? lit_upto(i - w - 1) : 0;   // hybrid: literal j < i-w
        for (int e = lane; e < cntr; e += 32) {
            int j;
            if (c == 0) j = wlo + e;
            else if (c == 1) j = fl[i] ? lit[e] : i;
            else j = e < nfar ? lit[e] : wlo + (e - nfar);
            cidx[rptr[i] + e] = j;
        }
        const int cntc = cptr[i + 1] - cptr[i];
        const int whi = imin(n - 1, i + w);
        const int nwin = whi - i + 1;
        for (int e = lane; e < cntc; e += 32) {
            int q;
            if (c == 0) q = i + e;
            else if (c == 1) q = fl[i] ? lit[pre[i] - 1 + e] : i;
            else q = e < nwin ? i + e : lit[pre[whi] + (e - nwin)];
            ridx[cptr[i] + e] = q;
        }
    }
}

__device__ __forceinline__ void build_csr_sample(const CsrArgs& a, int c, int s, uint8_t* dsm,
                                                 bool flags_ready = false) {
    build_csr_sample(a, c, s, dsm, flags_ready, CtaGroup{});
}

__global__ void __launch_bounds__(kThreads) build_csr_kernel(CsrArgs a) {
    extern __shared__ __align__(16) uint8_t dsm[];
    // grid (classes built, sample); a select, not an indexed read, keeps the
    // parameters out of local memory
    const int c = blockIdx.x == 0 ? a.cls[0] : (blockIdx.x == 1 ? a.cls[1] : a.cls[2]);
    build_csr_sample(a, c, blockIdx.y, dsm);
}

inline size_t csr_smem_bytes(int n) {
    return static_cast<size_t>((n + 15) & ~15) + sizeof(int) * (2 * static_cast<size_t>(n) + 2 * (n + 1) + 64);
}

}  // namespace mask
}  // namespace gsa
