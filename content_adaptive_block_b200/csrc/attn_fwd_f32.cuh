// Block-sparse causal attention forward in float32 on the CUDA cores.
//
// Gzip-guided Sparse Attention (daiwk.github.io), section "复现边界": the
// reproduction evaluates softmax(Q K^T / sqrt(d) + mask) V; section "核心公式"
// defines the mask.  This kernel visits only the live key blocks of each
// query block (the CSR row of its sample and head class) and applies the
// token-level causal cut inside the diagonal block, with an online softmax
// in float32 (IEEE expf/logf).  It is the precision path for small float32
// problems; the bf16 tensor-core kernel is the throughput path.
//
// One CTA per (query block, head, sample); thread r owns query row r of the
// block and its d-wide accumulator; K and V tiles of each live block are
// staged in shared memory and read by all rows.
#pragma once

#include "common.cuh"

namespace gsa {
namespace f32 {

constexpr int kMaxHeads = 256;

struct Params {
    const float* q;
    const float* k;
    const float* v;
    float* o;
    float* lse;
    const int32_t* row_ptr;
    const int32_t* col_idx;
    int64_t cap;
    int S, H, nblk, b;
    int64_t L;
    float scale;
    uint8_t cls[kMaxHeads];
    int local_implicit;   // the local class's lists are not stored: derived from (nblk, w)
    int w;                // the lists' window
};

template <int D>
__global__ void __launch_bounds__(128) attn_fwd_f32_kernel(Params p) {
    extern __shared__ __align__(16) float fsm[];
    const int b = p.b;
    float* sq = fsm;              // [b][D]
    float* sk = sq + b * D;       // [b][D]
    float* sv = sk + b * D;       // [b][D]
    const int i = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int c = p.cls[h];
    const int64_t g = static_cast<int64_t>(s) * 3 + c;
    const bool implicit = c == 0 && p.local_implicit;
    const int64_t head_off = (static_cast<int64_t>(s) * p.H + h) * p.L;
    const int r = threadIdx.x;
    const int64_t row0 = head_off + static_cast<int64_t>(i) * b;

    for (int e = threadIdx.x; e < b * D; e += blockDim.x) sq[e] = p.q[row0 * D + e];

    float acc[D];
#pragma unroll
    for (int e = 0; e < D; ++e) acc[e] = 0.f;
    float m = -INFINITY, l = 0.f;

    // key blocks of query block i: the stored row, or the implicit local window
    const int32_t* rp = p.row_ptr + g * (p.nblk + 1);
    const int32_t* ci = p.col_idx + g * p.cap;
    const int beg = implicit ? (i - p.w > 0 ? i - p.w : 0) : rp[i];
    const int end = implicit ? i + 1 : rp[i + 1];
    for (int e = beg; e < end; ++e) {
        const int j = implicit ? e : ci[e];
        const int64_t krow = head_off + static_cast<int64_t>(j) * b;
        __syncthreads();
        for (int x = threadIdx.x; x < b * D; x += blockDim.x) {
            sk[x] = p.k[krow * D + x];
            sv[x] = p.v[krow * D + x];
        }
        __syncthreads();
        if (r < b) {
            const int last = (j == i) ? r : b - 1;   // causal inside the diagonal block
            float bm = -INFINITY;
            for (int u = 0; u <= last; ++u) {
                float dot = 0.f;
#pragma unroll
                for (int e2 = 0; e2 < D; ++e2) dot = fmaf(sq[r * D + e2], sk[u * D + e2], dot);
                bm = fmaxf(bm, dot * p.scale);
            }
            const float mn = fmaxf(m, bm);
            const float alpha = expf(m - mn);   // 0 when m = -inf
            l *= alpha;
#pragma unroll
            for (int e2 = 0; e2 < D; ++e2) acc[e2] *= alpha;
            for (int u = 0; u <= last; ++u) {
                float dot = 0.f;
#pragma unroll
                for (int e2 = 0; e2 < D; ++e2) dot = fmaf(sq[r * D + e2], sk[u * D + e2], dot);
                const float pu = expf(dot * p.scale - mn);
                l += pu;
#pragma unroll
                for (int e2 = 0; e2 < D; ++e2) acc[e2] = fmaf(pu, sv[u * D + e2], acc[e2]);
            }
            m = mn;
        }
    }
    if (r < b) {
        const float inv = 1.f / l;
        float* out = p.o + (row0 + r) * D;
#pragma unroll
        for (int e2 = 0; e2 < D; ++e2) out[e2] = acc[e2] * inv;
        if (p.lse) p.lse[row0 + r] = m + logf(l);
    }
}

}  // namespace f32
}  // namespace gsa
