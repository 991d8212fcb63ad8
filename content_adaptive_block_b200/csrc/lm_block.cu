// One ByteLM transformer block, forward and backward, around the block-sparse
// attention of gsa.cu.
//
// The pages train a byte-level LM with the adaptive mask (Gzip-guided Sparse
// Attention, daiwk.github.io: fidelity line and section "论文离线与线上效果",
// 92M parameters at 8K bytes; the arXiv abstract, same model) but give no
// block layout.  This file takes the plainest one: byte embedding, pre-LN
// residual block x1 = x0 + Attn(LN1 x0) W_o^T, y = x1 + GELU(LN2 x1 W_1^T) W_2^T,
// LayerNorm with gain and bias, linear layers without bias, tanh-form GELU.
//
// Hand-written kernels here: the embedding gather fused with LN1, LayerNorm
// forward and backward (with deterministic column sums for the gain and bias
// gradients) and the embedding gradient (a deterministic per-byte
// reduction).  The attention is gsa_attn_fwd / gsa_attn_bwd, reading Q, K, V
// straight out of the QKV projection's [token][3][head][64] rows and writing
// O, dQ, dK, dV in the projections' layouts (gsa_attn_layout), so no head
// transposes run.  The
// projections are bf16 GEMMs with float32 accumulation on this library's
// tcgen05 GEMM (gemm.cuh), the residual additions folded into them
// (D = A B + C) and the GELU and its derivative into their epilogues.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>
#include <utility>

#include "gemm_api.h"
#include "gsa.h"
#include "gsa_lm.h"
#include "host_attr.h"

namespace gsa {
namespace lm {

using bf16 = __nv_bfloat16;

constexpr int kLnWarps = 8;        // rows per CTA step in the LayerNorm kernels
constexpr int kLnParts = 296;      // CTAs of the LayerNorm backward (2 per SM; partial column sums)

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void load8(const bf16* p, float* v) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
        const float2 f = __bfloat1622float2(h);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ void load8f(const float* p, float* v) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void store8(bf16* p, const float* v) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// ---------------------------------------------------------------- LayerNorm
// One warp per token row of D = 256 NC features; lane l holds the features
// 256 j + 8 l .. 256 j + 8 l + 7 (16-byte loads).  Two-pass statistics in
// float32 from the row in registers.  GATHER: the row is emb[bytes[t]] and is
// also written out (x0, the residual stream).
template <int NC, bool GATHER>
__global__ void __launch_bounds__(32 * kLnWarps)
ln_fwd_kernel(const uint8_t* __restrict__ bytes, const bf16* __restrict__ src, const float* __restrict__ g,
              const float* __restrict__ bb, bf16* __restrict__ xcopy, bf16* __restrict__ y,
              float2* __restrict__ stats, int64_t T, float eps) {
    constexpr int D = 256 * NC;
    const int lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kLnWarps + (threadIdx.x >> 5);
    if (t >= T) return;
    const int64_t srow = GATHER ? static_cast<int64_t>(bytes[t]) : t;
    float v[NC * 8];
#pragma unroll
    for (int j = 0; j < NC; ++j) load8(src + srow * D + 256 * j + 8 * lane, v + 8 * j);
    if (GATHER) {
#pragma unroll
        for (int j = 0; j < NC; ++j) store8(xcopy + t * D + 256 * j + 8 * lane, v + 8 * j);
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < NC * 8; ++i) s += v[i];
    const float mean = warp_sum(s) * (1.f / D);
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < NC * 8; ++i) q += (v[i] - mean) * (v[i] - mean);
    const float rstd = rsqrtf(warp_sum(q) * (1.f / D) + eps);
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        float o[8], gg[8], bv[8];
        load8f(g + 256 * j + 8 * lane, gg);
        load8f(bb + 256 * j + 8 * lane, bv);
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = (v[8 * j + e] - mean) * rstd * gg[e] + bv[e];
        store8(y + t * D + 256 * j + 8 * lane, o);
    }
    if (lane == 0) stats[t] = make_float2(mean, rstd);
}

// dx = rstd (g dy - mean(g dy) - xhat mean(g dy xhat)) + dres, with the
// gain / bias gradient sums of this CTA's rows (a contiguous range) written
// to part[cta][0 / 1][D].  Each warp keeps its running sums in its own
// shared-memory rows (lane-contiguous, no bank conflicts), which keeps the
// registers low enough for two CTAs per SM; the warps' sums are added in
// warp order at the end.
template <int NC>
__global__ void __launch_bounds__(32 * kLnWarps)
ln_bwd_kernel(const bf16* __restrict__ dy, const bf16* __restrict__ x, const float2* __restrict__ stats,
              const float* __restrict__ g, const bf16* __restrict__ dres, bf16* __restrict__ dx,
              float* __restrict__ part, int64_t T, int64_t rows_per_cta) {
    constexpr int D = 256 * NC;
    extern __shared__ float ln_smem[];
    float* acc = ln_smem + (threadIdx.x >> 5) * 2 * D;   // this warp's [2][D]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int c = lane; c < 2 * D; c += 32) acc[c] = 0.f;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per_cta;
    const int64_t r1 = r0 + rows_per_cta < T ? r0 + rows_per_cta : T;
    for (int64_t t = r0 + warp; t < r1; t += kLnWarps) {
        float xv[NC * 8], dv[NC * 8];
#pragma unroll
        for (int j = 0; j < NC; ++j) {
            load8(x + t * D + 256 * j + 8 * lane, xv + 8 * j);
            load8(dy + t * D + 256 * j + 8 * lane, dv + 8 * j);
        }
        const float2 st = stats[t];
        float s1 = 0.f, s2 = 0.f;
#pragma unroll
        for (int j = 0; j < NC; ++j) {
            float gv[8];
            load8f(g + 256 * j + 8 * lane, gv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int i = 8 * j + e, c = 256 * j + 8 * lane + e;
                xv[i] = (xv[i] - st.x) * st.y;   // xhat
                const float gd = gv[e] * dv[i];
                s1 += gd;
                s2 += gd * xv[i];
                acc[c] += dv[i] * xv[i];
                acc[D + c] += dv[i];
            }
        }
        const float m1 = warp_sum(s1) * (1.f / D), m2 = warp_sum(s2) * (1.f / D);
#pragma unroll
        for (int j = 0; j < NC; ++j) {
            float o[8], rv[8], gv[8];
            load8f(g + 256 * j + 8 * lane, gv);
            if (dres) load8(dres + t * D + 256 * j + 8 * lane, rv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int i = 8 * j + e;
                o[e] = st.y * (gv[e] * dv[i] - m1 - xv[i] * m2) + (dres ? rv[e] : 0.f);
            }
            store8(dx + t * D + 256 * j + 8 * lane, o);
        }
    }
    __syncthreads();
    // the warps' sums in warp order
    for (int c = threadIdx.x; c < 2 * D; c += blockDim.x) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kLnWarps; ++w) s += ln_smem[w * 2 * D + c];
        part[static_cast<int64_t>(blockIdx.x) * 2 * D + c] = s;
    }
}

// dg[c] = sum_p part[p][0][c], db[c] = sum_p part[p][1][c] in a fixed order:
// CTA of 8 warps per 32 of the 2D columns; warp w sums the parts p = w mod 8
// ascending, then the eight warp sums are added in warp order.
__global__ void __launch_bounds__(256)
colsum_kernel(const float* __restrict__ part, int nparts, int D, float* __restrict__ dg, float* __restrict__ db) {
    __shared__ float ws[8][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c = blockIdx.x * 32 + lane;
    float s = 0.f;
    if (c < 2 * D)
        for (int p = warp; p < nparts; p += 8) s += part[static_cast<int64_t>(p) * 2 * D + c];
    ws[warp][lane] = s;
    __syncthreads();
    if (warp == 0 && c < 2 * D) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += ws[w][lane];
        if (c < D) dg[c] = t;
        else db[c - D] = t;
    }
}

// ------------------------------------------------------ embedding gradient
// dE[v][c] = sum over tokens t with bytes[t] == v of dx0[t][c], in a fixed
// order: CTA (chunk of kEmbChunk tokens, slice of 32 columns) has two warps,
// each walking its half of the chunk in order, lane = column, adding each
// row into its own shared-memory table [256][32] (the lane's own bank);
// the CTA then writes table 0 + table 1 as the chunk's partial, and
// embed_reduce_kernel sums the partials of each (v, c) in chunk order.
constexpr int kEmbChunk = 1024;
constexpr int kEmbCols = 32;
constexpr int kEmbWarps = 2;
constexpr int kEmbSmem = kEmbWarps * 256 * kEmbCols * 4;

__global__ void __launch_bounds__(32 * kEmbWarps)
embed_part_kernel(const uint8_t* __restrict__ bytes, const bf16* __restrict__ dx0, int64_t T, int D,
                  float* __restrict__ part) {
    extern __shared__ float emb_smem[];
    auto acc = reinterpret_cast<float (*)[256][kEmbCols]>(emb_smem);   // [kEmbWarps][256][kEmbCols]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c = blockIdx.y * kEmbCols + lane;
    for (int v = 0; v < 256; ++v) acc[warp][v][lane] = 0.f;
    __syncwarp();
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kEmbChunk + warp * (kEmbChunk / kEmbWarps);
    const int64_t t1 = t0 + kEmbChunk / kEmbWarps < T ? t0 + kEmbChunk / kEmbWarps : T;
    for (int64_t tb = t0; tb < t1; tb += 32) {
        // 32 rows' loads in flight before the table updates
        const int n = t1 - tb < 32 ? static_cast<int>(t1 - tb) : 32;
        const int mine = lane < n ? bytes[tb + lane] : 0;
        const bf16* row = dx0 + tb * D + c;
        float x[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) x[k] = k < n ? __bfloat162float(row[static_cast<int64_t>(k) * D]) : 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const int v = __shfl_sync(0xffffffffu, mine, k);
            if (k < n) acc[warp][v][lane] += x[k];
        }
    }
    __syncthreads();
    float* out = part + static_cast<int64_t>(blockIdx.x) * 256 * D + blockIdx.y * kEmbCols;
    for (int e = threadIdx.x; e < 256 * kEmbCols; e += 32 * kEmbWarps) {
        const int v = e / kEmbCols, cc = e % kEmbCols;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kEmbWarps; ++w) s += acc[w][v][cc];
        out[static_cast<int64_t>(v) * D + cc] = s;
    }
}

__global__ void embed_reduce_kernel(const float* __restrict__ part, int nchunks, int D, float* __restrict__ dE) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t n = 256 * static_cast<int64_t>(D);
    if (i >= n) return;
    float s = 0.f;
    for (int k = 0; k < nchunks; ++k) s += part[k * n + i];
    dE[i] = s;
}

// ------------------------------------------------------------- projections
// Row-major D[M][N] = op(A)[M][K] op(B)[K][N] + beta C on this library's
// tcgen05 GEMM (gemm.cuh): bf16 operands, float32 accumulation; C and D bf16
// (residual folded in) or float32 (weight gradients, beta 0).  ta: A is
// stored [K][M]; tb: B is stored [N][K].  Epilogues on the float32
// accumulator (tanh-form GELU):
//   kEpiGeluAux: D = GELU(A B), aux = A B (bf16, row-major, ld aux_ld);
//   kEpiDGelu:   D = (A B) * GELU'(aux).
// ws / ws_bytes: float32 scratch for the K-split weight gradients.
enum Epi { kEpiNone = 0, kEpiGeluAux = 1, kEpiDGelu = 2 };

struct GemmWs {
    float* p;
    size_t bytes;
};

gsa_status gemm_rm(bool ta, bool tb, int M, int N, int K, const bf16* A, int lda, const bf16* B, int ldb,
                   float beta, const void* C, int ldc, void* Dp, int ldd, bool out32, GemmWs ws, cudaStream_t st,
                   Epi epi = kEpiNone, void* aux = nullptr, int64_t aux_ld = 0) {
    const gsa::gemm::Epi e = epi == kEpiGeluAux ? gsa::gemm::kGeluAux : (epi == kEpiDGelu ? gsa::gemm::kDGelu
                                                                                          : gsa::gemm::kNone);
    return gsa::gemm::run(ta, tb, M, N, K, A, lda, B, ldb, beta, static_cast<const bf16*>(C), ldc, Dp, ldd, out32, e,
                          static_cast<bf16*>(aux), aux_ld, ws.p, ws.bytes, st);
}

// Split scratch of the block's weight-gradient products (K = B L tokens).
size_t gemm_ws_bytes(const gsa_lm_desc* d) {
    const int T = d->B * d->L, D = d->D, F = d->F;
    size_t m = 0;
    for (const auto& mn : {std::make_pair(D, F), std::make_pair(F, D), std::make_pair(D, D), std::make_pair(3 * D, D)}) {
        const size_t b = gsa::gemm::split_ws_bytes(mn.first, mn.second, T);
        if (b > m) m = b;
    }
    return m;
}

// ------------------------------------------------------------ workspace
struct Layout {
    size_t x0, h, st1, qkv, lse, om, x1, h2, st2, pre, act;       // saved by the forward
    size_t dpre, dh2, dx1, dom, dqkv, dh, dx0, part, epart, attn_ws;   // backward scratch
    size_t lt, lt_bytes, total;
    size_t attn_ws_bytes;
};

inline size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

Layout layout(const gsa_lm_desc* d, const gsa_attn_desc& ad) {
    const size_t T = static_cast<size_t>(d->B) * d->L;
    const size_t TD = T * d->D * 2, TF = T * d->F * 2;
    Layout l;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = up256(off + bytes);
        return at;
    };
    l.x0 = take(TD);
    l.h = take(TD);
    l.st1 = take(T * 8);
    l.qkv = take(3 * TD);
    l.lse = take(T * d->H * 4);
    l.om = take(TD);
    l.x1 = take(TD);
    l.h2 = take(TD);
    l.st2 = take(T * 8);
    l.pre = take(TF);
    l.act = take(TF);
    l.dpre = take(TF);
    l.dh2 = take(TD);
    l.dx1 = take(TD);
    l.dom = take(TD);
    l.dqkv = take(3 * TD);
    l.dh = take(TD);
    l.dx0 = take(TD);
    l.part = take(static_cast<size_t>(kLnParts) * 2 * d->D * 4);
    l.epart = take((T + kEmbChunk - 1) / kEmbChunk * 256 * d->D * 4);
    l.attn_ws_bytes = gsa_attn_bwd_workspace(&ad);
    l.attn_ws = take(l.attn_ws_bytes);
    l.lt_bytes = gemm_ws_bytes(d);
    l.lt = take(l.lt_bytes);
    l.total = off;
    return l;
}

// Q, K, V (and dQ, dK, dV) inside [T][3][H][64] rows; O and dO inside [T][H][64] rows.
gsa_attn_layout attn_layout(const gsa_lm_desc* d) {
    const int64_t D = d->D, L = d->L;
    return gsa_attn_layout{3 * D * L, 64, 3 * D, D * L, 64, D};
}

gsa_status check(const gsa_lm_desc* d, gsa_attn_desc* ad) {
    if (!d || d->B < 1 || d->L < 1 || d->H < 1 || d->H > GSA_MAX_HEADS || !d->head_classes || d->b != 64 ||
        d->L % d->b != 0 || d->D != 64 * d->H || d->F < 8 || d->F % 8 != 0 || !(d->ln_eps > 0.f))
        return GSA_ERR_INVALID_ARGUMENT;
    // the GEMM tiles 256 output columns and 64-wide K slices
    if (d->D % 256 != 0 || d->D > 2048 || d->F % 256 != 0 || d->L / d->b > GSA_MAX_BLOCKS_BF16)
        return GSA_ERR_UNSUPPORTED;
    for (int h = 0; h < d->H; ++h)
        if (d->head_classes[h] > 2) return GSA_ERR_INVALID_ARGUMENT;
    ad->B = d->B;
    ad->H = d->H;
    ad->L = d->L;
    ad->d = 64;
    ad->b = d->b;
    ad->dtype = GSA_BF16;
    ad->scale = 0.f;
    ad->head_classes = d->head_classes;
    ad->layout = nullptr;   // the calls point it at their own layout
    return GSA_OK;
}

inline bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline gsa_status last_launch() { return cudaGetLastError() == cudaSuccess ? GSA_OK : GSA_ERR_CUDA; }

template <int NC>
void ln_fwd_launch(bool gather, const uint8_t* bytes, const bf16* src, const float* g, const float* b, bf16* xcopy,
                   bf16* y, float2* stats, int64_t T, float eps, cudaStream_t st) {
    const unsigned grid = static_cast<unsigned>((T + kLnWarps - 1) / kLnWarps);
    if (gather) ln_fwd_kernel<NC, true><<<grid, 32 * kLnWarps, 0, st>>>(bytes, src, g, b, xcopy, y, stats, T, eps);
    else ln_fwd_kernel<NC, false><<<grid, 32 * kLnWarps, 0, st>>>(bytes, src, g, b, xcopy, y, stats, T, eps);
}

void ln_fwd(int D, bool gather, const uint8_t* bytes, const bf16* src, const float* g, const float* b, bf16* xcopy,
            bf16* y, float2* stats, int64_t T, float eps, cudaStream_t st) {
    switch (D / 256) {
        case 1: ln_fwd_launch<1>(gather, bytes, src, g, b, xcopy, y, stats, T, eps, st); break;
        case 2: ln_fwd_launch<2>(gather, bytes, src, g, b, xcopy, y, stats, T, eps, st); break;
        case 3: ln_fwd_launch<3>(gather, bytes, src, g, b, xcopy, y, stats, T, eps, st); break;
        case 4: ln_fwd_launch<4>(gather, bytes, src, g, b, xcopy, y, stats, T, eps, st); break;
        case 5: ln_fwd_launch<5>(gather, bytes, src, g, b, xcopy, y, stats, T, eps, st); break;
        case 6: ln_fwd_launch<6>(gather, bytes, src, g, b, xcopy, y, stats, T, eps, st); break;
        case 7: ln_fwd_launch<7>(gather, bytes, src, g, b, xcopy, y, stats, T, eps, st); break;
        default: ln_fwd_launch<8>(gather, bytes, src, g, b, xcopy, y, stats, T, eps, st); break;
    }
}

template <int NC>
bool ln_bwd_launch(const bf16* dy, const bf16* x, const float2* stats, const float* g, const bf16* dres, bf16* dx,
                   float* part, int64_t T, cudaStream_t st) {
    constexpr int kSmem = kLnWarps * 2 * 256 * NC * 4;
    if (!gsa::smem_opt_in(ln_bwd_kernel<NC>, kSmem)) return false;
    const int64_t rpc = (T + kLnParts - 1) / kLnParts;
    ln_bwd_kernel<NC><<<kLnParts, 32 * kLnWarps, kSmem, st>>>(dy, x, stats, g, dres, dx, part, T, rpc);
    return true;
}

// False when the kernel could not be opted in to its shared memory (nothing launched).
bool ln_bwd(int D, const bf16* dy, const bf16* x, const float2* stats, const float* g, const bf16* dres, bf16* dx,
            float* part, float* dg, float* db, int64_t T, cudaStream_t st) {
    bool ok = false;
    switch (D / 256) {
        case 1: ok = ln_bwd_launch<1>(dy, x, stats, g, dres, dx, part, T, st); break;
        case 2: ok = ln_bwd_launch<2>(dy, x, stats, g, dres, dx, part, T, st); break;
        case 3: ok = ln_bwd_launch<3>(dy, x, stats, g, dres, dx, part, T, st); break;
        case 4: ok = ln_bwd_launch<4>(dy, x, stats, g, dres, dx, part, T, st); break;
        case 5: ok = ln_bwd_launch<5>(dy, x, stats, g, dres, dx, part, T, st); break;
        case 6: ok = ln_bwd_launch<6>(dy, x, stats, g, dres, dx, part, T, st); break;
        case 7: ok = ln_bwd_launch<7>(dy, x, stats, g, dres, dx, part, T, st); break;
        default: ok = ln_bwd_launch<8>(dy, x, stats, g, dres, dx, part, T, st); break;
    }
    if (!ok) return false;
    colsum_kernel<<<(2 * D + 31) / 32, 256, 0, st>>>(part, kLnParts, D, dg, db);
    return true;
}

}  // namespace lm
}  // namespace gsa

// ------------------------------------------------------------- the calls
using namespace gsa::lm;

extern "C" {

gsa_status gsa_lm_gemm(int32_t ta, int32_t tb, int32_t M, int32_t N, int32_t K, const void* A, int64_t lda,
                       const void* B, int64_t ldb, float beta, const void* C, int64_t ldc, void* D, int64_t ldd,
                       int32_t out32, int32_t epi, void* aux, int64_t aux_ld, void* workspace, size_t ws_bytes,
                       void* stream) {
    const gsa::CallRange nvtx_range("gsa_lm_gemm");
    if (epi < 0 || epi > 2) return GSA_ERR_INVALID_ARGUMENT;
    return gsa::gemm::run(ta != 0, tb != 0, M, N, K, static_cast<const bf16*>(A), lda, static_cast<const bf16*>(B),
                          ldb, beta, static_cast<const bf16*>(C), ldc, D, ldd, out32 != 0,
                          static_cast<gsa::gemm::Epi>(epi), static_cast<bf16*>(aux), aux_ld,
                          static_cast<float*>(workspace), ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t gsa_lm_gemm_workspace(int32_t M, int32_t N, int32_t K, int32_t out32) {
    if (M < 1 || N < 1 || K < 1 || !out32) return 0;
    return gsa::gemm::split_ws_bytes(M, N, K);
}

size_t gsa_lm_block_workspace(const gsa_lm_desc* desc) {
    gsa_attn_desc ad;
    if (check(desc, &ad) != GSA_OK) return 0;
    return layout(desc, ad).total;
}

#define GSA_TRY(x)                         \
    do {                                   \
        const gsa_status s_ = (x);         \
        if (s_ != GSA_OK) return s_;       \
    } while (0)

gsa_status gsa_lm_block_fwd(const uint8_t* bytes, const gsa_lm_weights* w, const gsa_block_csr* csr,
                            const gsa_lm_desc* desc, void* y, void* workspace, size_t ws_bytes, void* stream) {
    const gsa::CallRange nvtx_range("gsa_lm_block_fwd");
    gsa_attn_desc ad;
    GSA_TRY(check(desc, &ad));
    if (!bytes || !w || !csr || !y || !workspace || !w->emb || !w->ln1_g || !w->ln1_b || !w->w_qkv || !w->w_o ||
        !w->ln2_g || !w->ln2_b || !w->w_1 || !w->w_2)
        return GSA_ERR_INVALID_ARGUMENT;
    if (!a16(y) || !a16(workspace) || !a16(w->emb) || !a16(w->ln1_g) || !a16(w->ln1_b) || !a16(w->w_qkv) ||
        !a16(w->w_o) || !a16(w->ln2_g) || !a16(w->ln2_b) || !a16(w->w_1) || !a16(w->w_2))
        return GSA_ERR_INVALID_ARGUMENT;
    const Layout l = layout(desc, ad);
    if (ws_bytes < l.total) return GSA_ERR_CAPACITY;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    auto P = [&](size_t off) { return reinterpret_cast<bf16*>(ws + off); };
    const int64_t T = static_cast<int64_t>(desc->B) * desc->L;
    const int D = desc->D, F = desc->F, Mi = static_cast<int>(T);
    if (T > 0x7fffffff) return GSA_ERR_UNSUPPORTED;
    const auto* emb = static_cast<const bf16*>(w->emb);
    const GemmWs lt{reinterpret_cast<float*>(ws + l.lt), l.lt_bytes};

    // x0 = E[bytes], h = LN1(x0)
    ln_fwd(D, true, bytes, emb, w->ln1_g, w->ln1_b, P(l.x0), P(l.h), reinterpret_cast<float2*>(ws + l.st1), T,
           desc->ln_eps, st);
    GSA_TRY(last_launch());
    // qkv = h W_qkv^T; the attention reads Q, K, V from its rows and writes O as W_o's input rows
    GSA_TRY(gemm_rm(false, true, Mi, 3 * D, D, P(l.h), D, static_cast<const bf16*>(w->w_qkv), D, 0.f, nullptr,
                    3 * D, P(l.qkv), 3 * D, false, lt, st));
    const gsa_attn_layout al = attn_layout(desc);
    ad.layout = &al;
    GSA_TRY(gsa_attn_fwd(P(l.qkv), P(l.qkv) + D, P(l.qkv) + 2 * D, csr, &ad, P(l.om),
                         reinterpret_cast<float*>(ws + l.lse), stream));
    // x1 = x0 + O W_o^T, h2 = LN2(x1)
    GSA_TRY(gemm_rm(false, true, Mi, D, D, P(l.om), D, static_cast<const bf16*>(w->w_o), D, 1.f, P(l.x0), D,
                    P(l.x1), D, false, lt, st));
    ln_fwd(D, false, nullptr, P(l.x1), w->ln2_g, w->ln2_b, nullptr, P(l.h2), reinterpret_cast<float2*>(ws + l.st2),
           T, desc->ln_eps, st);
    GSA_TRY(last_launch());
    // y = x1 + GELU(h2 W_1^T) W_2^T
    GSA_TRY(gemm_rm(false, true, Mi, F, D, P(l.h2), D, static_cast<const bf16*>(w->w_1), D, 0.f, nullptr, F,
                    P(l.act), F, false, lt, st, kEpiGeluAux, P(l.pre), F));
    return gemm_rm(false, true, Mi, D, F, P(l.act), F, static_cast<const bf16*>(w->w_2), F, 1.f, P(l.x1), D, y, D,
                   false, lt, st);
}

gsa_status gsa_lm_block_bwd(const uint8_t* bytes, const gsa_lm_weights* w, const gsa_block_csr* csr,
                            const gsa_lm_desc* desc, const void* dy, const gsa_lm_grads* g, void* workspace,
                            size_t ws_bytes, void* stream) {
    const gsa::CallRange nvtx_range("gsa_lm_block_bwd");
    gsa_attn_desc ad;
    GSA_TRY(check(desc, &ad));
    if (!bytes || !w || !csr || !dy || !g || !workspace || !w->emb || !w->ln1_g || !w->w_qkv || !w->w_o ||
        !w->ln2_g || !w->w_1 || !w->w_2 || !g->emb || !g->ln1_g || !g->ln1_b || !g->w_qkv || !g->w_o || !g->ln2_g ||
        !g->ln2_b || !g->w_1 || !g->w_2)
        return GSA_ERR_INVALID_ARGUMENT;
    if (!a16(dy) || !a16(workspace) || !a16(w->emb) || !a16(w->ln1_g) || !a16(w->w_qkv) || !a16(w->w_o) ||
        !a16(w->ln2_g) || !a16(w->w_1) || !a16(w->w_2) || !a16(g->emb) || !a16(g->ln1_g) || !a16(g->ln1_b) ||
        !a16(g->w_qkv) || !a16(g->w_o) || !a16(g->ln2_g) || !a16(g->ln2_b) || !a16(g->w_1) || !a16(g->w_2))
        return GSA_ERR_INVALID_ARGUMENT;
    const Layout l = layout(desc, ad);
    if (ws_bytes < l.total) return GSA_ERR_CAPACITY;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    auto P = [&](size_t off) { return reinterpret_cast<bf16*>(ws + off); };
    const int64_t T = static_cast<int64_t>(desc->B) * desc->L;
    const int D = desc->D, F = desc->F, Mi = static_cast<int>(T);
    if (T > 0x7fffffff) return GSA_ERR_UNSUPPORTED;
    const auto* dyb = static_cast<const bf16*>(dy);
    const GemmWs lt{reinterpret_cast<float*>(ws + l.lt), l.lt_bytes};
    float* part = reinterpret_cast<float*>(ws + l.part);

    // MLP: dpre = (dy W_2) GELU'(pre) (one GEMM with its epilogue), dW_2 = dy^T act, dW_1 = dpre^T h2,
    // dh2 = dpre W_1
    GSA_TRY(gemm_rm(false, false, Mi, F, D, dyb, D, static_cast<const bf16*>(w->w_2), F, 0.f, nullptr, F, P(l.dpre),
                    F, false, lt, st, kEpiDGelu, P(l.pre), F));
    GSA_TRY(gemm_rm(true, false, D, F, Mi, dyb, D, P(l.act), F, 0.f, nullptr, F, g->w_2, F, true, lt, st));
    GSA_TRY(gemm_rm(true, false, F, D, Mi, P(l.dpre), F, P(l.h2), D, 0.f, nullptr, D, g->w_1, D, true, lt, st));
    GSA_TRY(gemm_rm(false, false, Mi, D, F, P(l.dpre), F, static_cast<const bf16*>(w->w_1), D, 0.f, nullptr, D,
                    P(l.dh2), D, false, lt, st));
    // dx1 = dy + LN2'(dh2)
    if (!ln_bwd(D, P(l.dh2), P(l.x1), reinterpret_cast<const float2*>(ws + l.st2), w->ln2_g, dyb, P(l.dx1), part,
                g->ln2_g, g->ln2_b, T, st))
        return GSA_ERR_CUDA;
    GSA_TRY(last_launch());
    // attention: dO = dx1 W_o, dW_o = dx1^T O, then the attention's own backward (dQ, dK, dV as dqkv rows)
    GSA_TRY(gemm_rm(false, false, Mi, D, D, P(l.dx1), D, static_cast<const bf16*>(w->w_o), D, 0.f, nullptr, D,
                    P(l.dom), D, false, lt, st));
    GSA_TRY(gemm_rm(true, false, D, D, Mi, P(l.dx1), D, P(l.om), D, 0.f, nullptr, D, g->w_o, D, true, lt, st));
    const gsa_attn_layout al = attn_layout(desc);
    ad.layout = &al;
    GSA_TRY(gsa_attn_bwd(P(l.qkv), P(l.qkv) + D, P(l.qkv) + 2 * D, P(l.om), reinterpret_cast<const float*>(ws + l.lse),
                         P(l.dom), csr, &ad, P(l.dqkv), P(l.dqkv) + D, P(l.dqkv) + 2 * D, ws + l.attn_ws,
                         l.attn_ws_bytes, stream));
    // dW_qkv = dqkv^T h, dh = dqkv W_qkv, dx0 = dx1 + LN1'(dh)
    GSA_TRY(gemm_rm(true, false, 3 * D, D, Mi, P(l.dqkv), 3 * D, P(l.h), D, 0.f, nullptr, D, g->w_qkv, D, true, lt,
                    st));
    GSA_TRY(gemm_rm(false, false, Mi, D, 3 * D, P(l.dqkv), 3 * D, static_cast<const bf16*>(w->w_qkv), D, 0.f,
                    nullptr, D, P(l.dh), D, false, lt, st));
    if (!ln_bwd(D, P(l.dh), P(l.x0), reinterpret_cast<const float2*>(ws + l.st1), w->ln1_g, P(l.dx1), P(l.dx0),
                part, g->ln1_g, g->ln1_b, T, st))
        return GSA_ERR_CUDA;
    GSA_TRY(last_launch());
    // dE: per byte value, the sum of its tokens' dx0 rows
    const int nchunks = static_cast<int>((T + kEmbChunk - 1) / kEmbChunk);
    float* epart = reinterpret_cast<float*>(ws + l.epart);
    if (!gsa::smem_opt_in(embed_part_kernel, kEmbSmem)) return GSA_ERR_CUDA;
    embed_part_kernel<<<dim3(nchunks, D / kEmbCols), 32 * kEmbWarps, kEmbSmem, st>>>(bytes, P(l.dx0), T, D,
                                                                                      epart);
    embed_reduce_kernel<<<(256 * D + 255) / 256, 256, 0, st>>>(epart, nchunks, D, g->emb);
    return last_launch();
}

}  // extern "C"
