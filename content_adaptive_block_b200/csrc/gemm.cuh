// Dense bf16 GEMM on the 5th-generation tensor cores, for the ByteLM block's
// projections and weight gradients (the block of section
// "论文离线与线上效果": a 92M-parameter byte-level model at 8K bytes; its
// layout is this library's reading, see lm_block.cu).
//
// Row-major D[M][N] = op(A)[M][K] op(B)[K][N] with float32 accumulation in
// TMEM.  One persistent CTA per SM walks 128 x 256 output tiles (N fastest,
// so the CTAs in flight share rows of A in L2), optionally with K split in
// parts whose float32 partial tiles a second kernel sums in a fixed order
// (deterministic).  Roles:
//   warp 0      TMA producer: 64-wide K slices of A (128 rows) and B (256
//               rows) into a 4-stage ring, 128-byte swizzled; an operand
//               stored with M (or N) contiguous arrives as 64-column boxes
//               side by side (the MN-major UMMA layout);
//   warp 1      TMEM owner and MMA issuer: per slice four
//               tcgen05.mma.kind::f16 (M 128, N 256, K 16) into one of two
//               accumulators, so one tile's epilogue overlaps the next tile's
//               products;
//   warps 2-9   epilogue, two warpgroups: one output row per thread (its
//               TMEM lane), 64 (or 32 float32) columns at a time, each
//               warpgroup half of them: the epilogue arithmetic (C or the
//               GELU input of the next chunk already loaded), then into a
//               128-byte swizzled staging box that one thread stores with TMA.
// Every wait is bounded: on a timeout the CTA records an error code, drains
// what it issued and leaves.
#pragma once

#include "common.cuh"
#include "gemm_api.h"

namespace gsa {
namespace gemm {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK * 2;               // 16 KB
constexpr int kBBytes = BN * BK * 2;               // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;     // 48 KB
constexpr int kBoxBytes = 128 * 128;               // a staging box: 128 rows x 128 bytes
constexpr int kOffStage = 0;
constexpr int kOffOut = kOffStage + kStages * kStageBytes;   // D staging box
constexpr int kOffAux = kOffOut + kBoxBytes;                 // aux staging box
constexpr int kOffBar = kOffAux + kBoxBytes;
// full[st], empty[st], acc_full[2], acc_empty[2], drain
constexpr int kNumBars = 2 * kStages + 5;
constexpr int kOffMisc = kOffBar + kNumBars * 8;             // tmem base, abort
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
constexpr int kThreads = 320;
constexpr int kEpiThreads = 256;

struct Params {
    int M, N, K;
    int tiles_m, tiles_n, splits, kslices;   // kslices: BK-slices per split
    int ta, tb, out32, epi;
    float beta;
    const __nv_bfloat16* C;
    int64_t ldc;
    const __nv_bfloat16* aux_in;             // kDGelu
    int64_t aux_ld;
    int split_out;                           // write split partials to ws (float32 [splits][M][N])
    float* ws;
};

// Instruction descriptor, kind::f16, bf16 A and B, float32 D, A and B K- or
// MN-major.
__host__ __device__ constexpr uint32_t idesc_gemm(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
           (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// the four epilogue warps only
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory"); }

// GELU, tanh form, and its derivative, with the hardware tanh approximation
// (tanh.approx.f32: relative error about 2^-11, below the bf16 rounding of
// the results).
__device__ __forceinline__ float tanh_fast(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float gelu_tanh(float x) {
    const float k0 = 0.7978845608028654f, k1 = 0.044715f;
    return 0.5f * x * (1.f + tanh_fast(k0 * (x + k1 * x * x * x)));
}
__device__ __forceinline__ float gelu_tanh_grad(float x) {
    const float k0 = 0.7978845608028654f, k1 = 0.044715f;
    const float t = tanh_fast(k0 * (x + k1 * x * x * x));
    return 0.5f * (1.f + t) + 0.5f * x * (1.f - t * t) * k0 * (1.f + 3.f * k1 * x * x);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmAux, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;
    uint64_t* acc_full = bars + 2 * kStages;    // [buf]: the tile's last products completed
    uint64_t* acc_empty = acc_full + 2;         // [buf]: its epilogue read the accumulator (128 arrivals)
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = p.tiles_m * p.tiles_n * p.splits;

    if (threadIdx.x == 0) {
        for (int st = 0; st < kStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiThreads);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmD);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // tile t: split t / (tiles_m tiles_n), then row block, then column block (fastest)
    auto tile_of = [&](int t, int& mb, int& nb, int& ks) {
        const int per = p.tiles_m * p.tiles_n;
        ks = t / per;
        const int r = t - ks * per;
        mb = r / p.tiles_n;
        nb = r - mb * p.tiles_n;
    };

    int issued = 0;   // producer: slices loaded (lane 0)
    if (warp == 0) {
        if (lane == 0) {
            bool ok = true;
            for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
                int mb, nb, ks;
                tile_of(t, mb, nb, ks);
                const int m0 = mb * BM, n0 = nb * BN;
                for (int s = 0; s < p.kslices; ++s, ++issued) {
                    const int st = issued % kStages;
                    if (issued >= kStages &&
                        !mbar_wait(&empty[st], ((issued / kStages) - 1) & 1, abort_flag, kErrTimeoutProducer)) {
                        ok = false;
                        break;
                    }
                    const int k0 = (ks * p.kslices + s) * BK;
                    uint8_t* sa = smem + kOffStage + st * kStageBytes;
                    uint8_t* sb = sa + kABytes;
                    mbar_arrive_expect_tx(&full[st], kStageBytes);
                    if (p.ta) {   // A stored [K][M]: two boxes of 64 M columns x 64 K rows
                        tma_load_2d(sa, &tmA, &full[st], m0, k0);
                        tma_load_2d(sa + kABytes / 2, &tmA, &full[st], m0 + 64, k0);
                    } else {      // A stored [M][K]: one box of 64 K columns x 128 M rows
                        tma_load_2d(sa, &tmA, &full[st], k0, m0);
                    }
                    if (p.tb) {   // B stored [N][K]: one box of 64 K columns x 256 N rows
                        tma_load_2d(sb, &tmB, &full[st], k0, n0);
                    } else {      // B stored [K][N]: four boxes of 64 N columns x 64 K rows
                        for (int q = 0; q < 4; ++q) tma_load_2d(sb + q * (kBBytes / 4), &tmB, &full[st], n0 + 64 * q, k0);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // MMA issuer: the warp runs converged, one elected lane issues
        const uint32_t idesc = idesc_gemm(BM, BN, p.ta, p.tb ? 0 : 1);
        bool ok = true;
        int slice = 0, local = 0;
        for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++local) {
            const int buf = local & 1;
            // the accumulator was read by the epilogue of the tile two before
            if (local >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&acc_empty[buf], ((local - 2) >> 1) & 1,
                                                                     abort_flag, kErrTimeoutMma));
            if (!ok) break;
            tc_fence_after();
            const uint32_t acc = tmem + buf * BN;
            for (int s = 0; s < p.kslices; ++s, ++slice) {
                const int st = slice % kStages;
                if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (slice / kStages) & 1, abort_flag, kErrTimeoutMma))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + kOffStage + st * kStageBytes);
                const uint32_t sb = sa + kABytes;
                // K-major: 128-byte rows, 8-row groups 1024 bytes apart, K steps of 32 bytes;
                // MN-major: 64-column atoms 8 KB apart, K steps of 16 rows (2048 bytes)
                const uint64_t da = p.ta ? sdesc_sw128(sa, 8192, 1024) : sdesc_sw128(sa, 16, 1024);
                const uint64_t db = p.tb ? sdesc_sw128(sb, 16, 1024) : sdesc_sw128(sb, 8192, 1024);
                const uint32_t astep = p.ta ? 2048 : 32, bstep = p.tb ? 32 : 2048;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    umma_bf16_w(acc, sdesc_advance(da, kk * astep), sdesc_advance(db, kk * bstep), idesc,
                                (s > 0 || kk > 0) ? 1u : 0u);
                umma_commit_w(&empty[st]);
            }
            if (ok) umma_commit_w(&acc_full[buf]);
        }
    } else {
        // epilogue: thread = output row (TMEM lane quadrant of its warp) and
        // column half hc of every chunk
        const int quad = warp & 3;
        const int hc = (warp - 2) >> 2;
        const int r = quad * 32 + lane;
        const int et = threadIdx.x - 64;   // 0 .. 255
        uint8_t* out_box = smem + kOffOut;
        uint8_t* aux_box = smem + kOffAux;
        const bool f32 = p.out32 || p.split_out;
        const int cw = f32 ? 32 : 64;      // columns per staging box (128 bytes a row)
        const int hw = cw / 2;             // this thread's columns of a chunk: 64 bytes
        // the chunk's second operand (C for beta C, the GELU input for its
        // derivative): 32 bf16 of this thread's row, loaded one chunk ahead
        const __nv_bfloat16* side = (!f32 && p.epi == kNone && p.beta != 0.f) ? p.C
                                    : ((!f32 && p.epi == kDGelu) ? p.aux_in : nullptr);
        const int64_t side_ld = p.epi == kDGelu ? p.aux_ld : p.ldc;
        auto load_side = [&](int row, int col, uint4* dst) {
            if (side && row < p.M) {
                const uint4* src = reinterpret_cast<const uint4*>(side + static_cast<int64_t>(row) * side_ld + col);
#pragma unroll
                for (int x = 0; x < 4; ++x) dst[x] = src[x];
            }
        };
        // without a GELU output the aux box is free: the chunks alternate
        // between the two boxes, so a chunk waits only for the store of the
        // chunk two before
        const bool dbl = p.epi != kGeluAux;
        int chunk = 0;
        bool ok = true;
        int local = 0;
        for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++local) {
            int mb, nb, ks;
            tile_of(t, mb, nb, ks);
            const int m0 = mb * BM, n0 = nb * BN;
            const int buf = local & 1;
            const int row = m0 + r;
            uint4 nxt[4];
            load_side(row, n0 + hc * hw, nxt);   // in flight while the products run
            if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (local >> 1) & 1, abort_flag, kErrTimeoutSoftmax))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tacc = tmem + (static_cast<uint32_t>(quad * 32) << 16) + buf * BN;
            for (int c0 = 0; c0 < BN; c0 += cw, ++chunk) {
                const int cc = c0 + hc * hw;   // this thread's first column in the tile
                uint8_t* box = (dbl && (chunk & 1)) ? aux_box : out_box;
                uint4 cur[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) cur[x] = nxt[x];
                if (c0 + cw < BN) load_side(row, n0 + cc + cw, nxt);
                float v[32];
                if (f32) tmem_ld16(tacc + cc, v);
                else tmem_ld32(tacc + cc, v);
                tmem_wait_ld();
                // the staging box is free once the store that last used it read it
                if (et == 0) {
                    if (dbl) bulk_wait_read1();
                    else bulk_wait_read0();
                }
                epi_sync();
                const int xb = hc * 4;   // this thread's four 16-byte pieces of the box row
                if (f32) {
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        uint4 q;
                        q.x = __float_as_uint(v[4 * x + 0]);
                        q.y = __float_as_uint(v[4 * x + 1]);
                        q.z = __float_as_uint(v[4 * x + 2]);
                        q.w = __float_as_uint(v[4 * x + 3]);
                        *reinterpret_cast<uint4*>(box + r * 128 + (((xb + x) ^ (r & 7)) * 16)) = q;
                    }
                } else {
                    if (side && row < p.M) {
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            const uint32_t w[4] = {cur[x].x, cur[x].y, cur[x].z, cur[x].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                if (p.epi == kDGelu) {
                                    v[8 * x + 2 * e] *= gelu_tanh_grad(bf16_lo(w[e]));
                                    v[8 * x + 2 * e + 1] *= gelu_tanh_grad(bf16_hi(w[e]));
                                } else {
                                    v[8 * x + 2 * e] += p.beta * bf16_lo(w[e]);
                                    v[8 * x + 2 * e + 1] += p.beta * bf16_hi(w[e]);
                                }
                            }
                        }
                    }
                    if (p.epi == kGeluAux) {
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            uint4 q;
                            q.x = pack_bf16x2(v[8 * x + 0], v[8 * x + 1]);
                            q.y = pack_bf16x2(v[8 * x + 2], v[8 * x + 3]);
                            q.z = pack_bf16x2(v[8 * x + 4], v[8 * x + 5]);
                            q.w = pack_bf16x2(v[8 * x + 6], v[8 * x + 7]);
                            *reinterpret_cast<uint4*>(aux_box + r * 128 + (((xb + x) ^ (r & 7)) * 16)) = q;
                        }
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = gelu_tanh(v[i]);
                    }
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        uint4 q;
                        q.x = pack_bf16x2(v[8 * x + 0], v[8 * x + 1]);
                        q.y = pack_bf16x2(v[8 * x + 2], v[8 * x + 3]);
                        q.z = pack_bf16x2(v[8 * x + 4], v[8 * x + 5]);
                        q.w = pack_bf16x2(v[8 * x + 6], v[8 * x + 7]);
                        *reinterpret_cast<uint4*>(box + r * 128 + (((xb + x) ^ (r & 7)) * 16)) = q;
                    }
                }
                fence_proxy_async_smem();
                epi_sync();
                if (et == 0) {
                    // split partials: rows of split ks follow the previous splits' M rows
                    tma_store_2d(&tmD, box, n0 + c0, p.split_out ? ks * p.M + m0 : m0);
                    if (p.epi == kGeluAux) tma_store_2d(&tmAux, aux_box, n0 + c0, m0);
                    bulk_commit();
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[buf]);
        }
        if (et == 0) bulk_wait0();   // every store landed before the CTA leaves
    }
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        if (warp == 0 && lane == 0) drain_fills(full, kStages, issued);
        if (warp == 1) {
            umma_commit_w(drain);
            if (lane == 0) mbar_wait_drain(drain, 0);
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Sum of the K-split partials, in split order (deterministic): D[m][n] =
// Σ_s ws[s][m][n], float32.
__global__ void split_reduce_kernel(const float* __restrict__ ws, int splits, int64_t mn, int N, float* __restrict__ D,
                                    int64_t ldd) {
    const int64_t i4 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
    if (i4 >= mn) return;
    float4 acc = *reinterpret_cast<const float4*>(ws + i4);
    for (int s = 1; s < splits; ++s) {
        const float4 q = *reinterpret_cast<const float4*>(ws + s * mn + i4);
        acc.x += q.x;
        acc.y += q.y;
        acc.z += q.z;
        acc.w += q.w;
    }
    const int64_t m = i4 / N, n = i4 - m * N;
    *reinterpret_cast<float4*>(D + m * ldd + n) = acc;
}

// ------------------------------------------------------------------ host

inline bool make_map(CUtensorMap* map, CUtensorMapDataType dt, int esz, const void* base, int64_t rows, int64_t cols,
                     int64_t ld, int box_cols, int box_rows) {
    auto fn = tmap_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * esz};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K splits of a float32 product: enough tiles for every SM (each split at
// least 8 slices).
inline int choose_splits(int tiles, int K, int sms) {
    int s = 1;
    while (tiles * s < sms && (K / BK) % (2 * s) == 0 && K / BK / (2 * s) >= 8) s *= 2;
    return s;
}

inline size_t split_bytes(int M, int N, int K, int sms) {
    if (M % BM != 0 || N % BN != 0 || K % BK != 0) return 0;
    const int tiles = (M / BM) * (N / BN);
    const int s = choose_splits(tiles, K, sms);
    return s > 1 ? static_cast<size_t>(s) * M * N * sizeof(float) : 0;
}

}  // namespace gemm
}  // namespace gsa

// ------------------------------------------------------------------ the call
// (defined here, in the one translation unit that includes this header; the
// ByteLM block calls it through gemm_api.h)
namespace gsa {
namespace gemm {

size_t split_ws_bytes(int M, int N, int K) { return split_bytes(M, N, K, gsa::bwd::sm_count()); }

gsa_status run(bool ta, bool tb, int M, int N, int K, const __nv_bfloat16* A, int64_t lda, const __nv_bfloat16* B,
               int64_t ldb, float beta, const __nv_bfloat16* C, int64_t ldc, void* D, int64_t ldd, bool out32, Epi epi,
               __nv_bfloat16* aux, int64_t aux_ld, float* split_ws, size_t split_ws_bytes_, cudaStream_t st) {
    if (M < 1 || N < 1 || K < 1 || !A || !B || !D) return GSA_ERR_INVALID_ARGUMENT;
    if (N % BN != 0 || K % BK != 0 || (ta && M % BM != 0)) return GSA_ERR_UNSUPPORTED;
    if (lda % 8 || ldb % 8 || ldd % (out32 ? 4 : 8) || (beta != 0.f && (!C || ldc % 8)) ||
        (epi != kNone && (!aux || aux_ld % 8)))
        return GSA_ERR_INVALID_ARGUMENT;
    if (out32 && (epi != kNone || beta != 0.f)) return GSA_ERR_UNSUPPORTED;
    const int sms = gsa::bwd::sm_count();
    Params p{};
    p.M = M;
    p.N = N;
    p.K = K;
    p.tiles_m = (M + BM - 1) / BM;
    p.tiles_n = N / BN;
    // only whole 128-row tiles split: the parts' rows lie one split after another in the scratch
    p.splits = (out32 && M % BM == 0) ? choose_splits(p.tiles_m * p.tiles_n, K, sms) : 1;
    p.kslices = K / BK / p.splits;
    p.ta = ta;
    p.tb = tb;
    p.out32 = out32;
    p.epi = epi;
    p.beta = beta;
    p.C = C;
    p.ldc = ldc;
    p.aux_in = epi == kDGelu ? aux : nullptr;
    p.aux_ld = aux_ld;
    p.split_out = p.splits > 1;
    if (p.split_out && (!split_ws || split_ws_bytes_ < static_cast<size_t>(p.splits) * M * N * sizeof(float)))
        return GSA_ERR_CAPACITY;
    CUtensorMap ma, mb, md, maux;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    bool ok = ta ? make_map(&ma, BF, 2, A, K, M, lda, 64, 64) : make_map(&ma, BF, 2, A, M, K, lda, 64, 128);
    ok = ok && (tb ? make_map(&mb, BF, 2, B, N, K, ldb, 64, 256) : make_map(&mb, BF, 2, B, K, N, ldb, 64, 64));
    if (p.split_out) ok = ok && make_map(&md, F32, 4, split_ws, static_cast<int64_t>(p.splits) * M, N, N, 32, 128);
    else if (out32) ok = ok && make_map(&md, F32, 4, D, M, N, ldd, 32, 128);
    else ok = ok && make_map(&md, BF, 2, D, M, N, ldd, 64, 128);
    if (epi == kGeluAux) ok = ok && make_map(&maux, BF, 2, aux, M, N, aux_ld, 64, 128);
    else maux = md;
    if (!ok) return GSA_ERR_CUDA;
    if (!gsa::smem_opt_in(gemm_kernel, kSmemBytes)) return GSA_ERR_CUDA;
    const int ntiles = p.tiles_m * p.tiles_n * p.splits;
    const int grid = ntiles < sms ? ntiles : sms;
    gemm_kernel<<<grid, kThreads, kSmemBytes, st>>>(ma, mb, md, maux, p);
    if (cudaGetLastError() != cudaSuccess) return GSA_ERR_CUDA;
    if (p.split_out) {
        const int64_t mn = static_cast<int64_t>(M) * N;
        split_reduce_kernel<<<static_cast<unsigned>((mn / 4 + 255) / 256), 256, 0, st>>>(
            split_ws, p.splits, mn, N, static_cast<float*>(D), ldd);
        if (cudaGetLastError() != cudaSuccess) return GSA_ERR_CUDA;
    }
    return GSA_OK;
}

}  // namespace gemm
}  // namespace gsa
