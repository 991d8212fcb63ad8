// Block-sparse causal attention backward, bf16 in / fp32 accumulate, on
// tcgen05 tensor cores (sm_100a).
//
// The pages train the model with this mask (Gzip-guided Sparse Attention,
// daiwk.github.io, "论文离线与线上效果": 20K steps), so the gradient of the
// masked softmax attention is part of the path.  With P = softmax (from the
// forward's LSE), D_t = Σ_e dO_te O_te:
//   dS = P ∘ (dO V^T − D),  dQ = scale · dS K,  dK = scale · dS^T Q,  dV = P^T dO,
// over live pairs only.  Three launches, no atomics (deterministic):
//   1. dot_kernel   D_t for every query row (read O and dO once);
//   2. dq_kernel    one CTA per query tile (two query blocks from the class's
//                   pairing order); walks the union of their CSR rows:
//                     S = Q K^T, dP = dO V^T  -> TMEM (double-buffered)
//                     dS (bf16, back to TMEM) <- elementwise warps
//                     dQ += dS K              (A from TMEM; TMEM accumulator)
//   3. dkdv_kernel  one CTA per key tile (two key blocks from the class's key
//                   pairing order); walks the union of their CSC columns:
//                     S^T = K Q^T, dP^T = V dO^T -> TMEM (double-buffered)
//                     P^T, dS^T (bf16, back to TMEM) <- elementwise warps
//                     dV += P^T dO, dK += dS^T Q (A from TMEM; TMEM accumulators)
// Warp roles as in the forward: warp 0 TMA producer, warp 1 TMEM owner,
// warps 2-9 two elementwise groups with one thread per TMEM lane; one thread
// of each group issues that group's MMAs right after its rows are in TMEM.
// The bf16 operands written by the elementwise warps stay in TMEM as packed
// pairs (lane = row, column c = elements 2c, 2c+1), the layout of an M=128
// A operand, so they never pass through shared memory.
// At d = 64, steps 2 and 3 run as persistent kernels over the same items
// (dq_persist_kernel, two CTAs per SM; dkdv_persist_kernel, one CTA per SM
// with double-buffered scores): attn_bwd_dq_persist.cuh, attn_bwd_persist.cuh.
#pragma once

#include <atomic>

#include "common.cuh"
#include "tiles.cuh"

namespace gsa {
namespace bwd {

constexpr int kBlk = 64;
constexpr int kMaxHeads = 256;
constexpr float kLog2e = 1.4426950408889634f;
// Elementwise warpgroups: group g takes the tiles n with n % G == g, one
// thread per tile row (TMEM lane), all 64 columns.  d = 64 runs one group
// per CTA and two CTAs per SM (a CTA then fits in 256 TMEM columns and half
// the shared memory), so one CTA's set-up and epilogue overlap the other's
// tiles; d = 128 runs two groups in one CTA per SM.
#ifndef GSA_BWD64_GROUPS
#define GSA_BWD64_GROUPS 1
#endif
// With one group, each tile's 64 columns are split between two warpgroups
// (32 columns per thread), so eight elementwise warps share a tile.
#ifndef GSA_BWD64_HALVES
#define GSA_BWD64_HALVES 2
#endif
template <int D>
struct Shape {
    static constexpr int kGroups = D == 64 ? GSA_BWD64_GROUPS : 2;
    static constexpr int kHalves = kGroups == 1 ? GSA_BWD64_HALVES : 1;
    static constexpr int kThreads = 64 + 128 * kGroups * kHalves;
    static constexpr int kCtasPerSm = kGroups == 1 ? 2 : 1;
};

struct Params {
    const int32_t* ptr;     // CSR row_ptr (dq) or CSC col_ptr (dkdv)
    const int32_t* idx;     // col_idx or row_idx
    const int32_t* order;   // q_order or k_order
    int64_t cap;
    int S, H, nblk;
    int64_t L;
    const float* lse;
    const float* nlse2;     // -LSE_t log2(e), written next to -D_t by dot_kernel
    const float* ndvec;     // -D_t (negated: the exponent and dS take them as addends)
    __nv_bfloat16* out0;    // dq (dq_kernel) or dv (dkdv_kernel)
    __nv_bfloat16* out1;    // dk (dkdv_kernel)
    TokLayout lq;           // layout of q, k, v and of dq, dk, dv
    float scale;
    float scale_log2;
    int* ticket;            // work counter of the persistent kernel (dot_kernel zeroes both)
    uint8_t cls[kMaxHeads];
    int local_implicit;   // the local class's lists are not stored: derived from (nblk, w)
    int w;                // the lists' window
};

// ------------------------------------------------------------ D_t = dO·O

// Grid (L / (kRows kRowsPerCta), y): CTA (x, y) takes the tokens
// [x kRows kRowsPerCta, (x + 1) kRows kRowsPerCta) of the (sample, head)
// pairs sh = y, y + gridDim.y, ..., kRows rows per thread with their loads in
// flight together (L is a multiple of 64; consecutive CTAs read consecutive
// rows).
#ifndef GSA_DOT_ROWS
#define GSA_DOT_ROWS 2
#endif
template <int D>
__global__ void __launch_bounds__(256) dot_kernel(const __nv_bfloat16* __restrict__ o,
                                                  const __nv_bfloat16* __restrict__ dO, TokLayout lo, int64_t L,
                                                  int H, int SH, float* __restrict__ ndvec,
                                                  const float* __restrict__ lse, float* __restrict__ nlse2,
                                                  int* __restrict__ ticket) {
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < 2) ticket[threadIdx.x] = 0;   // for the persistent kernels
    constexpr int kTpr = D / 8;                  // threads per row, 8 elements (16 bytes) each
    constexpr int kRowsPerCta = 256 / kTpr;
    constexpr int kRows = GSA_DOT_ROWS;
    const int64_t l0 = static_cast<int64_t>(blockIdx.x) * (kRows * kRowsPerCta) + threadIdx.x / kTpr;
    const int part = threadIdx.x % kTpr;
    for (int sh = blockIdx.y; sh < SH; sh += gridDim.y) {
        const int s = sh / H, h = sh - s * H;
        uint4 a[kRows], b[kRows];
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            const int64_t off = s * lo.s + h * lo.h + (l0 + u * kRowsPerCta) * lo.l + part * 8;
            a[u] = *reinterpret_cast<const uint4*>(o + off);
            b[u] = *reinterpret_cast<const uint4*>(dO + off);
        }
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            const __nv_bfloat162* ah = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
            const __nv_bfloat162* bh = reinterpret_cast<const __nv_bfloat162*>(&b[u]);
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 fa = __bfloat1622float2(ah[e]);
                const float2 fb = __bfloat1622float2(bh[e]);
                acc = fmaf(fa.x, fb.x, acc);
                acc = fmaf(fa.y, fb.y, acc);
            }
#pragma unroll
            for (int o2 = kTpr / 2; o2 > 0; o2 >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o2);
            if (part == 0) {
                const int64_t row = static_cast<int64_t>(sh) * L + l0 + u * kRowsPerCta;
                ndvec[row] = -acc;
                nlse2[row] = -(lse[row] * kLog2e);   // the backward's exponents are in log2 units
            }
        }
    }
}

// ------------------------------------------------------------ dQ

// Ring depths: a stage is released after the last MMA that reads it.
#ifndef GSA_DQ64_STAGES
#define GSA_DQ64_STAGES (GSA_BWD64_GROUPS == 1 ? 4 : 8)
#endif
#ifndef GSA_DQ128_STAGES
#define GSA_DQ128_STAGES 4
#endif
#ifndef GSA_DKV64_STAGES
#define GSA_DKV64_STAGES (GSA_BWD64_GROUPS == 1 ? 4 : 8)
#endif
#ifndef GSA_DKV128_STAGES
#define GSA_DKV128_STAGES 4
#endif

template <int D>
struct DqCfg {
    static constexpr int G = Shape<D>::kGroups;
    static constexpr int kAtoms = D / 64;
    static constexpr int kStages = D == 64 ? GSA_DQ64_STAGES : GSA_DQ128_STAGES;
    static constexpr int kTileBytes = 128 * D * 2;      // Q or dO tile (128 rows)
    static constexpr int kKVBytes = kBlk * D * 2;       // one key block of K or V
    static constexpr int kOffQ = 0;
    static constexpr int kOffDO = kOffQ + kTileBytes;
    static constexpr int kOffK = kOffDO + kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kKVBytes;
    static constexpr int kOffBar = kOffV + kStages * kKVBytes;
    // full[st], empty[st], q_full, s_full[2], ds_full[2], done
    static constexpr int kNumBars = 2 * kStages + 8;   // + drain[2]
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kOffList = kOffMisc + 16;
    static constexpr int kOffLive = kOffList + kListMaxBlocks * 2;
    static constexpr int kOffBits = kOffLive + kListMaxBlocks;
    static constexpr int kEnd = kOffBits + 2 * (kListMaxBlocks / 32) * 4;
    static constexpr int kSmemBytes = kEnd + 1024;
    static_assert(kSmemBytes <= 232448 / Shape<D>::kCtasPerSm - 1024, "shared memory per CTA");
    // S[g] at 128 g (dS over its first 32 columns), dP[g] at 128 g + 64,
    // dQ_g (group g's share of the sum) at 128 G + g D
    static constexpr int kTmemDQ = 128 * G;
    static constexpr int kTmemCols = kTmemDQ + G * D <= 256 ? 256 : 512;
    static_assert(kTmemCols * Shape<D>::kCtasPerSm <= 512, "TMEM per SM");
};

template <int D, bool K4>   // K4: strided tensors through 4-D maps (see load_rows)
__global__ void __launch_bounds__(Shape<D>::kThreads, Shape<D>::kCtasPerSm)
dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO, const Params p) {
    using C = DqCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sDO = smem + C::kOffDO;
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::kStages;
    uint64_t* q_full = bars + 2 * C::kStages;
    uint64_t* s_full = q_full + 1;
    uint64_t* ds_full = s_full + 2;
    uint64_t* done = ds_full + 2;   // one phase: every product of the CTA completed
    uint64_t* drain = done + 1;     // [G] each group's MMA thread at exit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    TileList tl;
    tl.count = reinterpret_cast<int*>(smem + C::kOffMisc + 8);
    tl.list = reinterpret_cast<int16_t*>(smem + C::kOffList);
    tl.live = smem + C::kOffLive;
    tl.bitsA = reinterpret_cast<uint32_t*>(smem + C::kOffBits);
    tl.bitsB = tl.bitsA + kListMaxBlocks / 32;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sh = blockIdx.x;
    const int s = sh / p.H, h = sh % p.H;
    const int tile = blockIdx.y;
    const int c = p.cls[h];
    const int nblk = p.nblk;
    const int64_t g = static_cast<int64_t>(s) * 3 + c;
    const bool implicit = c == 0 && p.local_implicit;
    const int32_t* ord = implicit ? nullptr : p.order + g * nblk;
    const int qa = order_at(ord, 2 * tile);
    const int qb = (2 * tile + 1 < nblk) ? order_at(ord, 2 * tile + 1) : -1;
    const int64_t head_row0 = static_cast<int64_t>(sh) * p.L;

    if (threadIdx.x == 0) {
        for (int st = 0; st < C::kStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        mbar_init(&ds_full[0], 128 * Shape<D>::kHalves);
        mbar_init(&ds_full[1], 128 * Shape<D>::kHalves);
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        // Q and dO of the tile load while the key lists merge
        mbar_arrive_expect_tx(q_full, (qb >= 0 ? 2 : 1) * 2 * kBlk * D * 2);
        for (int half = 0; half < 2; ++half) {
            const int blk = half ? qb : qa;
            if (blk < 0) continue;
            const int l0 = blk * kBlk;   // token coordinate in the (sample, head)
            for (int at = 0; at < C::kAtoms; ++at) {
                load_rows<K4>(sQ + at * (128 * 128) + half * (kBlk * 128), &tmQ, q_full, at * 64, l0, h, s, head_row0);
                load_rows<K4>(sDO + at * (128 * 128) + half * (kBlk * 128), &tmDO, q_full, at * 64, l0, h, s, head_row0);
            }
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    build_tile_list(tl, ListRef{implicit ? nullptr : p.ptr + g * (nblk + 1), p.idx + g * p.cap, p.w, nblk, false}, qa,
                    qb, nblk);
    if (threadIdx.x == 0) {
        mbar_init(done, *tl.count >= C::G ? C::G : 1);   // one arrival per group that has tiles
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int T = *tl.count;
    const uint32_t tmem = *tmem_slot;
    int fills = 0;   // producer: stages issued

    if (warp == 0) {
        if (lane == 0) {
            int n = 0;
            for (; n < T; ++n) {
                const int st = n % C::kStages;
                if (n >= C::kStages &&
                    !mbar_wait(&empty[st], ((n / C::kStages) - 1) & 1, abort_flag, kErrTimeoutProducer))
                    break;
                mbar_arrive_expect_tx(&full[st], 2 * C::kKVBytes);
                const int l0 = tl.list[n] * kBlk;   // token coordinate in the (sample, head)
                for (int at = 0; at < C::kAtoms; ++at) {
                    load_rows<K4>(sK + st * C::kKVBytes + at * (kBlk * 128), &tmK, &full[st], at * 64, l0, h, s, head_row0);
                    load_rows<K4>(sV + st * C::kKVBytes + at * (kBlk * 128), &tmV, &full[st], at * 64, l0, h, s, head_row0);
                }
            }
            fills = n;
        }
    } else if (warp >= 2) {
        // warp e = warp - 2: group (e / 4) % G, column half (e / 4) / G
        constexpr int H = Shape<D>::kHalves;
        constexpr int kCols = kBlk / H;         // key columns per thread
        constexpr int kW = 16 / H;              // chunk width (four chunks)
        const int e4 = (warp - 2) >> 2;
        const int quad = warp & 3;              // TMEM lane quadrant this warp may access
        const int grp = e4 % C::G;              // this group takes the tiles n % G == grp
        const int hc = e4 / C::G;               // key columns [kCols hc, kCols (hc + 1))
        const int c0 = kCols * hc;
        const int r = quad * 32 + lane;
        const int half = r >> 6;
        const int my_blk = half ? qb : qa;
        const int rr = r & 63;
        const uint32_t tlane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const int64_t tok = head_row0 + static_cast<int64_t>(my_blk < 0 ? 0 : my_blk) * kBlk + rr;
        const float nlse2 = my_blk >= 0 ? p.nlse2[tok] : 0.f;
        const float ndt = my_blk >= 0 ? p.ndvec[tok] : 0.f;
        // the group's MMA issuer: lane 0 of its first warp
        const bool issuer_warp = ((warp - 2) & 3) == 0 && hc == 0;
        constexpr uint32_t idesc_s = idesc_bf16(128, kBlk, 0);
        constexpr uint32_t idesc_dq = idesc_bf16(128, D, 1);
        const uint32_t aQ = smem_u32(sQ), aDO = smem_u32(sDO), aK = smem_u32(sK), aV = smem_u32(sV);
        auto issue_s = [&](int t) {   // S[grp] = Q K_t^T, dP[grp] = dO V_t^T, then s_full[grp]
            const int st = t % C::kStages;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int at = kk >> 2, ko = (kk & 3) * 32;
                const uint64_t aq = sdesc_sw128(aQ + at * (128 * 128) + ko, 16, 1024);
                const uint64_t bk = sdesc_sw128(aK + st * C::kKVBytes + at * (kBlk * 128) + ko, 16, 1024);
                umma_bf16(tmem + grp * 128, aq, bk, idesc_s, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int at = kk >> 2, ko = (kk & 3) * 32;
                const uint64_t ado = sdesc_sw128(aDO + at * (128 * 128) + ko, 16, 1024);
                const uint64_t bv = sdesc_sw128(aV + st * C::kKVBytes + at * (kBlk * 128) + ko, 16, 1024);
                umma_bf16(tmem + grp * 128 + 64, ado, bv, idesc_s, kk > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[grp]);
        };
        if (issuer_warp) {
            if (lane == 0 && grp < T &&
                mbar_wait(q_full, 0, abort_flag, kErrTimeoutMma) &&
                mbar_wait(&full[grp % C::kStages], (grp / C::kStages) & 1, abort_flag, kErrTimeoutMma)) {
                tc_fence_after();
                issue_s(grp);
            }
            __syncwarp();
        }
        bool ok = true;
        for (int n = grp; n < T; n += C::G) {
            const int ph = (n / C::G) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&s_full[grp], ph, abort_flag, kErrTimeoutSoftmax))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int j = tl.list[n];
            const bool is_live = (tl.live[n] >> half) & 1;
            const int last = !is_live ? -1 : (j == my_blk ? rr : kBlk - 1);   // visible key columns 0..last
            uint32_t pk[kCols / 2];
            if (last < c0) {
#pragma unroll
                for (int e = 0; e < kCols / 2; ++e) pk[e] = 0u;
            } else {
                // four chunks of kW columns; the next chunk's TMEM loads are in
                // flight while one is computed
                float sv[2][kW], dp[2][kW];
                tmem_ldw<kW>(tlane + grp * 128 + c0, sv[0]);
                tmem_ldw<kW>(tlane + grp * 128 + 64 + c0, dp[0]);
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    tmem_wait_ld();
                    if (ch < 3) {
                        tmem_ldw<kW>(tlane + grp * 128 + c0 + kW * (ch + 1), sv[(ch + 1) & 1]);
                        tmem_ldw<kW>(tlane + grp * 128 + 64 + c0 + kW * (ch + 1), dp[(ch + 1) & 1]);
                    }
                    float* s_ = sv[ch & 1];
                    const float* d_ = dp[ch & 1];
                    const int cb = c0 + kW * ch;   // first key column of the chunk
#pragma unroll
                    for (int cc = 0; cc < kW; ++cc) s_[cc] = ex2(fmaf(s_[cc], p.scale_log2, nlse2)) * (d_[cc] + ndt);
                    if (last < cb + kW - 1) {
#pragma unroll
                        for (int cc = 0; cc < kW; ++cc) s_[cc] = cb + cc <= last ? s_[cc] : 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < kW / 2; ++e) pk[(kW / 2) * ch + e] = pack_bf16x2(s_[2 * e], s_[2 * e + 1]);
                }
            }
            // this thread's dS, packed, over the first kCols / 2 of its own S
            // columns (all read above): key pairs of columns [c0, c0 + kCols)
            // sit at S[grp] columns c0 .. c0 + kCols / 2 - 1
            tmem_stn<kCols / 2>(tlane + grp * 128 + c0, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&ds_full[grp]);
            if (issuer_warp) {
                if (lane == 0 && mbar_wait(&ds_full[grp], ph, abort_flag, kErrTimeoutMma)) {
                    // dQ_grp += dS K (dS read from TMEM), then S and dP of the group's next tile
                    tc_fence_after();
                    const int st = n % C::kStages;
#pragma unroll
                    for (int kk = 0; kk < kBlk / 16; ++kk) {
                        const int h_ = (16 * kk) / kCols;   // the half holding keys 16 kk ..
                        const uint32_t acol = kCols * h_ + (16 * kk - kCols * h_) / 2;
                        const uint64_t bd = sdesc_sw128(aK + st * C::kKVBytes + kk * (16 * 128), kBlk * 128, 1024);
                        umma_bf16_ts(tmem + C::kTmemDQ + grp * D, tmem + grp * 128 + acol, bd, idesc_dq,
                                     (n >= C::G || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[st]);
                    if (n + C::G < T) {
                        if (mbar_wait(&full[(n + C::G) % C::kStages], ((n + C::G) / C::kStages) & 1, abort_flag,
                                      kErrTimeoutMma)) {
                            tc_fence_after();
                            issue_s(n + C::G);
                        }
                    } else {
                        umma_commit(done);
                    }
                }
                __syncwarp();
            }
        }
        if (ok && T > 0 &&
            __all_sync(0xffffffffu, mbar_wait(done, 0, abort_flag, kErrTimeoutSoftmax))) {
            tc_fence_after();
            const bool has1 = C::G == 2 && T >= 2;   // dQ_1 holds products only if group 1 had a tile
            __nv_bfloat16* orow = p.out0 + (K4 ? tok_off(tok, p.L, p.H, p.lq) : tok * D);
            constexpr int kOc = D / (C::G * H);   // output columns per thread (split among a row's threads)
            const int slot = grp * H + hc;
#pragma unroll
            for (int cb = slot * kOc; cb < (slot + 1) * kOc; cb += 32) {
                float ov[32];
                tmem_ld32(tlane + C::kTmemDQ + cb, ov);
                tmem_wait_ld();
                if (has1) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float o2[16];
                        tmem_ld16(tlane + C::kTmemDQ + D + cb + 16 * hh, o2);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) ov[16 * hh + e] += o2[e];
                    }
                }
                if (my_blk >= 0) store_scaled_bf16(orow + cb, ov, p.scale);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // a role gave up a wait: the loads and products issued must land before
        // shared memory and TMEM go (without one, every one of them was waited for)
        if (warp == 0 && lane == 0) {
            mbar_wait_drain(q_full, 0);
            drain_fills(full, C::kStages, fills);
        }
        const int e4 = (warp - 2) >> 2;
        if (warp >= 2 && ((warp - 2) & 3) == 0 && e4 / C::G == 0 && lane == 0) {   // each group's MMA thread
            umma_commit(&drain[e4 % C::G]);
            mbar_wait_drain(&drain[e4 % C::G], 0);
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ------------------------------------------------------------ dK, dV

template <int D>
struct DkvCfg {
    static constexpr int G = Shape<D>::kGroups;
    static constexpr int kAtoms = D / 64;
    static constexpr int kStages = D == 64 ? GSA_DKV64_STAGES : GSA_DKV128_STAGES;
    static constexpr int kTileBytes = 128 * D * 2;      // K or V tile (128 key rows)
    static constexpr int kQBytes = kBlk * D * 2;        // one query block of Q or dO
    static constexpr int kVecBytes = kBlk * 4;          // LSE or D of one query block
    static constexpr int kStageBytes = 2 * kQBytes;          // stage: Q, dO (TMA, 1024-aligned)
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + kTileBytes;
    static constexpr int kOffStage = kOffV + kTileBytes;
    static constexpr int kOffVec = kOffStage + kStages * kStageBytes;   // per stage: LSE[64], D[64]
    static constexpr int kOffBar = kOffVec + kStages * 2 * kVecBytes;
    // full[st], empty[st], kv_full, s_full[2], p_full[2], acc[2], done
    static constexpr int kNumBars = 2 * kStages + 10;   // + drain[2]
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kOffList = kOffMisc + 16;
    static constexpr int kOffLive = kOffList + kListMaxBlocks * 2;
    static constexpr int kOffBits = kOffLive + kListMaxBlocks;
    static constexpr int kEnd = kOffBits + 2 * (kListMaxBlocks / 32) * 4;
    static constexpr int kSmemBytes = kEnd + 1024;
    static_assert(kSmemBytes <= 232448 / Shape<D>::kCtasPerSm - 1024, "shared memory per CTA");
    static_assert(kStageBytes % 1024 == 0, "stages keep 1024-byte alignment");
    // S^T[g] at 128 g (P^T over its first 32 columns), dP^T[g] at 128 g + 64
    // (dS^T over its first 32), accumulators from 128 G.  With two groups at
    // d = 64 each group keeps its own dV_g, dK_g (at 128 G + 2 D g and
    // 128 G + 2 D g + D) and the epilogue adds them; two groups at d = 128
    // leave room for one dV and one dK, which the groups' products take in
    // turn (the acc barriers order them).
    static constexpr bool kSplit = G == 1 || D == 64;
    static constexpr uint32_t kAcc = 128 * G;
    __host__ __device__ static constexpr uint32_t dv_col(int grp) { return kSplit ? kAcc + 2 * D * grp : kAcc; }
    __host__ __device__ static constexpr uint32_t dk_col(int grp) {
        return kSplit ? kAcc + 2 * D * grp + D : kAcc + D;
    }
    static constexpr int kTmemCols = kAcc + (kSplit ? G : 1) * 2 * D <= 256 ? 256 : 512;
    static_assert(kTmemCols * Shape<D>::kCtasPerSm <= 512, "TMEM per SM");
};

template <int D, bool K4>   // K4: strided tensors through 4-D maps (see load_rows)
__global__ void __launch_bounds__(Shape<D>::kThreads, Shape<D>::kCtasPerSm)
dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
            const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO, const Params p) {
    using C = DkvCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint8_t* sStage = smem + C::kOffStage;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::kStages;
    uint64_t* kv_full = bars + 2 * C::kStages;
    uint64_t* s_full = kv_full + 1;
    uint64_t* p_full = s_full + 2;
    uint64_t* acc = p_full + 2;     // d = 128: group g's dV/dK products of its latest tile completed
    uint64_t* done = acc + 2;       // one phase: every product of the CTA completed
    uint64_t* drain = done + 1;     // [G] each group's MMA thread at exit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    TileList tl;
    tl.count = reinterpret_cast<int*>(smem + C::kOffMisc + 8);
    tl.list = reinterpret_cast<int16_t*>(smem + C::kOffList);
    tl.live = smem + C::kOffLive;
    tl.bitsA = reinterpret_cast<uint32_t*>(smem + C::kOffBits);
    tl.bitsB = tl.bitsA + kListMaxBlocks / 32;
    auto stage_q = [&](int st) { return sStage + st * C::kStageBytes; };
    auto stage_do = [&](int st) { return sStage + st * C::kStageBytes + C::kQBytes; };
    auto stage_lse = [&](int st) { return reinterpret_cast<float*>(smem + C::kOffVec + st * 2 * C::kVecBytes); };
    auto stage_d = [&](int st) {
        return reinterpret_cast<float*>(smem + C::kOffVec + st * 2 * C::kVecBytes + C::kVecBytes);
    };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sh = blockIdx.x;
    const int s = sh / p.H, h = sh % p.H;
    const int tile = blockIdx.y;
    const int c = p.cls[h];
    const int nblk = p.nblk;
    const int64_t g = static_cast<int64_t>(s) * 3 + c;
    const bool implicit = c == 0 && p.local_implicit;
    const int32_t* ord = implicit ? nullptr : p.order + g * nblk;
    const int ka = order_at(ord, 2 * tile);
    const int kb = (2 * tile + 1 < nblk) ? order_at(ord, 2 * tile + 1) : -1;
    const int64_t head_row0 = static_cast<int64_t>(sh) * p.L;

    if (threadIdx.x == 0) {
        for (int st = 0; st < C::kStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
        }
        mbar_init(kv_full, 1);
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        mbar_init(&p_full[0], 128 * Shape<D>::kHalves);
        mbar_init(&p_full[1], 128 * Shape<D>::kHalves);
        mbar_init(&acc[0], 1);
        mbar_init(&acc[1], 1);
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmDO);
        // K and V of the tile load while the query lists merge
        mbar_arrive_expect_tx(kv_full, (kb >= 0 ? 2 : 1) * 2 * kBlk * D * 2);
        for (int half = 0; half < 2; ++half) {
            const int blk = half ? kb : ka;
            if (blk < 0) continue;
            const int l0 = blk * kBlk;   // token coordinate in the (sample, head)
            for (int at = 0; at < C::kAtoms; ++at) {
                load_rows<K4>(sK + at * (128 * 128) + half * (kBlk * 128), &tmK, kv_full, at * 64, l0, h, s, head_row0);
                load_rows<K4>(sV + at * (128 * 128) + half * (kBlk * 128), &tmV, kv_full, at * 64, l0, h, s, head_row0);
            }
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    build_tile_list(tl, ListRef{implicit ? nullptr : p.ptr + g * (nblk + 1), p.idx + g * p.cap, p.w, nblk, true}, ka,
                    kb, nblk);
    if (threadIdx.x == 0) {
        mbar_init(done, *tl.count >= C::G ? C::G : 1);   // one arrival per group that has tiles
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int T = *tl.count;
    const uint32_t tmem = *tmem_slot;
    int fills = 0;   // producer: stages issued

    if (warp == 0) {
        if (lane == 0) {
            int n = 0;
            for (; n < T; ++n) {
                const int st = n % C::kStages;
                if (n >= C::kStages &&
                    !mbar_wait(&empty[st], ((n / C::kStages) - 1) & 1, abort_flag, kErrTimeoutProducer))
                    break;
                mbar_arrive_expect_tx(&full[st], C::kStageBytes + 2 * C::kVecBytes);
                const int64_t row64 = head_row0 + static_cast<int64_t>(tl.list[n]) * kBlk;
                const int l0 = static_cast<int>(row64 - head_row0);   // token coordinate in the (sample, head)
                for (int at = 0; at < C::kAtoms; ++at) {
                    load_rows<K4>(stage_q(st) + at * (kBlk * 128), &tmQ, &full[st], at * 64, l0, h, s, head_row0);
                    load_rows<K4>(stage_do(st) + at * (kBlk * 128), &tmDO, &full[st], at * 64, l0, h, s, head_row0);
                }
                bulk_load(stage_lse(st), p.nlse2 + row64, C::kVecBytes, &full[st]);
                bulk_load(stage_d(st), p.ndvec + row64, C::kVecBytes, &full[st]);
            }
            fills = n;
        }
    } else if (warp >= 2) {
        // warp e = warp - 2: group (e / 4) % G, column half (e / 4) / G
        constexpr int H = Shape<D>::kHalves;
        constexpr int kCols = kBlk / H;          // query columns per thread
        constexpr int kW = 16 / H;               // chunk width (four chunks)
        const int e4 = (warp - 2) >> 2;
        const int quad = warp & 3;
        const int grp = e4 % C::G;               // this group takes the tiles n % G == grp
        const int hc = e4 / C::G;                // query columns [kCols hc, kCols (hc + 1))
        const int c0 = kCols * hc;
        const int u = quad * 32 + lane;          // key row of the tile = TMEM lane
        const int half = u >> 6;
        const int my_blk = half ? kb : ka;
        const int uu = u & 63;
        const uint32_t tlane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        // the group's MMA issuer: lane 0 of its first warp
        const bool issuer_warp = ((warp - 2) & 3) == 0 && hc == 0;
        constexpr uint32_t idesc_s = idesc_bf16(128, kBlk, 0);
        constexpr uint32_t idesc_acc = idesc_bf16(128, D, 1);
        const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
        auto issue_s = [&](int t) {   // S^T[grp] = K Q_t^T, dP^T[grp] = V dO_t^T, then s_full[grp]
            const int st = t % C::kStages;
            const uint32_t aQs = smem_u32(stage_q(st)), aDOs = smem_u32(stage_do(st));
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int at = kk >> 2, ko = (kk & 3) * 32;
                const uint64_t ak = sdesc_sw128(aK + at * (128 * 128) + ko, 16, 1024);
                const uint64_t bq = sdesc_sw128(aQs + at * (kBlk * 128) + ko, 16, 1024);
                umma_bf16(tmem + grp * 128, ak, bq, idesc_s, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int at = kk >> 2, ko = (kk & 3) * 32;
                const uint64_t av = sdesc_sw128(aV + at * (128 * 128) + ko, 16, 1024);
                const uint64_t bdo = sdesc_sw128(aDOs + at * (kBlk * 128) + ko, 16, 1024);
                umma_bf16(tmem + grp * 128 + 64, av, bdo, idesc_s, kk > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[grp]);
        };
        if (issuer_warp) {
            if (lane == 0 && grp < T &&
                mbar_wait(kv_full, 0, abort_flag, kErrTimeoutMma) &&
                mbar_wait(&full[grp % C::kStages], (grp / C::kStages) & 1, abort_flag, kErrTimeoutMma)) {
                tc_fence_after();
                issue_s(grp);
            }
            __syncwarp();
        }
        bool ok = true;
        for (int n = grp; n < T; n += C::G) {
            const int st = n % C::kStages;
            const int ph = (n / C::G) & 1;
            bool w_ok = mbar_wait(&s_full[grp], ph, abort_flag, kErrTimeoutSoftmax);
            // the stage's LSE and D came in by TMA: observe its barrier too
            w_ok = w_ok && mbar_wait(&full[st], (n / C::kStages) & 1, abort_flag, kErrTimeoutSoftmax);
            if (!__all_sync(0xffffffffu, w_ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int i = tl.list[n];
            const bool is_live = (tl.live[n] >> half) & 1;
            // query columns allowed: live block, and in the diagonal block t >= u
            const int first = !is_live ? kBlk : (i == my_blk ? uu : 0);
            uint32_t pp[kCols / 2], pd[kCols / 2];
            if (first >= c0 + kCols) {
#pragma unroll
                for (int e = 0; e < kCols / 2; ++e) pp[e] = pd[e] = 0u;
            } else {
                const float4* lse4 = reinterpret_cast<const float4*>(stage_lse(st));
                const float4* dv4 = reinterpret_cast<const float4*>(stage_d(st));
                // four chunks of kW columns; the next chunk's TMEM loads are in
                // flight while one is computed
                float sv[2][kW], dp[2][kW];
                tmem_ldw<kW>(tlane + grp * 128 + c0, sv[0]);
                tmem_ldw<kW>(tlane + grp * 128 + 64 + c0, dp[0]);
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    tmem_wait_ld();
                    if (ch < 3) {
                        tmem_ldw<kW>(tlane + grp * 128 + c0 + kW * (ch + 1), sv[(ch + 1) & 1]);
                        tmem_ldw<kW>(tlane + grp * 128 + 64 + c0 + kW * (ch + 1), dp[(ch + 1) & 1]);
                    }
                    float* s_ = sv[ch & 1];
                    float* d_ = dp[ch & 1];
                    const int cb = c0 + kW * ch;   // first query column of the chunk
#pragma unroll
                    for (int c4 = 0; c4 < kW / 4; ++c4) {
                        const float4 l4 = lse4[cb / 4 + c4];
                        const float4 d4 = dv4[cb / 4 + c4];
                        const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
                        const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int cc = 4 * c4 + e;
                            float pr = ex2(fmaf(s_[cc], p.scale_log2, lv[e]));
                            if (first > cb) pr = cb + cc >= first ? pr : 0.f;
                            s_[cc] = pr;
                            d_[cc] = pr * (d_[cc] + dd[e]);
                        }
                    }
#pragma unroll
                    for (int e = 0; e < kW / 2; ++e) {
                        pp[(kW / 2) * ch + e] = pack_bf16x2(s_[2 * e], s_[2 * e + 1]);
                        pd[(kW / 2) * ch + e] = pack_bf16x2(d_[2 * e], d_[2 * e + 1]);
                    }
                }
            }
            // this thread's P^T and dS^T, packed, over the first kCols / 2 of its
            // own S^T and dP^T columns (all read above)
            tmem_stn<kCols / 2>(tlane + grp * 128 + c0, pp);
            tmem_stn<kCols / 2>(tlane + grp * 128 + 64 + c0, pd);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[grp]);
            if (issuer_warp) {
                bool go = lane == 0 && mbar_wait(&p_full[grp], ph, abort_flag, kErrTimeoutMma);
                // shared accumulators: the other group's products of tile n - 1 completed first
                if (!C::kSplit && go && n >= 1)
                    go = mbar_wait(&acc[grp ^ 1], ((n - 1) >> 1) & 1, abort_flag, kErrTimeoutMma);
                if (go) {
                    // dV += P^T dO, dK += dS^T Q (A from TMEM), then the group's next S^T, dP^T
                    tc_fence_after();
                    const uint32_t aQs = smem_u32(stage_q(st)), aDOs = smem_u32(stage_do(st));
                    const bool first_prod = C::kSplit ? n < C::G : n < 1;
#pragma unroll
                    for (int kk = 0; kk < kBlk / 16; ++kk) {
                        const int h_ = (16 * kk) / kCols;   // the half holding queries 16 kk ..
                        const uint32_t acol = kCols * h_ + (16 * kk - kCols * h_) / 2;
                        const uint64_t bdo = sdesc_sw128(aDOs + kk * (16 * 128), kBlk * 128, 1024);
                        umma_bf16_ts(tmem + C::dv_col(grp), tmem + grp * 128 + acol, bdo, idesc_acc,
                                     (!first_prod || kk > 0) ? 1u : 0u);
                    }
#pragma unroll
                    for (int kk = 0; kk < kBlk / 16; ++kk) {
                        const int h_ = (16 * kk) / kCols;
                        const uint32_t acol = kCols * h_ + (16 * kk - kCols * h_) / 2;
                        const uint64_t bq = sdesc_sw128(aQs + kk * (16 * 128), kBlk * 128, 1024);
                        umma_bf16_ts(tmem + C::dk_col(grp), tmem + grp * 128 + 64 + acol, bq, idesc_acc,
                                     (!first_prod || kk > 0) ? 1u : 0u);
                    }
                    if (!C::kSplit) umma_commit(&acc[grp]);
                    umma_commit(&empty[st]);
                    if (n + C::G < T) {
                        if (mbar_wait(&full[(n + C::G) % C::kStages], ((n + C::G) / C::kStages) & 1, abort_flag,
                                      kErrTimeoutMma)) {
                            tc_fence_after();
                            issue_s(n + C::G);
                        }
                    } else {
                        umma_commit(done);
                    }
                }
                __syncwarp();
            }
        }
        if (ok && T > 0 &&
            __all_sync(0xffffffffu, mbar_wait(done, 0, abort_flag, kErrTimeoutSoftmax))) {
            tc_fence_after();
            const bool has1 = C::G == 2 && C::kSplit && T >= 2;   // the group-1 accumulators hold products
            const int64_t tok = head_row0 + static_cast<int64_t>(my_blk < 0 ? 0 : my_blk) * kBlk + uu;
            constexpr int kOc = D / (C::G * H);   // output columns per thread (split among a row's threads)
            const int slot = grp * H + hc;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                __nv_bfloat16* orow = (which == 0 ? p.out0 : p.out1) + (K4 ? tok_off(tok, p.L, p.H, p.lq) : tok * D);
                const float mul = which == 0 ? 1.f : p.scale;
                const uint32_t col0 = which == 0 ? C::dv_col(0) : C::dk_col(0);
                const uint32_t col1 = which == 0 ? C::dv_col(1) : C::dk_col(1);
#pragma unroll
                for (int cb = slot * kOc; cb < (slot + 1) * kOc; cb += 32) {
                    float ov[32];
                    tmem_ld32(tlane + col0 + cb, ov);
                    tmem_wait_ld();
                    if (has1) {
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            float o2[16];
                            tmem_ld16(tlane + col1 + cb + 16 * hh, o2);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 16; ++e) ov[16 * hh + e] += o2[e];
                        }
                    }
                    if (my_blk >= 0) store_scaled_bf16(orow + cb, ov, mul);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // a role gave up a wait: the loads and products issued must land before
        // shared memory and TMEM go (without one, every one of them was waited for)
        if (warp == 0 && lane == 0) {
            mbar_wait_drain(kv_full, 0);
            drain_fills(full, C::kStages, fills);
        }
        const int e4 = (warp - 2) >> 2;
        if (warp >= 2 && ((warp - 2) & 3) == 0 && e4 / C::G == 0 && lane == 0) {   // each group's MMA thread
            umma_commit(&drain[e4 % C::G]);
            mbar_wait_drain(&drain[e4 % C::G], 0);
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace bwd
}  // namespace gsa

#include "attn_bwd_persist.cuh"
#include "attn_bwd_dq_persist.cuh"

namespace gsa {
namespace bwd {

// ------------------------------------------------------------ launch

#ifndef GSA_DKV_PERSIST
#define GSA_DKV_PERSIST 1
#endif
#ifndef GSA_DQ_PERSIST
#define GSA_DQ_PERSIST 1
#endif

// Streaming multiprocessors of the current device (cached per device).
inline int sm_count() {
    static std::atomic<int> cached[64] = {};   // calls may come from several host threads
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

template <int D, bool K4>
gsa_status launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                    const __nv_bfloat16* o, const __nv_bfloat16* dO, const TokLayout& lo, Params pq, Params pkv,
                    int S, int H, int nblk, cudaStream_t st) {
    const bool persist_q = D == 64 && GSA_DQ_PERSIST, persist_kv = D == 64 && GSA_DKV_PERSIST;
    if (!(persist_q ? smem_opt_in(dq_persist_kernel<K4>, DqPCfg::kSmemBytes)
                    : smem_opt_in(dq_kernel<D, K4>, DqCfg<D>::kSmemBytes)) ||
        !(persist_kv ? smem_opt_in(dkdv_persist_kernel<K4>, DkvPCfg::kSmemBytes)
                     : smem_opt_in(dkdv_kernel<D, K4>, DkvCfg<D>::kSmemBytes)))
        return GSA_ERR_CUDA;
    constexpr int kRowsPerCta = GSA_DOT_ROWS * 256 / (D / 8);   // 32 or 16 rows a thread row group: divides L
    static_assert(64 % kRowsPerCta == 0, "rows per CTA divide a 64-token block");
    const int sh_grid = S * H < 65535 ? S * H : 65535;
    dot_kernel<D><<<dim3(static_cast<unsigned>(pq.L / kRowsPerCta), static_cast<unsigned>(sh_grid)), 256, 0, st>>>(
        o, dO, lo, pq.L, pq.H, S * H, const_cast<float*>(pq.ndvec), pq.lse, const_cast<float*>(pq.nlse2), pkv.ticket);
    dim3 grid(S * H, (nblk + 1) / 2);
    if (persist_q) {
        const int64_t items = static_cast<int64_t>(S) * H * ((nblk + 1) / 2);
        const int64_t ctas = items < 2 * sm_count() ? items : 2 * sm_count();
        dq_persist_kernel<K4><<<static_cast<unsigned>(ctas), DqPCfg::kThreads, DqPCfg::kSmemBytes, st>>>(tq, tk, tv,
                                                                                                         tdo, pq);
    } else {
        dq_kernel<D, K4><<<grid, Shape<D>::kThreads, DqCfg<D>::kSmemBytes, st>>>(tq, tk, tv, tdo, pq);
    }
    if (persist_kv) {   // one CTA per SM, double-buffered scores
        const int64_t items = static_cast<int64_t>(S) * H * ((nblk + 1) / 2);
        const int64_t ctas = items < sm_count() ? items : sm_count();
        dkdv_persist_kernel<K4><<<static_cast<unsigned>(ctas), DkvPCfg::kThreads, DkvPCfg::kSmemBytes, st>>>(
            tq, tk, tv, tdo, pkv);
    } else {
        dkdv_kernel<D, K4><<<grid, Shape<D>::kThreads, DkvCfg<D>::kSmemBytes, st>>>(tq, tk, tv, tdo, pkv);
    }
    return cudaGetLastError() == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

inline gsa_status launch(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                         const gsa_block_csr* csr, const gsa_attn_desc* desc, const uint8_t* cls, float scale,
                         void* dq, void* dk, void* dv, float* work, const TokLayout& lq, const TokLayout& lo,
                         cudaStream_t st) {
    if ((reinterpret_cast<uintptr_t>(lse) & 15u) || (reinterpret_cast<uintptr_t>(work) & 15u))
        return GSA_ERR_INVALID_ARGUMENT;
    const int64_t rows = static_cast<int64_t>(desc->B) * desc->H * desc->L;
    // one load kind for all four inputs: 2-D maps only when every one is dense
    const bool k4 = !is_dense(lq, desc->d, desc->L, desc->H) || !is_dense(lo, desc->d, desc->L, desc->H);
    CUtensorMap tq, tk, tv, tdo;
    if (!make_tmap_tok(&tq, q, desc->d, desc->L, desc->H, desc->B, lq, k4) ||
        !make_tmap_tok(&tk, k, desc->d, desc->L, desc->H, desc->B, lq, k4) ||
        !make_tmap_tok(&tv, v, desc->d, desc->L, desc->H, desc->B, lq, k4) ||
        !make_tmap_tok(&tdo, dO, desc->d, desc->L, desc->H, desc->B, lo, k4))
        return GSA_ERR_CUDA;
    Params base{};
    base.lq = lq;
    base.cap = csr->capacity;
    base.S = desc->B;
    base.H = desc->H;
    base.nblk = csr->nblk;
    base.L = desc->L;
    base.lse = lse;
    base.nlse2 = work + ((rows + 63) & ~int64_t(63));   // after -D, 256-byte aligned
    base.ndvec = work;
    base.scale = scale;
    base.scale_log2 = scale * kLog2e;
    base.ticket = reinterpret_cast<int*>(work + 2 * ((rows + 63) & ~int64_t(63)));   // after D and LSE2
    for (int h = 0; h < desc->H; ++h) base.cls[h] = cls[h];
    base.local_implicit = (csr->classes >> 3) & 1;
    base.w = csr->w;
    Params pq = base, pkv = base;
    pq.ticket = base.ticket + 1;
    pq.ptr = csr->row_ptr;
    pq.idx = csr->col_idx;
    pq.order = csr->q_order;
    pq.out0 = static_cast<__nv_bfloat16*>(dq);
    pq.out1 = nullptr;
    pkv.ptr = csr->col_ptr;
    pkv.idx = csr->row_idx;
    pkv.order = csr->k_order;
    pkv.out0 = static_cast<__nv_bfloat16*>(dv);
    pkv.out1 = static_cast<__nv_bfloat16*>(dk);
    const auto* ob = static_cast<const __nv_bfloat16*>(o);
    const auto* dob = static_cast<const __nv_bfloat16*>(dO);
    if (desc->d == 64)
        return k4 ? launch_d<64, true>(tq, tk, tv, tdo, ob, dob, lo, pq, pkv, desc->B, desc->H, csr->nblk, st)
                  : launch_d<64, false>(tq, tk, tv, tdo, ob, dob, lo, pq, pkv, desc->B, desc->H, csr->nblk, st);
    return k4 ? launch_d<128, true>(tq, tk, tv, tdo, ob, dob, lo, pq, pkv, desc->B, desc->H, csr->nblk, st)
              : launch_d<128, false>(tq, tk, tv, tdo, ob, dob, lo, pq, pkv, desc->B, desc->H, csr->nblk, st);
}

}  // namespace bwd
}  // namespace gsa
