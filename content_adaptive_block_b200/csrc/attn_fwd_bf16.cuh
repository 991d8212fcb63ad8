// Block-sparse causal attention forward, bf16 in / fp32 accumulate, on the
// 5th-generation tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// Gzip-guided Sparse Attention (daiwk.github.io), section "复现边界": the
// reproduction forms the dense score matrix and masks it, so the sparsity
// buys no time.  Here only live (query block, key block) pairs are computed:
// section "核心公式" gives the mask, the CSR rows list the live key blocks.
//
// Work unit (one CTA): 128 query rows = two query blocks of 64 tokens (qa,
// qb), taken from the class's pairing order, of one (sample, head).  The key
// tiles are the union of the two CSR rows (merged through a bitmap), each
// one key block of 64 tokens.  Rows of a half whose block is not live for a
// key tile are masked out of it; the diagonal block gets the token causal cut.
//
// Roles (320 threads):
//   thread 0 issues the TMA load of Q as soon as the barriers exist, so it
//           overlaps the merge of the key lists;
//   warp 0  one thread issues the TMA loads of K and V of each key tile
//           into a ring of shared-memory stages;
//   warp 1  allocates TMEM;
//   warps 2-9  softmax, two warpgroups; group g takes the tiles n with
//           n % 2 == g, one thread per query row (TMEM lane), all 64 key
//           columns.  Each group keeps its own running max m_g, row sum l_g
//           and accumulator O_g = Σ P V over its tiles (split-key online
//           softmax), so the groups run independently and their exp2 (MUFU)
//           and ALU phases overlap.  O_g is rescaled in TMEM only when m_g
//           grows by more than 8 (log2 units): exact for any reference max,
//           the threshold bounds P <= 256.  P goes back to TMEM as packed
//           bf16 pairs over the first 32 columns of S[g] (lane = query row,
//           column c = key columns 2c, 2c+1: the layout of an M=128 A operand
//           in TMEM), so it never passes through shared memory.  The
//           tensor pipe runs one thread's MMAs in issue order, so the QK^T of
//           tile n+2 may overwrite S[g] once the P V of tile n is issued.
//           One thread of each group issues that group's MMAs,
//             S[g]  = Q K^T   (M=128, N=64, K=d;  A and B from shared memory)
//             O_g  += P V     (M=128, N=d,  K=64; A = P from TMEM, B = V),
//           right after the group's 128 rows of P are in TMEM: two
//           independent MMA streams per CTA, and every product a group's
//           rows read was issued (so ordered and tracked) by one thread.
//           At the end the two halves combine:
//           m = max(m_0, m_1), O = Σ_g O_g 2^(m_g - m) / Σ_g l_g 2^(m_g - m).
// The QK^T of tile n+1 overlaps the softmax of tile n.
//
// Shared memory (128-byte swizzle, 1024-byte aligned):
//   Q  [d/64 column atoms][128 rows][128 B]
//   K  stage [d/64 atoms][64 rows][128 B]          (B operand, K-major)
//   V  stage [d/64 atoms][64 rows][128 B]          (B operand, MN-major)
// TMEM (lanes = query rows): S[0], S[1] at columns 0 and 64 (P over their
// first 32 columns), O_0 and O_1 at columns 128 and 128 + d.
#pragma once

#include "common.cuh"
#include "tiles.cuh"

namespace gsa {
namespace bf16 {

constexpr int kMaxHeads = 256;
constexpr int kMaxBlocks = 2048;
constexpr int kBlk = 64;   // block size in tokens
constexpr float kRescaleThreshold = 8.0f;   // log2 units
// Softmax warpgroups: group g owns the tiles n with n % G == g.  d = 64
// runs one group per CTA and three CTAs per SM (128 TMEM columns each), so
// CTAs overlap each other's set-up and epilogue; d = 128 runs two groups in
// one CTA per SM.
#ifndef GSA_FWD64_GROUPS
#define GSA_FWD64_GROUPS 1
#endif
#ifndef GSA_FWD64_CTAS_PER_SM
#define GSA_FWD64_CTAS_PER_SM (GSA_FWD64_GROUPS == 1 ? 3 : 2)
#endif
template <int D>
struct FwdShape {
    static constexpr int kGroups = D == 64 ? GSA_FWD64_GROUPS : 2;
    static constexpr int kThreads = 64 + 128 * kGroups;
    static constexpr int kCtasPerSm = D == 64 ? GSA_FWD64_CTAS_PER_SM : 1;
};

// Named barrier (ids 1..4) joining the two warps that share a TMEM lane quadrant.
__device__ __forceinline__ void pair_barrier(int quad) {
    switch (quad) {
        case 0: asm volatile("bar.sync 1, 64;" ::: "memory"); break;
        case 1: asm volatile("bar.sync 2, 64;" ::: "memory"); break;
        case 2: asm volatile("bar.sync 3, 64;" ::: "memory"); break;
        default: asm volatile("bar.sync 4, 64;" ::: "memory"); break;
    }
}

struct FwdParams {
    const int32_t* row_ptr;
    const int32_t* col_idx;
    const int32_t* q_order;
    int64_t cap;
    int S, H, nblk;
    int64_t L;
    __nv_bfloat16* o;
    float* lse;
    float scale_log2;   // softmax scale * log2(e)
    uint8_t cls[kMaxHeads];
};

// K/V ring depth (one stage = one 64-key block of K and of V).
#ifndef GSA_FWD64_STAGES
#define GSA_FWD64_STAGES (GSA_FWD64_GROUPS == 1 ? 3 : 5)
#endif
#ifndef GSA_FWD128_STAGES
#define GSA_FWD128_STAGES 5
#endif

template <int D>
struct FwdCfg {
    static constexpr int G = FwdShape<D>::kGroups;
    static constexpr int kAtoms = D / 64;
    static constexpr int kStages = D == 64 ? GSA_FWD64_STAGES : GSA_FWD128_STAGES;
    static constexpr int kQBytes = 128 * D * 2;
    static constexpr int kKVBytes = kBlk * D * 2;   // one block of K (or V)
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + kStages * kKVBytes;
    static constexpr int kOffBar = kOffV + kStages * kKVBytes;
    // barriers: full[st], empty[st], q_full, s_full[2], p_full[2], done
    static constexpr int kNumBars = 2 * kStages + 6;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;   // tmem base, abort, ntiles
    static constexpr int kOffList = kOffMisc + 16;            // int16 key block per tile
    static constexpr int kOffLive = kOffList + kMaxBlocks * 2;
    static constexpr int kOffBits = kOffLive + kMaxBlocks;    // two bitmaps
    static constexpr int kOffMl = kOffBits + 2 * (kMaxBlocks / 32) * 4;   // [G group][2][128]: m_g, l_g
    static constexpr int kEnd = kOffMl + G * 2 * 128 * 4;
    static constexpr int kSmemBytes = kEnd + 1024;            // + alignment slack
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kSmemBytes <= 232448 / FwdShape<D>::kCtasPerSm - 1024, "shared memory per SM");
    static constexpr int kTmemS = 0;       // S[g] at columns 64 g
    static constexpr int kTmemO = 64 * G;  // O_g at columns 64 G + g D
    static constexpr int kTmemNeed = kTmemO + G * D;
    static constexpr int kTmemCols = kTmemNeed <= 128 ? 128 : (kTmemNeed <= 256 ? 256 : 512);
    static_assert(kTmemCols * FwdShape<D>::kCtasPerSm <= 512, "TMEM per SM");
};

template <int D>
__global__ void __launch_bounds__(FwdShape<D>::kThreads, FwdShape<D>::kCtasPerSm)
attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::kStages;
    uint64_t* q_full = bars + 2 * C::kStages;
    uint64_t* s_full = q_full + 1;
    uint64_t* p_full = s_full + 2;
    uint64_t* done = p_full + 2;    // one phase: every product of the CTA completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    int* ntiles_slot = reinterpret_cast<int*>(smem + C::kOffMisc + 8);
    int16_t* list = reinterpret_cast<int16_t*>(smem + C::kOffList);
    uint8_t* live = smem + C::kOffLive;
    uint32_t* bitsA = reinterpret_cast<uint32_t*>(smem + C::kOffBits);
    uint32_t* bitsB = bitsA + kMaxBlocks / 32;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sh = blockIdx.x;          // s * H + h
    const int s = sh / p.H, h = sh % p.H;
    const int tile = blockIdx.y;
    const int c = p.cls[h];
    const int nblk = p.nblk;
    const int64_t g = static_cast<int64_t>(s) * 3 + c;
    const int qa = p.q_order[g * nblk + 2 * tile];
    const int qb = (2 * tile + 1 < nblk) ? p.q_order[g * nblk + 2 * tile + 1] : -1;
    const int nwords = (nblk + 31) >> 5;

    // ---- set-up: barriers, TMEM, merged key list
    if (threadIdx.x == 0) {
        for (int st = 0; st < C::kStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        mbar_init(&p_full[0], 128);
        mbar_init(&p_full[1], 128);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        // Q of the tile: needs only qa and qb, so it loads while the key lists merge
        const int64_t row0 = static_cast<int64_t>(sh) * p.L;
        mbar_arrive_expect_tx(q_full, (qb >= 0 ? 2 : 1) * kBlk * D * 2);
        for (int half = 0; half < 2; ++half) {
            const int blk = half ? qb : qa;
            if (blk < 0) continue;
            const int row = static_cast<int>(row0 + static_cast<int64_t>(blk) * kBlk);
            for (int at = 0; at < C::kAtoms; ++at)
                tma_load_2d(sQ + at * (128 * 128) + half * (kBlk * 128), &tmQ, q_full, at * 64, row);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    for (int k = threadIdx.x; k < nwords; k += blockDim.x) {
        bitsA[k] = 0u;
        bitsB[k] = 0u;
    }
    __syncthreads();
    {
        const int32_t* rp = p.row_ptr + g * (nblk + 1);
        const int32_t* ci = p.col_idx + g * p.cap;
        const int a0 = rp[qa], a1 = rp[qa + 1];
        for (int e = a0 + threadIdx.x; e < a1; e += blockDim.x) {
            const int j = ci[e];
            atomicOr(&bitsA[j >> 5], 1u << (j & 31));
        }
        if (qb >= 0) {
            const int b0 = rp[qb], b1 = rp[qb + 1];
            for (int e = b0 + threadIdx.x; e < b1; e += blockDim.x) {
                const int j = ci[e];
                atomicOr(&bitsB[j >> 5], 1u << (j & 31));
            }
        }
    }
    __syncthreads();
    if (warp == 0) {
        // ordered compaction of bitsA | bitsB; lane handles a contiguous range of words
        const int per = (nwords + 31) >> 5;
        const int w0 = lane * per, w1 = min(nwords, w0 + per);
        int cnt = 0;
        for (int k = w0; k < w1; ++k) cnt += __popc(bitsA[k] | bitsB[k]);
        int incl = cnt;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int pos = incl - cnt;
        for (int k = w0; k < w1; ++k) {
            uint32_t u = bitsA[k] | bitsB[k];
            while (u) {
                const int bit = __ffs(u) - 1;
                u &= u - 1;
                list[pos] = static_cast<int16_t>(32 * k + bit);
                live[pos] = static_cast<uint8_t>(((bitsA[k] >> bit) & 1u) | (((bitsB[k] >> bit) & 1u) << 1));
                ++pos;
            }
        }
        if (lane == 31) {
            *ntiles_slot = incl;
            mbar_init(done, incl >= C::G ? C::G : 1);   // one arrival per group that has tiles
            fence_mbar_init();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int T = *ntiles_slot;
    const uint32_t tmem = *tmem_slot;
    const int64_t head_row0 = static_cast<int64_t>(sh) * p.L;   // first row of this (s, h) in the 2-D views

    if (warp == 0) {
        // ================= TMA producer
        if (lane == 0) {
            for (int n = 0; n < T; ++n) {
                const int st = n % C::kStages;
                if (n >= C::kStages) {
                    if (!mbar_wait(&empty[st], ((n / C::kStages) - 1) & 1, abort_flag, kErrTimeoutProducer)) break;
                }
                mbar_arrive_expect_tx(&full[st], 2 * C::kKVBytes);
                const int row = static_cast<int>(head_row0 + static_cast<int64_t>(list[n]) * kBlk);
                uint8_t* dk = sK + st * C::kKVBytes;
                uint8_t* dv = sV + st * C::kKVBytes;
                for (int at = 0; at < C::kAtoms; ++at) {
                    tma_load_2d(dk + at * (kBlk * 128), &tmK, &full[st], at * 64, row);
                    tma_load_2d(dv + at * (kBlk * 128), &tmV, &full[st], at * 64, row);
                }
            }
        }
    } else if (warp >= 2) {
        // ================= softmax warpgroups (warps 2..9)
        const int quad = warp & 3;              // TMEM lane quadrant this warp may access
        const int grp = (warp - 2) >> 2;        // this group takes the tiles n % 2 == grp
        const int r = quad * 32 + lane;         // query row in the tile = TMEM lane
        const int half = r >> 6;
        const int my_blk = half ? qb : qa;
        const int rr = r & 63;
        const uint32_t tl = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const uint32_t tS = tl + C::kTmemS + grp * kBlk;
        const uint32_t tO = tl + C::kTmemO + grp * D;
        float m = -INFINITY, l = 0.f;           // this group's running max and sum
        bool ok = true;
        // the group's MMA issuer: lane 0 of its first warp
        const bool issuer_warp = ((warp - 2) & 3) == 0;
        constexpr uint32_t idesc_qk = idesc_bf16(128, kBlk, 0);
        constexpr uint32_t idesc_pv = idesc_bf16(128, D, 1);
        const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
        auto issue_qk = [&](int t) {   // S[grp] = Q K_t^T, then arrive on s_full[grp]
            const int st = t % C::kStages;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int at = kk >> 2, ko = (kk & 3) * 32;
                const uint64_t ad = sdesc_sw128(aQ + at * (128 * 128) + ko, 16, 1024);
                const uint64_t bd = sdesc_sw128(aK + st * C::kKVBytes + at * (kBlk * 128) + ko, 16, 1024);
                umma_bf16(tmem + C::kTmemS + grp * kBlk, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[grp]);
        };
        if (issuer_warp) {
            if (lane == 0 && grp < T) {
                const int st = grp % C::kStages;
                if (mbar_wait(q_full, 0, abort_flag, kErrTimeoutMma) &&
                    mbar_wait(&full[st], (grp / C::kStages) & 1, abort_flag, kErrTimeoutMma)) {
                    tc_fence_after();
                    issue_qk(grp);
                }
            }
            __syncwarp();
        }
        for (int n = grp; n < T; n += C::G) {
            const int ph = (n / C::G) & 1;      // phase of this group's barriers
            if (!__all_sync(0xffffffffu, mbar_wait(&s_full[grp], ph, abort_flag, kErrTimeoutSoftmax))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int j = list[n];
            const bool is_live = (live[n] >> half) & 1;
            const int last = !is_live ? -1 : (j == my_blk ? rr : kBlk - 1);   // visible columns 0..last
            // pass 1: raw-score maximum (the scale is positive)
            float mt = -INFINITY;
            if (last >= 0) {
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    float v[32];
                    tmem_ld32(tS + 32 * ch, v);
                    tmem_wait_ld();
                    if (last < 32 * ch + 31) {
#pragma unroll
                        for (int cc = 0; cc < 32; ++cc) v[cc] = 32 * ch + cc <= last ? v[cc] : -INFINITY;
                    }
                    mt = fmaxf(mt, max_reduce<32>(v));
                }
            }
            mt *= p.scale_log2;
            const float m_new = fmaxf(m, mt);
            float alpha = 1.f;
            bool rescale = false;
            float m_use = m;
            if (m == -INFINITY) {
                m_use = m_new;
            } else if (m_new > m + kRescaleThreshold) {
                m_use = m_new;
                alpha = ex2(m - m_new);
                rescale = true;
            }
            const float msafe = m_use == -INFINITY ? 0.f : m_use;
            // pass 2: p = 2^(s * scale * log2 e - m), packed to bf16
            uint32_t pk[32];
            float sum = 0.f;
            if (last < 0) {
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = 0u;
            } else {
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    float v[32];
                    tmem_ld32(tS + 32 * ch, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int cc = 0; cc < 32; ++cc) v[cc] = ex2(fmaf(v[cc], p.scale_log2, -msafe));
                    if (last < 32 * ch + 31) {
#pragma unroll
                        for (int cc = 0; cc < 32; ++cc) v[cc] = 32 * ch + cc <= last ? v[cc] : 0.f;
                    }
                    sum += sum_reduce<32>(v);
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[16 * ch + e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
                }
            }
            l = l * alpha + sum;
            m = m_use;

            // P over the first 32 columns of S[grp] (both score chunks were
            // loaded and waited for above).  O_grp is free to rescale: the
            // QK^T of this tile completed, and with it every earlier product.
            tmem_st32u(tS, pk);
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int cb = 0; cb < D; cb += 32) {
                    float ov[32];
                    tmem_ld32(tO + cb, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] *= alpha;
                    tmem_st32(tO + cb, ov);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[grp]);
            if (issuer_warp) {
                if (lane == 0 && mbar_wait(&p_full[grp], ph, abort_flag, kErrTimeoutMma)) {
                    // O_grp += P V (P read from S[grp]), then the next QK^T into S[grp]
                    tc_fence_after();
                    const int st = n % C::kStages;
#pragma unroll
                    for (int kk = 0; kk < kBlk / 16; ++kk) {
                        const uint64_t bd = sdesc_sw128(aV + st * C::kKVBytes + kk * (16 * 128), kBlk * 128, 1024);
                        umma_bf16_ts(tmem + C::kTmemO + grp * D, tmem + C::kTmemS + grp * kBlk + kk * 8, bd,
                                     idesc_pv, (n >= C::G || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[st]);
                    if (n + C::G < T) {
                        if (mbar_wait(&full[(n + C::G) % C::kStages], ((n + C::G) / C::kStages) & 1, abort_flag,
                                      kErrTimeoutMma)) {
                            tc_fence_after();
                            issue_qk(n + C::G);
                        }
                    } else {
                        umma_commit(done);
                    }
                }
                __syncwarp();
            }
        }
        // combine the groups: exchange (m_g, l_g) through shared memory
        float m0 = m, l0 = l, m1 = -INFINITY, l1 = 0.f;
        if constexpr (C::G == 2) {
            float* ml = reinterpret_cast<float*>(smem + C::kOffMl);
            ml[(grp * 2 + 0) * 128 + r] = m;
            ml[(grp * 2 + 1) * 128 + r] = l;
            pair_barrier(quad);
            m0 = ml[0 * 128 + r];
            l0 = ml[1 * 128 + r];
            m1 = ml[2 * 128 + r];
            l1 = ml[3 * 128 + r];
        }
        // every product of the CTA completed (a single-phase barrier: the other
        // group's buffer barriers may be more than one phase behind)
        if (ok && T > 0 && __all_sync(0xffffffffu, mbar_wait(done, 0, abort_flag, kErrTimeoutSoftmax))) {
            tc_fence_after();
            const bool has1 = C::G == 2 && T >= 2;   // O_1 holds products only if group 1 had a tile
            const float mm = fmaxf(m0, has1 ? m1 : -INFINITY);
            const float w0 = m0 == -INFINITY ? 0.f : ex2(m0 - mm);
            const float w1 = (!has1 || m1 == -INFINITY) ? 0.f : ex2(m1 - mm);
            const float lt = l0 * w0 + l1 * w1;
            const float inv = 1.f / lt;
            const bool store = my_blk >= 0;
            const int64_t tok = head_row0 + static_cast<int64_t>(store ? my_blk : 0) * kBlk + rr;
            __nv_bfloat16* orow = p.o + tok * D;
#pragma unroll
            for (int cb = grp * (D / C::G); cb < (grp + 1) * (D / C::G); cb += 32) {
                float a[32];
                tmem_ld32(tl + C::kTmemO + cb, a);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) a[e] *= w0;
                if (has1) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float b2[16];
                        tmem_ld16(tl + C::kTmemO + D + cb + 16 * hh, b2);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) a[16 * hh + e] = fmaf(b2[e], w1, a[16 * hh + e]);
                    }
                }
                if (store) store_scaled_bf16(orow + cb, a, inv);
            }
            if (store && grp == 0 && p.lse) p.lse[tok] = (mm + log2f(lt)) * 0.69314718055994531f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace bf16
}  // namespace gsa
