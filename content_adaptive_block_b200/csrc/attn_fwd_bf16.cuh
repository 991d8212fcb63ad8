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
// Roles (64 + 128 G threads):
//   thread 0 issues the TMA load of Q as soon as the barriers exist, so it
//           overlaps the merge of the key lists;
//   warp 0  one thread issues the TMA loads of K and V of each key tile
//           into a ring of shared-memory stages;
//   warp 1  allocates TMEM; one thread issues every MMA of the CTA, in tile
//           order, as soon as its operands are ready:
//             S[g][b] = Q K^T   (M=128, N=64, K=d;  A and B from shared memory)
//             O_g    += P_g V   (M=128, N=d,  K=64; A = P from TMEM, B = V)
//           The QK^T of a tile needs its K/V stage and a free S buffer of its
//           group; with two S buffers per group it runs while the group's
//           softmax works on the previous tile.
//   warps 2..  softmax, G warpgroups; group g takes the tiles n with
//           n % G == g, one thread per query row (TMEM lane), all 64 key
//           columns.  Each group keeps its own running max m_g, row sum l_g
//           and accumulator O_g = Σ P V over its tiles (split-key online
//           softmax).  O_g is rescaled in TMEM only when m_g grows by more
//           than 8 (log2 units): exact for any reference max, the threshold
//           bounds P <= 256.  P goes to TMEM as packed bf16 pairs (lane =
//           query row, column c = key columns 2c, 2c+1: the layout of an
//           M=128 A operand in TMEM), so it never passes through shared
//           memory.  With G = 2 the halves combine at the end:
//           m = max(m_0, m_1), O = Σ_g O_g 2^(m_g - m) / Σ_g l_g 2^(m_g - m).
// d = 64 runs one softmax group per CTA with two S buffers and two CTAs per
// SM; d = 128 runs two groups with one S buffer each in one CTA per SM.
//
// Shared memory (128-byte swizzle, 1024-byte aligned):
//   Q  [d/64 column atoms][128 rows][128 B]
//   K  stage [d/64 atoms][64 rows][128 B]          (B operand, K-major)
//   V  stage [d/64 atoms][64 rows][128 B]          (B operand, MN-major)
// TMEM (lanes = query rows): S[g][b] at columns 64 (g NS + b), O_g at
// 64 G NS + g d, P_g (32 columns) after the O accumulators.
#pragma once

#include "common.cuh"
#include "tiles.cuh"

namespace gsa {
namespace bf16 {

constexpr int kMaxHeads = 256;
constexpr int kMaxBlocks = 2048;
constexpr int kBlk = 64;   // block size in tokens
constexpr float kRescaleThreshold = 8.0f;   // log2 units

#ifndef GSA_FWD64_GROUPS
#define GSA_FWD64_GROUPS 1
#endif
#ifndef GSA_FWD64_SBUF
#define GSA_FWD64_SBUF 2
#endif
#ifndef GSA_FWD64_CTAS_PER_SM
#define GSA_FWD64_CTAS_PER_SM 2
#endif
// K/V ring depth (one stage = one 64-key block of K and of V).
#ifndef GSA_FWD64_STAGES
#define GSA_FWD64_STAGES 5
#endif
// d = 64 through the persistent kernel (attn_fwd_persist.cuh).
#ifndef GSA_FWD_PERSIST
#define GSA_FWD_PERSIST 1
#endif
#ifndef GSA_FWD128_STAGES
#define GSA_FWD128_STAGES 5
#endif

template <int D>
struct FwdShape {
    static constexpr int kGroups = D == 64 ? GSA_FWD64_GROUPS : 2;
    static constexpr int kSBuf = D == 64 ? GSA_FWD64_SBUF : 1;   // S buffers per group
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
    TokLayout lo;       // layout of o
    float* lse;
    float scale_log2;   // softmax scale * log2(e)
    int* ticket;        // persistent kernel: work counter, CTAs finished (both zero at launch)
    uint8_t cls[kMaxHeads];
    int local_implicit;   // the local class's lists are not stored: derived from (nblk, w)
    int w;                // the lists' window
};

template <int D>
struct FwdCfg {
    static constexpr int G = FwdShape<D>::kGroups;
    static constexpr int NS = FwdShape<D>::kSBuf;
    static constexpr int kAtoms = D / 64;
    static constexpr int kStages = D == 64 ? GSA_FWD64_STAGES : GSA_FWD128_STAGES;
    static constexpr int kQBytes = 128 * D * 2;
    static constexpr int kKVBytes = kBlk * D * 2;   // one block of K (or V)
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + kStages * kKVBytes;
    static constexpr int kOffBar = kOffV + kStages * kKVBytes;
    // barriers: full[st], empty[st], q_full, done, s_full[G][NS], s_free[G][NS], p_full[G], p_free[G]
    static constexpr int kNumBars = 2 * kStages + 2 + 2 * G * NS + 2 * G;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;   // tmem base, abort, ntiles
    static constexpr int kOffList = kOffMisc + 16;            // int16 key block per tile
    static constexpr int kOffLive = kOffList + kMaxBlocks * 2;
    static constexpr int kOffBits = kOffLive + kMaxBlocks;    // two bitmaps
    static constexpr int kOffMl = kOffBits + 2 * (kMaxBlocks / 32) * 4;   // [G group][2][128]: m_g, l_g
    static constexpr int kEnd = kOffMl + G * 2 * 128 * 4;
    static constexpr int kSmemBytes = kEnd + 1024;            // + alignment slack
    static_assert(kSmemBytes <= 232448 / FwdShape<D>::kCtasPerSm - 1024, "shared memory per SM");
    static constexpr int kTmemS = 0;                  // S[g][b] at 64 (g NS + b)
    static constexpr int kTmemO = 64 * G * NS;        // O_g at kTmemO + g D
    static constexpr int kTmemP = kTmemO + G * D;     // P_g at kTmemP + 32 g
    static constexpr int kTmemNeed = kTmemP + 32 * G;
    static constexpr int kTmemCols = kTmemNeed <= 128 ? 128 : (kTmemNeed <= 256 ? 256 : 512);
    static_assert(kTmemCols * FwdShape<D>::kCtasPerSm <= 512, "TMEM per SM");
};

template <int D, bool K4>   // K4: strided tensors through 4-D maps (see load_rows)
__global__ void __launch_bounds__(FwdShape<D>::kThreads, FwdShape<D>::kCtasPerSm)
attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using C = FwdCfg<D>;
    constexpr int G = C::G, NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::kStages;
    uint64_t* q_full = bars + 2 * C::kStages;
    uint64_t* done = q_full + 1;        // one phase: every product of the CTA completed
    uint64_t* s_full = done + 1;        // [G][NS] QK^T landed in S[g][b]
    uint64_t* s_free = s_full + G * NS; // [G][NS] the group read S[g][b]
    uint64_t* p_full = s_free + G * NS; // [G] the group's P is in TMEM
    uint64_t* p_free = p_full + G;      // [G] the group's P V completed
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
    const bool implicit = c == 0 && p.local_implicit;
    const int32_t* ord = implicit ? nullptr : p.q_order + g * nblk;
    const int qa = order_at(ord, 2 * tile);
    const int qb = (2 * tile + 1 < nblk) ? order_at(ord, 2 * tile + 1) : -1;
    const int nwords = (nblk + 31) >> 5;
    const int64_t head_row0 = static_cast<int64_t>(sh) * p.L;   // row of this (s, h)'s first token (LSE index)

    // ---- set-up: barriers, TMEM, merged key list
    if (threadIdx.x == 0) {
        for (int st = 0; st < C::kStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(done, 1);
        for (int i = 0; i < G * NS; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], 128);
        }
        for (int i = 0; i < G; ++i) {
            mbar_init(&p_full[i], 128);
            mbar_init(&p_free[i], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        // Q of the tile: needs only qa and qb, so it loads while the key lists merge
        mbar_arrive_expect_tx(q_full, (qb >= 0 ? 2 : 1) * kBlk * D * 2);
        for (int half = 0; half < 2; ++half) {
            const int blk = half ? qb : qa;
            if (blk < 0) continue;
            const int l0 = blk * kBlk;   // token coordinate in the (sample, head)
            for (int at = 0; at < C::kAtoms; ++at)
                load_rows<K4>(sQ + at * (128 * 128) + half * (kBlk * 128), &tmQ, q_full, at * 64, l0, h, s, head_row0);
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
        const ListRef rows{implicit ? nullptr : p.row_ptr + g * (nblk + 1), p.col_idx + g * p.cap, p.w, nblk, false};
        rows.each(qa, threadIdx.x, blockDim.x, [&](int j) { atomicOr(&bitsA[j >> 5], 1u << (j & 31)); });
        if (qb >= 0) rows.each(qb, threadIdx.x, blockDim.x, [&](int j) { atomicOr(&bitsB[j >> 5], 1u << (j & 31)); });
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
        if (lane == 31) *ntiles_slot = incl;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int T = *ntiles_slot;
    const uint32_t tmem = *tmem_slot;
    int fills = 0;          // producer: K / V stages issued
    int issued_qk = 0, issued_pv = 0;   // MMA thread: QK^T and P V products issued

    if (warp == 0) {
        // ================= TMA producer
        if (lane == 0) {
            int n = 0;
            for (; n < T; ++n) {
                const int st = n % C::kStages;
                if (n >= C::kStages) {
                    if (!mbar_wait(&empty[st], ((n / C::kStages) - 1) & 1, abort_flag, kErrTimeoutProducer)) break;
                }
                mbar_arrive_expect_tx(&full[st], 2 * C::kKVBytes);
                const int l0 = list[n] * kBlk;   // token coordinate in the (sample, head)
                uint8_t* dk = sK + st * C::kKVBytes;
                uint8_t* dv = sV + st * C::kKVBytes;
                for (int at = 0; at < C::kAtoms; ++at) {
                    load_rows<K4>(dk + at * (kBlk * 128), &tmK, &full[st], at * 64, l0, h, s, head_row0);
                    load_rows<K4>(dv + at * (kBlk * 128), &tmV, &full[st], at * 64, l0, h, s, head_row0);
                }
            }
            fills = n;
        }
    } else if (warp == 1) {
        // ================= MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(128, kBlk, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(128, D, 1);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
            // Q is waited for even without tiles: no load may be in flight at exit
            bool ok = mbar_wait(q_full, 0, abort_flag, kErrTimeoutMma);
            // Both streams advance in tile order: QK^T of tile ns (group ns % G,
            // its k-th, S buffer k % NS) once its K/V stage is loaded and the
            // group has read that buffer's previous scores; P V of tile na once
            // the group's P is in TMEM.
            int ns = 0, na = 0;   // QK^T and P V products issued
            PollGuard guard;
            while (ok && na < T) {
                bool moved = false;
                if (ns < T) {
                    const int st = ns % C::kStages;
                    const int gq = ns % G, kq = ns / G, sb = gq * NS + kq % NS;
                    if (mbar_test(&full[st], (ns / C::kStages) & 1) &&
                        (kq < NS || mbar_test(&s_free[sb], ((kq - NS) / NS) & 1))) {
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const int at = kk >> 2, ko = (kk & 3) * 32;
                            const uint64_t ad = sdesc_sw128(aQ + at * (128 * 128) + ko, 16, 1024);
                            const uint64_t bd =
                                sdesc_sw128(aK + st * C::kKVBytes + at * (kBlk * 128) + ko, 16, 1024);
                            umma_bf16(tmem + C::kTmemS + 64 * sb, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(&s_full[sb]);
                        ++ns;
                        moved = true;
                    }
                }
                if (na < ns) {
                    const int st = na % C::kStages;
                    const int gp = na % G, kp = na / G;
                    if (mbar_test(&p_full[gp], kp & 1)) {
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < kBlk / 16; ++kk) {
                            const uint64_t bd =
                                sdesc_sw128(aV + st * C::kKVBytes + kk * (16 * 128), kBlk * 128, 1024);
                            umma_bf16_ts(tmem + C::kTmemO + gp * D, tmem + C::kTmemP + 32 * gp + kk * 8, bd,
                                         idesc_pv, (kp > 0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit(&p_free[gp]);
                        umma_commit(&empty[st]);
                        ++na;
                        moved = true;
                    }
                }
                if (moved) guard.progress();
                else if (guard.stalled(abort_flag, kErrTimeoutMma)) ok = false;
            }
            if (ok && T > 0) umma_commit(done);
            issued_qk = ns;
            issued_pv = na;
        }
        __syncwarp();
    } else {
        // ================= softmax warpgroups (warps 2..)
        const int quad = warp & 3;              // TMEM lane quadrant this warp may access
        const int grp = (warp - 2) >> 2;        // this group takes the tiles n % G == grp
        const int r = quad * 32 + lane;         // query row in the tile = TMEM lane
        const int half = r >> 6;
        const int my_blk = half ? qb : qa;
        const int rr = r & 63;
        const uint32_t tl = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const uint32_t tO = tl + C::kTmemO + grp * D;
        const uint32_t tP = tl + C::kTmemP + 32 * grp;
        float m = -INFINITY, l = 0.f;           // this group's running max and sum
        bool ok = true;
        for (int n = grp, k = 0; n < T; n += G, ++k) {
            const int sb = grp * NS + k % NS;
            const uint32_t tS = tl + C::kTmemS + 64 * sb;
            if (!__all_sync(0xffffffffu, mbar_wait(&s_full[sb], (k / NS) & 1, abort_flag, kErrTimeoutSoftmax))) {
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
            // the scores are in registers: S[grp][b] may take the group's next QK^T
            tc_fence_before();
            mbar_arrive(&s_free[sb]);

            // P_grp and O_grp were last used by the P V product of the group's
            // previous tile
            if (k >= 1 &&
                !__all_sync(0xffffffffu, mbar_wait(&p_free[grp], (k - 1) & 1, abort_flag, kErrTimeoutSoftmax))) {
                ok = false;
                break;
            }
            tc_fence_after();
            tmem_st32u(tP, pk);
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
            __nv_bfloat16* orow = p.o + (K4 ? tok_off(tok, p.L, p.H, p.lo) : tok * D);
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
    if (*abort_flag) {
        // a role gave up a wait: the loads and products issued must land before
        // shared memory and TMEM go (without one, every one of them was waited for)
        if (warp == 0 && lane == 0) drain_fills(full, C::kStages, fills);
        if (warp == 1 && lane == 0) {
            // tcgen05 products complete in issue order: the phases the last QK^T
            // and the last P V committed cover every earlier one
            mbar_wait_drain(q_full, 0);
            if (issued_qk > 0) {
                const int n = issued_qk - 1, kq = n / G;
                mbar_wait_drain(&s_full[(n % G) * NS + kq % NS], (kq / NS) & 1);
            }
            if (issued_pv > 0) {
                const int n = issued_pv - 1;
                mbar_wait_drain(&p_free[n % G], (n / G) & 1);
            }
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace bf16
}  // namespace gsa

#include "attn_fwd_persist.cuh"
