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
// Roles (192 threads):
//   warp 0  one thread issues TMA loads: Q (once), then K and V of each key
//           tile into a ring of shared-memory stages;
//   warp 1  allocates TMEM; one thread issues the MMAs:
//             S[buf] = Q K^T       (M=128, N=64,  K=d;   double-buffered S)
//             O     += P V         (M=128, N=d,   K=64;  O accumulates in TMEM)
//   warps 2-5  softmax: thread = query row = TMEM lane; reads S, applies the
//           mask and scale, keeps the running max m and sum l, writes P
//           (bf16, 128-byte swizzled, the MMA's A layout) to shared memory,
//           and rescales O in TMEM when m grows by more than 2^8 (the
//           result is exact for any reference max; the threshold only bounds
//           P <= 256).  At the end O / l and the LSE are written out.
// The QK^T of tile n+1 overlaps the softmax of tile n.
//
// Shared memory (128-byte swizzle, 1024-byte aligned):
//   Q  [d/64 column atoms][128 rows][128 B]
//   K  stage [d/64 atoms][64 rows][128 B]          (B operand, K-major)
//   V  stage [d/64 atoms][64 rows][128 B]          (B operand, MN-major)
//   P  [128 rows][128 B]                           (A operand, K-major)
#pragma once

#include "common.cuh"
#include "tiles.cuh"

namespace gsa {
namespace bf16 {

constexpr int kMaxHeads = 256;
constexpr int kMaxBlocks = 2048;
constexpr int kBlk = 64;   // block size in tokens
constexpr float kRescaleThreshold = 8.0f;   // log2 units
// Softmax warpgroups: the two threads of a row (one per group) own 32 of the
// tile's 64 key columns each and exchange their partial row maxima.
constexpr int kSmGroups = 2;
constexpr int kCw = kBlk / kSmGroups;
constexpr int kSmThreads = 128 * kSmGroups;
constexpr int kFwdThreads = 64 + kSmThreads;

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

// K/V ring depth (one stage = one 64-key block of K and of V), and CTAs per
// SM for d = 64 (two CTAs overlap each other's hand-offs).
#ifndef GSA_FWD64_STAGES
#define GSA_FWD64_STAGES 4
#endif
#ifndef GSA_FWD128_STAGES
#define GSA_FWD128_STAGES 3
#endif
#ifndef GSA_FWD64_CTAS_PER_SM
#define GSA_FWD64_CTAS_PER_SM 2
#endif

template <int D>
struct FwdCfg {
    static constexpr int kAtoms = D / 64;
    static constexpr int kStages = D == 64 ? GSA_FWD64_STAGES : GSA_FWD128_STAGES;
    static constexpr int kQBytes = 128 * D * 2;
    static constexpr int kKVBytes = kBlk * D * 2;   // one block of K (or V)
    static constexpr int kPBytes = 128 * kBlk * 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + kStages * kKVBytes;
    static constexpr int kOffP = kOffV + kStages * kKVBytes;
    static constexpr int kOffBar = kOffP + kPBytes;
    // barriers: full[st], empty[st], q_full, s_full[2], s_free[2], p_full, p_free
    static constexpr int kNumBars = 2 * kStages + 7;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;   // tmem base, abort, ntiles
    static constexpr int kOffList = kOffMisc + 16;            // int16 key block per tile
    static constexpr int kOffLive = kOffList + kMaxBlocks * 2;
    static constexpr int kOffBits = kOffLive + kMaxBlocks;    // two bitmaps
    static constexpr int kOffRed = kOffBits + 2 * (kMaxBlocks / 32) * 4;   // [2 parity][2 group][128] partial maxima
    static constexpr int kOffOk = kOffRed + 2 * 2 * 128 * 4;               // [2 parity][2 group][4 quad] flags
    static constexpr int kOffLsum = kOffOk + 2 * 2 * 4 * 4;                // [2 group][128] partial sums
    static constexpr int kEnd = kOffLsum + 2 * 128 * 4;
    static constexpr int kSmemBytes = kEnd + 1024;            // + alignment slack
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static constexpr int kTmemCols = 256;
    static constexpr int kTmemS = 0;       // S buffers at columns 0 and 64
    static constexpr int kTmemO = 128;     // O at columns 128 .. 128 + D
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, D == 64 ? GSA_FWD64_CTAS_PER_SM : 1)
attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint8_t* sP = smem + C::kOffP;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::kStages;
    uint64_t* q_full = bars + 2 * C::kStages;
    uint64_t* s_full = q_full + 1;
    uint64_t* s_free = s_full + 2;
    uint64_t* p_full = s_free + 2;
    uint64_t* p_free = p_full + 1;
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
        mbar_init(&s_free[0], kSmThreads);
        mbar_init(&s_free[1], kSmThreads);
        mbar_init(p_full, kSmThreads);
        mbar_init(p_free, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
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
        if (lane == 31) *ntiles_slot = incl;
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
            const uint32_t qbytes = (qb >= 0 ? 2 : 1) * kBlk * D * 2;
            mbar_arrive_expect_tx(q_full, qbytes);
            for (int half = 0; half < 2; ++half) {
                const int blk = half ? qb : qa;
                if (blk < 0) continue;
                const int row = static_cast<int>(head_row0 + static_cast<int64_t>(blk) * kBlk);
                for (int at = 0; at < C::kAtoms; ++at)
                    tma_load_2d(sQ + at * (128 * 128) + half * (kBlk * 128), &tmQ, q_full, at * 64, row);
            }
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
    } else if (warp == 1) {
        // ================= MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(128, kBlk, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(128, D, 1);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
            bool ok = mbar_wait(q_full, 0, abort_flag, kErrTimeoutMma);
            auto issue_pv = [&](int m) -> bool {
                if (!mbar_wait(p_full, m & 1, abort_flag, kErrTimeoutMma)) return false;
                tc_fence_after();
                const int st = m % C::kStages;
#pragma unroll
                for (int kk = 0; kk < kBlk / 16; ++kk) {
                    const uint64_t ad = sdesc_sw128(aP + kk * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(aV + st * C::kKVBytes + kk * (16 * 128), kBlk * 128, 1024);
                    umma_bf16(tmem + C::kTmemO, ad, bd, idesc_pv, (m > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(p_free);
                umma_commit(&empty[st]);
                return true;
            };
            for (int n = 0; ok && n < T; ++n) {
                const int st = n % C::kStages;
                const int buf = n & 1;
                if (!mbar_wait(&full[st], (n / C::kStages) & 1, abort_flag, kErrTimeoutMma)) { ok = false; break; }
                if (n >= 2 && !mbar_wait(&s_free[buf], ((n - 2) >> 1) & 1, abort_flag, kErrTimeoutMma)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int at = kk >> 2, ko = (kk & 3) * 32;
                    const uint64_t ad = sdesc_sw128(aQ + at * (128 * 128) + ko, 16, 1024);
                    const uint64_t bd = sdesc_sw128(aK + st * C::kKVBytes + at * (kBlk * 128) + ko, 16, 1024);
                    umma_bf16(tmem + C::kTmemS + buf * kBlk, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[buf]);
                if (n >= 1 && !issue_pv(n - 1)) { ok = false; break; }
            }
            if (ok && T > 0) issue_pv(T - 1);
        }
        __syncwarp();
    } else {
        // ================= softmax warpgroups (warps 2..9)
        const int quad = warp & 3;              // TMEM lane quadrant this warp may access
        const int grp = (warp - 2) >> 2;        // column group
        const int c0 = grp * kCw;               // first key column of this thread
        const int r = quad * 32 + lane;         // query row in the tile = TMEM lane
        const int half = r >> 6;
        const int my_blk = half ? qb : qa;
        const int rr = r & 63;
        const uint32_t tl = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        float* red = reinterpret_cast<float*>(smem + C::kOffRed);
        volatile int* okf = reinterpret_cast<volatile int*>(smem + C::kOffOk);
        float* lsum = reinterpret_cast<float*>(smem + C::kOffLsum);
        float m = -INFINITY, l = 0.f;           // l: this thread's share of the row sum
        bool ok = true;
        for (int n = 0; n < T; ++n) {
            const int buf = n & 1;
            // waits are warp-uniform (the tcgen05 loads are warp-collective); the
            // two warps of a row pair leave the loop together, after their barrier
            const bool w = ok && __all_sync(0xffffffffu, mbar_wait(&s_full[buf], (n >> 1) & 1, abort_flag,
                                                                   kErrTimeoutSoftmax));
            float sv[kCw];
            if (w) {
                tc_fence_after();
                tmem_ld32(tl + C::kTmemS + buf * kBlk + c0, sv);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&s_free[buf]);
            }
            const int j = list[n];
            const bool is_live = (live[n] >> half) & 1;
            const int last = (!is_live ? -1 : (j == my_blk ? rr : kBlk - 1)) - c0;
            // raw-score maximum of this thread's columns (the scale is positive);
            // masked columns become -inf, so their exponentials below are 0
            float mt;
            if (last >= kCw - 1) {
                mt = max_reduce<kCw>(sv);
            } else {
#pragma unroll
                for (int cc = 0; cc < kCw; ++cc) sv[cc] = cc <= last ? sv[cc] : -INFINITY;
                mt = max_reduce<kCw>(sv);
            }
            mt *= p.scale_log2;
            red[(buf * 2 + grp) * 128 + r] = mt;
            if (lane == 0) okf[(buf * 2 + grp) * 4 + quad] = w ? 1 : 0;
            pair_barrier(quad);
            if (!(okf[(buf * 2 + 0) * 4 + quad] && okf[(buf * 2 + 1) * 4 + quad])) {
                ok = false;
                break;
            }
            mt = fmaxf(mt, red[(buf * 2 + (grp ^ 1)) * 128 + r]);
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
            // p = 2^(s * scale * log2 e - m): one FFMA and one MUFU.EX2 per score
            float sum;
            if (last < 0) {
#pragma unroll
                for (int cc = 0; cc < kCw; ++cc) sv[cc] = 0.f;
                sum = 0.f;
            } else {
#pragma unroll
                for (int cc = 0; cc < kCw; ++cc) sv[cc] = ex2(fmaf(sv[cc], p.scale_log2, -msafe));
                sum = sum_reduce<kCw>(sv);
            }
            l = l * alpha + sum;
            m = m_use;

            if (n >= 1 &&
                !__all_sync(0xffffffffu, mbar_wait(p_free, (n - 1) & 1, abort_flag, kErrTimeoutSoftmax))) {
                ok = false;   // reported to the partner warp at the next barrier
                continue;
            }
            tc_fence_after();
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int cb = grp * (D / kSmGroups); cb < (grp + 1) * (D / kSmGroups); cb += 32) {
                    float ov[32];
                    tmem_ld32(tl + C::kTmemO + cb, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] *= alpha;
                    tmem_st32(tl + C::kTmemO + cb, ov);
                }
                tmem_wait_st();
            }
            store_cols_sw128(sP, r, sv, c0 / 8, kCw / 8);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        lsum[grp * 128 + r] = l;
        pair_barrier(quad);
        l = lsum[r] + lsum[128 + r];
        if (ok && T > 0 &&
            __all_sync(0xffffffffu, mbar_wait(p_free, (T - 1) & 1, abort_flag, kErrTimeoutSoftmax))) {
            tc_fence_after();
            const float inv = 1.f / l;
            const bool store = my_blk >= 0;
            const int64_t tok = head_row0 + static_cast<int64_t>(store ? my_blk : 0) * kBlk + rr;
            __nv_bfloat16* orow = p.o + tok * D;
#pragma unroll
            for (int cb = grp * (D / kSmGroups); cb < (grp + 1) * (D / kSmGroups); cb += 32) {
                float ov[32];
                tmem_ld32(tl + C::kTmemO + cb, ov);
                tmem_wait_ld();
                if (store) store_scaled_bf16(orow + cb, ov, inv);
            }
            if (store && grp == 0 && p.lse) p.lse[tok] = (m + log2f(l)) * 0.69314718055994531f;
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
