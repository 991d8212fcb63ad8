// dQ at d = 64 with persistent CTAs.
//
// Same products and elementwise arithmetic as dq_kernel (see
// attn_bwd_bf16.cuh): per query tile (two query blocks from the class's
// pairing order) over the union of their CSR rows, S = Q K^T and dP = dO V^T
// into TMEM, dS = exp2(S c - LSE log2 e) ∘ (dP - D) by the elementwise warps
// (two warpgroups splitting the 64 key columns), packed back into TMEM over
// the scores, then dQ += dS K with A from TMEM.  Persistent as
// dkdv_persist_kernel: a fixed grid of CTAs (two per SM) takes the items
// from a device counter, the producer merges each item's key list and
// streams its K/V stages (with a metadata word each) straight after the
// previous item's, reloads Q and dO once the previous item's last S, dP
// products completed, and dQ passes from one item to the next through the
// acc_done / acc_free barriers.  Every wait is bounded.
#pragma once

namespace gsa {
namespace bwd {

#ifndef GSA_DQP_STAGES
#define GSA_DQP_STAGES 4
#endif

struct DqPCfg {
    static constexpr int D = 64;
    static constexpr int kStages = GSA_DQP_STAGES;
    static constexpr int kTileBytes = 128 * D * 2;      // Q or dO tile (128 query rows)
    static constexpr int kKVBytes = kBlk * D * 2;       // one key block of K or V
    static constexpr int kStageBytes = 2 * kKVBytes;    // stage: K, V (TMA, 1024-aligned)
    static constexpr int kOffQ = 0;
    static constexpr int kOffDO = kOffQ + kTileBytes;
    static constexpr int kOffStage = kOffDO + kTileBytes;
    static constexpr int kOffMeta = kOffStage + kStages * kStageBytes;   // per stage: block | live << 16 | last << 18
    static constexpr int kOffBar = kOffMeta + ((kStages * 4 + 7) & ~7);
    // full[st], empty[st], qd_full, qd_free, s_full, p_full, acc_done, acc_free, item_full[2]
    static constexpr int kNumBars = 2 * kStages + 9;   // + drain
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;              // tmem base, abort, item record[2]
    static constexpr int kOffBits = kOffMisc + 16;                       // producer's two bitmaps
    static constexpr int kEnd = kOffBits + 2 * (kListMaxBlocks / 32) * 4;
    static constexpr int kSmemBytes = kEnd + 1024;
    static_assert(kSmemBytes <= 232448 / 2 - 1024, "two CTAs per SM");
    static_assert(kStageBytes % 1024 == 0, "stages keep 1024-byte alignment");
    static constexpr int kTmemCols = 256;
    // S at 0 (dS packed over its columns 0..15 and 32..47), dP at 64, dQ at 128
    static constexpr uint32_t kTmemDQ = 128;
    static constexpr int kThreads = 64 + 256;
};

template <bool K4>   // strided tensors through 4-D maps (see load_rows)
__global__ void __launch_bounds__(DqPCfg::kThreads, 2)
dq_persist_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const Params p) {
    using C = DqPCfg;
    constexpr int D = C::D;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sDO = smem + C::kOffDO;
    uint8_t* sStage = smem + C::kOffStage;
    uint32_t* meta = reinterpret_cast<uint32_t*>(smem + C::kOffMeta);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::kStages;
    uint64_t* qd_full = bars + 2 * C::kStages;   // phase per item: Q, dO of the item loaded
    uint64_t* qd_free = qd_full + 1;             // phase per item: its last S, dP completed
    uint64_t* s_full = qd_free + 1;              // phase per tile: S, dP landed
    uint64_t* p_full = s_full + 1;               // phase per tile: dS in TMEM (256 arrivals)
    uint64_t* acc_done = p_full + 1;             // phase per item: its last dQ product completed
    uint64_t* acc_free = acc_done + 1;           // phase per item: its epilogue read dQ (256 arrivals)
    // [2] item k's record (or the end) published: barrier k & 1, phase k >> 1
    // (publishing into a slot again needs every elementwise thread to have
    // finished the slot's previous item, so no waiter is two phases behind)
    uint64_t* item_full = acc_free + 1;
    uint64_t* drain = item_full + 2;             // the MMA thread's products at exit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    int* rec = reinterpret_cast<int*>(smem + C::kOffMisc + 8);   // [2] item of phase k at rec[k & 1], -1: end
    uint32_t* bitsA = reinterpret_cast<uint32_t*>(smem + C::kOffBits);
    uint32_t* bitsB = bitsA + kListMaxBlocks / 32;
    auto stage_k = [&](int st) { return sStage + st * C::kStageBytes; };
    auto stage_v = [&](int st) { return sStage + st * C::kStageBytes + C::kKVBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nblk = p.nblk;
    const int SH = p.S * p.H;
    const int ntiles = (nblk + 1) / 2;
    const int items = SH * ntiles;
    // item it: query tile it / SH (heaviest first), sample-head it % SH
    auto item_keys = [&](int it, int& sh, int& qa, int& qb, int64_t& g) {
        sh = it % SH;
        const int tile = it / SH;
        const int s = sh / p.H, h = sh % p.H;
        g = (p.cls[h] == 0 && p.local_implicit) ? -1 : static_cast<int64_t>(s) * 3 + p.cls[h];   // -1: implicit
        const int32_t* ord = g < 0 ? nullptr : p.order + g * nblk;
        qa = order_at(ord, 2 * tile);
        qb = (2 * tile + 1 < nblk) ? order_at(ord, 2 * tile + 1) : -1;
    };

    if (threadIdx.x == 0) {
        for (int st = 0; st < C::kStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
        }
        mbar_init(qd_full, 1);
        mbar_init(qd_free, 1);
        mbar_init(s_full, 1);
        mbar_init(p_full, 256);
        mbar_init(acc_done, 1);
        mbar_init(acc_free, 256);
        mbar_init(&item_full[0], 1);
        mbar_init(&item_full[1], 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmDO);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    int fills = 0, loads = 0;   // producer (lane 0): stages and item tiles issued
    if (warp == 0) {
        // ================= producer: per item its key list, Q and dO, then one stage per key block
        const int nwords = (nblk + 31) >> 5;
        int gt = 0;   // stages issued so far, across items
        int nload = 0;   // items whose tile load was issued (lane 0)
        bool ok = true;
        for (int k = 0; ok; ++k) {
            int it = 0;
            if (lane == 0) it = atomicAdd(p.ticket, 1);
            it = __shfl_sync(0xffffffffu, it, 0);
            const bool have = it < items;
            int sh = 0, qa = 0, qb = -1;
            int64_t g = 0;
            if (have) {
                item_keys(it, sh, qa, qb, g);
                // union of the two CSR rows, ascending, with a live bit per query half
                for (int w = lane; w < nwords; w += 32) {
                    bitsA[w] = 0u;
                    bitsB[w] = 0u;
                }
                __syncwarp();
                const ListRef rows{g < 0 ? nullptr : p.ptr + g * (nblk + 1), p.idx + (g < 0 ? 0 : g) * p.cap, p.w,
                                   nblk, false};
                rows.each(qa, lane, 32, [&](int j) { atomicOr(&bitsA[j >> 5], 1u << (j & 31)); });
                if (qb >= 0) rows.each(qb, lane, 32, [&](int j) { atomicOr(&bitsB[j >> 5], 1u << (j & 31)); });
                __syncwarp();
            }
            const int64_t head_row0 = static_cast<int64_t>(sh) * p.L;
            const int s_ = sh / p.H, h_ = sh - s_ * p.H;   // the 4-D maps' head and sample
            if (lane == 0) {
                // the record slot k & 1 and the Q, dO tile are free once the
                // previous item's last S, dP completed
                if (k >= 1 && !mbar_wait(qd_free, (k - 1) & 1, abort_flag, kErrTimeoutProducer)) ok = false;
                rec[k & 1] = (ok && have) ? it : -1;
                mbar_arrive(&item_full[k & 1]);
                if (ok && have) {
                    ++nload;
                    mbar_arrive_expect_tx(qd_full, (qb >= 0 ? 2 : 1) * 2 * kBlk * D * 2);
                    for (int half = 0; half < 2; ++half) {
                        const int blk = half ? qb : qa;
                        if (blk < 0) continue;
                        const int l0 = blk * kBlk;   // token coordinate in the (sample, head)
                        load_rows<K4>(sQ + half * (kBlk * 128), &tmQ, qd_full, 0, l0, h_, s_, head_row0);
                        load_rows<K4>(sDO + half * (kBlk * 128), &tmDO, qd_full, 0, l0, h_, s_, head_row0);
                    }
                }
                int lastw = have ? nwords - 1 : -1;
                while (lastw >= 0 && (bitsA[lastw] | bitsB[lastw]) == 0u) --lastw;
                const int last_j = lastw >= 0 ? 32 * lastw + 31 - __clz(bitsA[lastw] | bitsB[lastw]) : -1;
                for (int w = 0; ok && w <= lastw; ++w) {
                    const uint32_t ua = bitsA[w], ub = bitsB[w];
                    uint32_t u = ua | ub;
                    while (u) {
                        const int bit = __ffs(u) - 1;
                        u &= u - 1;
                        const int j = 32 * w + bit;
                        const int st = gt % C::kStages;
                        if (gt >= C::kStages &&
                            !mbar_wait(&empty[st], ((gt / C::kStages) - 1) & 1, abort_flag, kErrTimeoutProducer)) {
                            ok = false;
                            break;
                        }
                        const uint32_t live = ((ua >> bit) & 1u) | (((ub >> bit) & 1u) << 1);
                        meta[st] = static_cast<uint32_t>(j) | (live << 16) | ((j == last_j ? 1u : 0u) << 18);
                        mbar_arrive_expect_tx(&full[st], C::kStageBytes);
                        const int l0 = j * kBlk;   // token coordinate in the (sample, head)
                        load_rows<K4>(stage_k(st), &tmK, &full[st], 0, l0, h_, s_, head_row0);
                        load_rows<K4>(stage_v(st), &tmV, &full[st], 0, l0, h_, s_, head_row0);
                        ++gt;
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            gt = __shfl_sync(0xffffffffu, gt, 0);
            __syncwarp();   // the bitmaps are rewritten for the next item
            if (!have) break;
        }
        fills = gt;
        loads = nload;
    } else if (warp >= 2) {
        // ================= elementwise: two warpgroups splitting the 64 key columns
        constexpr int kCols = 32, kW = 8;
        const int hc = (warp - 2) >> 2;           // key columns [32 hc, 32 hc + 32)
        const int c0 = kCols * hc;
        const int quad = warp & 3;
        const int r = quad * 32 + lane;           // query row of the tile = TMEM lane
        const int half = r >> 6;
        const int rr = r & 63;
        const uint32_t tlane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        // warp 2 issues every MMA of the CTA: converged, by vote, one elected lane issuing (the
        // loop state and operands stay warp-uniform)
        const bool issuer_warp = warp == 2;
        const auto wait_all = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, kErrTimeoutMma));
        };
        constexpr uint32_t idesc_s = idesc_bf16(128, kBlk, 0);
        constexpr uint32_t idesc_dq = idesc_bf16(128, D, 1);
        const uint32_t aQ = smem_u32(sQ), aDO = smem_u32(sDO);
        auto issue_s = [&](int st) {   // S = Q K^T, dP = dO V^T of the stage's key block
            const uint32_t aKs = smem_u32(stage_k(st)), aVs = smem_u32(stage_v(st));
            const uint64_t dq_ = sdesc_sw128(aQ, 16, 1024), dk_ = sdesc_sw128(aKs, 16, 1024);
            const uint64_t ddo = sdesc_sw128(aDO, 16, 1024), dv_ = sdesc_sw128(aVs, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                umma_bf16_w(tmem, sdesc_advance(dq_, kk * 32), sdesc_advance(dk_, kk * 32), idesc_s, kk > 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                umma_bf16_w(tmem + 64, sdesc_advance(ddo, kk * 32), sdesc_advance(dv_, kk * 32), idesc_s,
                            kk > 0 ? 1u : 0u);
            umma_commit_w(s_full);
            if ((meta[st] >> 18) & 1u) umma_commit_w(qd_free);   // the item's Q, dO are no longer read
        };
        bool ok = true;
        if (issuer_warp) {
            // the first item's first S, dP
            ok = wait_all(&item_full[0], 0);
            if (ok && rec[0] >= 0) {
                ok = wait_all(qd_full, 0) && wait_all(&full[0], 0);
                if (ok) {
                    tc_fence_after();
                    issue_s(0);
                }
            }
        }
        int gt = 0;   // tiles done so far, across items
        for (int k = 0; ok; ++k) {
            if (!__all_sync(0xffffffffu, mbar_wait(&item_full[k & 1], (k >> 1) & 1, abort_flag, kErrTimeoutSoftmax))) {
                ok = false;
                break;
            }
            const int it = rec[k & 1];
            if (it < 0) break;
            int sh, qa, qb;
            int64_t g;
            item_keys(it, sh, qa, qb, g);
            const int my_blk = half ? qb : qa;
            const int64_t head_row0 = static_cast<int64_t>(sh) * p.L;
            const int64_t tok = head_row0 + static_cast<int64_t>(my_blk < 0 ? 0 : my_blk) * kBlk + rr;
            const float nlse2 = my_blk >= 0 ? p.nlse2[tok] : 0.f;
            const float ndt = my_blk >= 0 ? p.ndvec[tok] : 0.f;
            const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nl2 = f2_pack(nlse2, nlse2), nd2 = f2_pack(ndt, ndt);
            for (int ti = 0; ok; ++ti, ++gt) {
                const int st = gt % C::kStages;
                bool w_ok = mbar_wait(s_full, gt & 1, abort_flag, kErrTimeoutSoftmax);
                // the stage's metadata came with its loads
                w_ok = w_ok && mbar_wait(&full[st], (gt / C::kStages) & 1, abort_flag, kErrTimeoutSoftmax);
                if (!__all_sync(0xffffffffu, w_ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t mt = meta[st];
                const int j = static_cast<int>(mt & 0xffffu);
                const bool is_live = (mt >> (16 + half)) & 1u;
                const bool last = (mt >> 18) & 1u;
                const int lastc = !is_live ? -1 : (j == my_blk ? rr : kBlk - 1);   // visible key columns 0..lastc
                uint32_t pk[kCols / 2];
                if (lastc < c0) {
#pragma unroll
                    for (int e = 0; e < kCols / 2; ++e) pk[e] = 0u;
                } else {
                    float sv[2][kW], dp[2][kW];
                    tmem_ldw<kW>(tlane + c0, sv[0]);
                    tmem_ldw<kW>(tlane + 64 + c0, dp[0]);
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        tmem_wait_ld();
                        if (ch < 3) {
                            tmem_ldw<kW>(tlane + c0 + kW * (ch + 1), sv[(ch + 1) & 1]);
                            tmem_ldw<kW>(tlane + 64 + c0 + kW * (ch + 1), dp[(ch + 1) & 1]);
                        }
                        float* s_ = sv[ch & 1];
                        const float* d_ = dp[ch & 1];
                        const int cb = c0 + kW * ch;
#pragma unroll
                        for (int e = 0; e < kW / 2; ++e) {   // dS = 2^(S c - LSE log2 e) (dP - D), in pairs
                            float x0, x1;
                            f2_unpack(f2_fma(f2_pack(s_[2 * e], s_[2 * e + 1]), sc2, nl2), x0, x1);
                            const uint64_t pr = f2_pack(ex2(x0), ex2(x1));
                            f2_unpack(f2_mul(pr, f2_add(f2_pack(d_[2 * e], d_[2 * e + 1]), nd2)), s_[2 * e], s_[2 * e + 1]);
                        }
                        if (lastc < cb + kW - 1) {
#pragma unroll
                            for (int cc = 0; cc < kW; ++cc) s_[cc] = cb + cc <= lastc ? s_[cc] : 0.f;
                        }
#pragma unroll
                        for (int e = 0; e < kW / 2; ++e) pk[(kW / 2) * ch + e] = pack_bf16x2(s_[2 * e], s_[2 * e + 1]);
                    }
                }
                // this thread's dS, packed, over its own (already read) S columns
                tmem_st16u(tlane + c0, pk);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(p_full);
                if (issuer_warp) {
                    bool go = wait_all(p_full, gt & 1);
                    // the item's first accumulating product: the previous item's epilogue has read dQ
                    if (go && ti == 0 && k >= 1) go = wait_all(acc_free, (k - 1) & 1);
                    if (go) {
                        tc_fence_after();
                        const uint64_t bk = sdesc_sw128(smem_u32(stage_k(st)), kBlk * 128, 1024);
#pragma unroll
                        for (int kk = 0; kk < kBlk / 16; ++kk) {
                            const int h_ = (16 * kk) / kCols;   // the half holding keys 16 kk ..
                            const uint32_t acol = kCols * h_ + (16 * kk - kCols * h_) / 2;
                            umma_bf16_ts_w(tmem + C::kTmemDQ, tmem + acol, sdesc_advance(bk, kk * (16 * 128)), idesc_dq,
                                           (ti > 0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit_w(&empty[st]);
                        if (last) umma_commit_w(acc_done);
                        // S, dP of the next tile, the next item's first after a last tile
                        bool next = !last;
                        if (last) {
                            go = wait_all(&item_full[(k + 1) & 1], ((k + 1) >> 1) & 1);
                            next = go && rec[(k + 1) & 1] >= 0;
                        }
                        if (next) {
                            const int nst = (gt + 1) % C::kStages;
                            go = wait_all(&full[nst], ((gt + 1) / C::kStages) & 1);
                            if (go && last) go = wait_all(qd_full, (k + 1) & 1);
                            if (go) {
                                tc_fence_after();
                                issue_s(nst);
                            }
                        }
                    }
                    if (!go) {
                        ok = false;
                        break;
                    }
                }
                if (last) {
                    ++gt;
                    // epilogue of the item: dQ of this thread's row, its 32 columns
                    if (!__all_sync(0xffffffffu, mbar_wait(acc_done, k & 1, abort_flag, kErrTimeoutSoftmax))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    float ov[32];
                    tmem_ld32(tlane + C::kTmemDQ + c0, ov);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(acc_free);   // dQ may take the next item's products
                    if (my_blk >= 0) store_scaled_bf16(p.out0 + (K4 ? tok_off(tok, p.L, p.H, p.lq) : tok * D) + c0, ov, p.scale);
                    break;
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
            if (loads > 0) mbar_wait_drain(qd_full, (loads - 1) & 1);
            drain_fills(full, C::kStages, fills);
        }
        if (warp == 2) {
            umma_commit_w(drain);   // from the lane that issued the products
            if (lane == 0) mbar_wait_drain(drain, 0);
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
