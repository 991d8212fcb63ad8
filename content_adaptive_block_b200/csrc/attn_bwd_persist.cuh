// dK, dV at d = 64 with persistent CTAs.
//
// Same products and elementwise arithmetic as dkdv_kernel (see
// attn_bwd_bf16.cuh): per key tile (two key blocks from the class's key
// pairing order) over the union of their CSC columns, S^T = K Q^T and
// dP^T = V dO^T into TMEM, P^T = exp2(S^T c - LSE log2 e) and dS^T = P^T ∘
// (dP^T - D) by the elementwise warps (two warpgroups splitting the 64 query
// columns), packed back into TMEM over the scores they replace, then
// dV += P^T dO and dK += dS^T Q with A from TMEM.
//
// What differs: a fixed grid of CTAs (two per SM) takes the work items —
// (sample·head, key tile) in the heaviest-first order of the plain launch —
// one at a time from a device counter (dot_kernel zeroes it), and the items
// follow each other without a gap.  The producer publishes each item (or the
// end) in a two-slot record ring behind an mbarrier.  The producer
// warp merges an item's query list itself (a private bitmap, no CTA
// barrier) and streams the item's Q, dO, LSE and D stages straight after the
// previous item's, each stage carrying its query block, live bits and an
// "item's last tile" mark in a word of shared memory; it reloads the K and V
// tile once the previous item's last S^T, dP^T products completed.  The MMA
// issuer waits for the previous item's epilogue to have read dV and dK
// before the new item's first accumulating product.  Phases follow a tile
// counter running across items.  Every wait is bounded; on a timeout the
// CTA records an error code and every role leaves.
#pragma once

namespace gsa {
namespace bwd {

#ifndef GSA_DKVP_STAGES
#define GSA_DKVP_STAGES 4
#endif

struct DkvPCfg {
    static constexpr int D = 64;
    static constexpr int kStages = GSA_DKVP_STAGES;
    static constexpr int kTileBytes = 128 * D * 2;      // K or V tile (128 key rows)
    static constexpr int kQBytes = kBlk * D * 2;        // one query block of Q or dO
    static constexpr int kVecBytes = kBlk * 4;          // LSE or D of one query block
    static constexpr int kStageBytes = 2 * kQBytes;     // stage: Q, dO (TMA, 1024-aligned)
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + kTileBytes;
    static constexpr int kOffStage = kOffV + kTileBytes;
    static constexpr int kOffVec = kOffStage + kStages * kStageBytes;   // per stage: LSE[64], D[64]
    static constexpr int kOffMeta = kOffVec + kStages * 2 * kVecBytes;  // per stage: block | live << 16 | last << 18
    static constexpr int kOffBar = kOffMeta + ((kStages * 4 + 7) & ~7);
    // full[st], empty[st], kv_full, kv_free, s_full, p_full, acc_done, acc_free, item_full[2]
    static constexpr int kNumBars = 2 * kStages + 9;   // + drain
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;              // tmem base, abort, item record[2]
    static constexpr int kOffBits = kOffMisc + 16;                       // producer's two bitmaps
    static constexpr int kEnd = kOffBits + 2 * (kListMaxBlocks / 32) * 4;
    static constexpr int kSmemBytes = kEnd + 1024;
    static_assert(kSmemBytes <= 232448 / 2 - 1024, "two CTAs per SM");
    static_assert(kStageBytes % 1024 == 0, "stages keep 1024-byte alignment");
    static constexpr int kTmemCols = 256;
    // S^T at 0 (P^T packed over its columns 0..15 and 32..47), dP^T at 64
    // (dS^T likewise), dV at 128, dK at 192
    static constexpr uint32_t kTmemDV = 128, kTmemDK = 192;
    static constexpr int kThreads = 64 + 256;
};

template <bool K4>   // strided tensors through 4-D maps (see load_rows)
__global__ void __launch_bounds__(DkvPCfg::kThreads, 2)
dkdv_persist_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const Params p) {
    using C = DkvPCfg;
    constexpr int D = C::D;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint8_t* sStage = smem + C::kOffStage;
    uint32_t* meta = reinterpret_cast<uint32_t*>(smem + C::kOffMeta);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::kStages;
    uint64_t* kv_full = bars + 2 * C::kStages;   // phase per item: K, V of the item loaded
    uint64_t* kv_free = kv_full + 1;             // phase per item: its last S^T, dP^T completed
    uint64_t* s_full = kv_free + 1;              // phase per tile: S^T, dP^T landed
    uint64_t* p_full = s_full + 1;               // phase per tile: P^T, dS^T in TMEM (256 arrivals)
    uint64_t* acc_done = p_full + 1;             // phase per item: its last dV, dK products completed
    uint64_t* acc_free = acc_done + 1;           // phase per item: its epilogue read dV, dK (256 arrivals)
    // [2] item k's record (or the end) published: barrier k & 1, phase k >> 1.  One
    // barrier per record slot: publishing into a slot again needs every
    // elementwise thread to have finished the slot's previous item, so no
    // waiter is ever two phases behind
    uint64_t* item_full = acc_free + 1;
    uint64_t* drain = item_full + 2;             // the MMA thread's products at exit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    int* rec = reinterpret_cast<int*>(smem + C::kOffMisc + 8);   // [2] item of phase k at rec[k & 1], -1: end
    uint32_t* bitsA = reinterpret_cast<uint32_t*>(smem + C::kOffBits);
    uint32_t* bitsB = bitsA + kListMaxBlocks / 32;
    auto stage_q = [&](int st) { return sStage + st * C::kStageBytes; };
    auto stage_do = [&](int st) { return sStage + st * C::kStageBytes + C::kQBytes; };
    auto stage_lse = [&](int st) { return reinterpret_cast<float*>(smem + C::kOffVec + st * 2 * C::kVecBytes); };
    auto stage_d = [&](int st) {
        return reinterpret_cast<float*>(smem + C::kOffVec + st * 2 * C::kVecBytes + C::kVecBytes);
    };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nblk = p.nblk;
    const int SH = p.S * p.H;
    const int ntiles = (nblk + 1) / 2;
    const int items = SH * ntiles;
    // item it: key tile it / SH (heaviest first), sample-head it % SH
    auto item_keys = [&](int it, int& sh, int& ka, int& kb, int64_t& g) {
        sh = it % SH;
        const int tile = it / SH;
        const int s = sh / p.H, h = sh % p.H;
        g = static_cast<int64_t>(s) * 3 + p.cls[h];
        ka = p.order[g * nblk + 2 * tile];
        kb = (2 * tile + 1 < nblk) ? p.order[g * nblk + 2 * tile + 1] : -1;
    };

    if (threadIdx.x == 0) {
        for (int st = 0; st < C::kStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
        }
        mbar_init(kv_full, 1);
        mbar_init(kv_free, 1);
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
        // ================= producer: per item its query list, K and V, then one stage per query block
        const int nwords = (nblk + 31) >> 5;
        int gt = 0;   // stages issued so far, across items
        int nload = 0;   // items whose tile load was issued (lane 0)
        bool ok = true;
        for (int k = 0; ok; ++k) {
            int it = 0;
            if (lane == 0) it = atomicAdd(p.ticket, 1);
            it = __shfl_sync(0xffffffffu, it, 0);
            const bool have = it < items;
            int sh = 0, ka = 0, kb = -1;
            int64_t g = 0;
            if (have) {
                item_keys(it, sh, ka, kb, g);
                // union of the two CSC columns, ascending, with a live bit per key half
                for (int w = lane; w < nwords; w += 32) {
                    bitsA[w] = 0u;
                    bitsB[w] = 0u;
                }
                __syncwarp();
                const int32_t* cp = p.ptr + g * (nblk + 1);
                const int32_t* ri = p.idx + g * p.cap;
                for (int e = cp[ka] + lane; e < cp[ka + 1]; e += 32) {
                    const int i = ri[e];
                    atomicOr(&bitsA[i >> 5], 1u << (i & 31));
                }
                if (kb >= 0) {
                    for (int e = cp[kb] + lane; e < cp[kb + 1]; e += 32) {
                        const int i = ri[e];
                        atomicOr(&bitsB[i >> 5], 1u << (i & 31));
                    }
                }
                __syncwarp();
            }
            const int64_t head_row0 = static_cast<int64_t>(sh) * p.L;
            const int s_ = sh / p.H, h_ = sh - s_ * p.H;   // the 4-D maps' head and sample
            if (lane == 0) {
                // the record slot k & 1 and the K, V tile are free once the previous
                // item's last S^T, dP^T completed (every reader of the slot's old
                // record had read it before that product was issued)
                if (k >= 1 && !mbar_wait(kv_free, (k - 1) & 1, abort_flag, kErrTimeoutProducer)) ok = false;
                rec[k & 1] = (ok && have) ? it : -1;
                mbar_arrive(&item_full[k & 1]);
                if (ok && have) {
                    ++nload;
                    mbar_arrive_expect_tx(kv_full, (kb >= 0 ? 2 : 1) * 2 * kBlk * D * 2);
                    for (int half = 0; half < 2; ++half) {
                        const int blk = half ? kb : ka;
                        if (blk < 0) continue;
                        const int l0 = blk * kBlk;   // token coordinate in the (sample, head)
                        load_rows<K4>(sK + half * (kBlk * 128), &tmK, kv_full, 0, l0, h_, s_, head_row0);
                        load_rows<K4>(sV + half * (kBlk * 128), &tmV, kv_full, 0, l0, h_, s_, head_row0);
                    }
                }
                int lastw = have ? nwords - 1 : -1;
                while (lastw >= 0 && (bitsA[lastw] | bitsB[lastw]) == 0u) --lastw;
                const int last_i = lastw >= 0 ? 32 * lastw + 31 - __clz(bitsA[lastw] | bitsB[lastw]) : -1;
                for (int w = 0; ok && w <= lastw; ++w) {
                    const uint32_t ua = bitsA[w], ub = bitsB[w];
                    uint32_t u = ua | ub;
                    while (u) {
                        const int bit = __ffs(u) - 1;
                        u &= u - 1;
                        const int i = 32 * w + bit;
                        const int st = gt % C::kStages;
                        if (gt >= C::kStages &&
                            !mbar_wait(&empty[st], ((gt / C::kStages) - 1) & 1, abort_flag, kErrTimeoutProducer)) {
                            ok = false;
                            break;
                        }
                        const uint32_t live = ((ua >> bit) & 1u) | (((ub >> bit) & 1u) << 1);
                        meta[st] = static_cast<uint32_t>(i) | (live << 16) | ((i == last_i ? 1u : 0u) << 18);
                        mbar_arrive_expect_tx(&full[st], C::kStageBytes + 2 * C::kVecBytes);
                        const int64_t row64 = head_row0 + static_cast<int64_t>(i) * kBlk;
                        load_rows<K4>(stage_q(st), &tmQ, &full[st], 0, static_cast<int>(row64 - head_row0), h_, s_, head_row0);
                        load_rows<K4>(stage_do(st), &tmDO, &full[st], 0, static_cast<int>(row64 - head_row0), h_, s_, head_row0);
                        bulk_load(stage_lse(st), p.lse2 + row64, C::kVecBytes, &full[st]);
                        bulk_load(stage_d(st), p.dvec + row64, C::kVecBytes, &full[st]);
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
        // ================= elementwise: two warpgroups splitting the 64 query columns
        constexpr int kCols = 32, kW = 8;
        const int hc = (warp - 2) >> 2;           // query columns [32 hc, 32 hc + 32)
        const int c0 = kCols * hc;
        const int quad = warp & 3;
        const int u = quad * 32 + lane;           // key row of the tile = TMEM lane
        const int half = u >> 6;
        const int uu = u & 63;
        const uint32_t tlane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const bool issuer_warp = warp == 2;       // lane 0 issues every MMA of the CTA
        constexpr uint32_t idesc_s = idesc_bf16(128, kBlk, 0);
        constexpr uint32_t idesc_acc = idesc_bf16(128, D, 1);
        const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
        auto issue_s = [&](int st) {   // S^T = K Q^T, dP^T = V dO^T of the stage's query block
            const uint32_t aQs = smem_u32(stage_q(st)), aDOs = smem_u32(stage_do(st));
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t ak = sdesc_sw128(aK + kk * 32, 16, 1024);
                const uint64_t bq = sdesc_sw128(aQs + kk * 32, 16, 1024);
                umma_bf16(tmem, ak, bq, idesc_s, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t av = sdesc_sw128(aV + kk * 32, 16, 1024);
                const uint64_t bdo = sdesc_sw128(aDOs + kk * 32, 16, 1024);
                umma_bf16(tmem + 64, av, bdo, idesc_s, kk > 0 ? 1u : 0u);
            }
            umma_commit(s_full);
            if ((meta[st] >> 18) & 1u) umma_commit(kv_free);   // the item's K, V are no longer read
        };
        bool ok = true;
        if (issuer_warp) {
            if (lane == 0) {
                // the first item's first S^T, dP^T
                ok = mbar_wait(&item_full[0], 0, abort_flag, kErrTimeoutMma);
                if (ok && rec[0] >= 0) {
                    ok = mbar_wait(kv_full, 0, abort_flag, kErrTimeoutMma) &&
                         mbar_wait(&full[0], 0, abort_flag, kErrTimeoutMma);
                    if (ok) {
                        tc_fence_after();
                        issue_s(0);
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        int gt = 0;   // tiles done so far, across items
        for (int k = 0; ok; ++k) {
            if (!__all_sync(0xffffffffu, mbar_wait(&item_full[k & 1], (k >> 1) & 1, abort_flag, kErrTimeoutSoftmax))) {
                ok = false;
                break;
            }
            const int it = rec[k & 1];
            if (it < 0) break;
            int sh, ka, kb;
            int64_t g;
            item_keys(it, sh, ka, kb, g);
            const int my_blk = half ? kb : ka;
            const int64_t head_row0 = static_cast<int64_t>(sh) * p.L;
            for (int ti = 0; ok; ++ti, ++gt) {
                const int st = gt % C::kStages;
                bool w_ok = mbar_wait(s_full, gt & 1, abort_flag, kErrTimeoutSoftmax);
                w_ok = w_ok && mbar_wait(&full[st], (gt / C::kStages) & 1, abort_flag, kErrTimeoutSoftmax);
                if (!__all_sync(0xffffffffu, w_ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t mt = meta[st];
                const int i = static_cast<int>(mt & 0xffffu);
                const bool is_live = (mt >> (16 + half)) & 1u;
                const bool last = (mt >> 18) & 1u;
                // query columns allowed: live block, and in the diagonal block t >= u
                const int first = !is_live ? kBlk : (i == my_blk ? uu : 0);
                uint32_t pp[kCols / 2], pd[kCols / 2];
                if (first >= c0 + kCols) {
#pragma unroll
                    for (int e = 0; e < kCols / 2; ++e) pp[e] = pd[e] = 0u;
                } else {
                    const float4* lse4 = reinterpret_cast<const float4*>(stage_lse(st));
                    const float4* dv4 = reinterpret_cast<const float4*>(stage_d(st));
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
                        float* d_ = dp[ch & 1];
                        const int cb = c0 + kW * ch;
#pragma unroll
                        for (int c4 = 0; c4 < kW / 4; ++c4) {
                            const float4 l4 = lse4[cb / 4 + c4];
                            const float4 d4 = dv4[cb / 4 + c4];
                            const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
                            const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int cc = 4 * c4 + e;
                                float pr = ex2(fmaf(s_[cc], p.scale_log2, -lv[e]));
                                if (first > cb) pr = cb + cc >= first ? pr : 0.f;
                                s_[cc] = pr;
                                d_[cc] = pr * (d_[cc] - dd[e]);
                            }
                        }
#pragma unroll
                        for (int e = 0; e < kW / 2; ++e) {
                            pp[(kW / 2) * ch + e] = pack_bf16x2(s_[2 * e], s_[2 * e + 1]);
                            pd[(kW / 2) * ch + e] = pack_bf16x2(d_[2 * e], d_[2 * e + 1]);
                        }
                    }
                }
                // this thread's P^T and dS^T, packed, over its own (already read) columns
                tmem_st16u(tlane + c0, pp);
                tmem_st16u(tlane + 64 + c0, pd);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(p_full);
                if (issuer_warp) {
                    bool go = true;
                    if (lane == 0) {
                        go = mbar_wait(p_full, gt & 1, abort_flag, kErrTimeoutMma);
                        // the item's first accumulating products: the previous item's
                        // epilogue has read dV and dK
                        if (go && ti == 0 && k >= 1) go = mbar_wait(acc_free, (k - 1) & 1, abort_flag, kErrTimeoutMma);
                        if (go) {
                            tc_fence_after();
                            const uint32_t aQs = smem_u32(stage_q(st)), aDOs = smem_u32(stage_do(st));
#pragma unroll
                            for (int kk = 0; kk < kBlk / 16; ++kk) {
                                const int h_ = (16 * kk) / kCols;   // the half holding queries 16 kk ..
                                const uint32_t acol = kCols * h_ + (16 * kk - kCols * h_) / 2;
                                const uint64_t bdo = sdesc_sw128(aDOs + kk * (16 * 128), kBlk * 128, 1024);
                                umma_bf16_ts(tmem + C::kTmemDV, tmem + acol, bdo, idesc_acc,
                                             (ti > 0 || kk > 0) ? 1u : 0u);
                            }
#pragma unroll
                            for (int kk = 0; kk < kBlk / 16; ++kk) {
                                const int h_ = (16 * kk) / kCols;
                                const uint32_t acol = kCols * h_ + (16 * kk - kCols * h_) / 2;
                                const uint64_t bq = sdesc_sw128(aQs + kk * (16 * 128), kBlk * 128, 1024);
                                umma_bf16_ts(tmem + C::kTmemDK, tmem + 64 + acol, bq, idesc_acc,
                                             (ti > 0 || kk > 0) ? 1u : 0u);
                            }
                            umma_commit(&empty[st]);
                            if (last) umma_commit(acc_done);
                            // S^T, dP^T of the next tile, the next item's first after a last tile
                            bool next = !last;
                            if (last) {
                                go = mbar_wait(&item_full[(k + 1) & 1], ((k + 1) >> 1) & 1, abort_flag, kErrTimeoutMma);
                                next = go && rec[(k + 1) & 1] >= 0;
                            }
                            if (next) {
                                const int nst = (gt + 1) % C::kStages;
                                go = mbar_wait(&full[nst], ((gt + 1) / C::kStages) & 1, abort_flag, kErrTimeoutMma);
                                if (go && last) go = mbar_wait(kv_full, (k + 1) & 1, abort_flag, kErrTimeoutMma);
                                if (go) {
                                    tc_fence_after();
                                    issue_s(nst);
                                }
                            }
                        }
                    }
                    if (!__shfl_sync(0xffffffffu, go, 0)) {
                        ok = false;
                        break;
                    }
                }
                if (last) {
                    ++gt;
                    // epilogue of the item: dV, dK of this thread's row, its 32 columns
                    if (!__all_sync(0xffffffffu, mbar_wait(acc_done, k & 1, abort_flag, kErrTimeoutSoftmax))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    float ov[32], ok_[32];
                    tmem_ld32(tlane + C::kTmemDV + c0, ov);
                    tmem_ld32(tlane + C::kTmemDK + c0, ok_);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(acc_free);   // the accumulators may take the next item's products
                    if (my_blk >= 0) {
                        const int64_t tok = head_row0 + static_cast<int64_t>(my_blk) * kBlk + uu;
                        const int64_t off = (K4 ? tok_off(tok, p.L, p.H, p.lq) : tok * D) + c0;
                        store_scaled_bf16(p.out0 + off, ov, 1.f);
                        store_scaled_bf16(p.out1 + off, ok_, p.scale);
                    }
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
            if (loads > 0) mbar_wait_drain(kv_full, (loads - 1) & 1);
            drain_fills(full, C::kStages, fills);
        }
        if (warp == 2 && lane == 0) {
            umma_commit(drain);
            mbar_wait_drain(drain, 0);
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
