// dK, dV at d = 64: one persistent CTA per SM with double-buffered scores.
//
// Same products and elementwise arithmetic as dkdv_kernel (see
// attn_bwd_bf16.cuh): per key tile (two key blocks from the class's key
// pairing order) over the union of their CSC columns, S^T = K Q^T and
// dP^T = V dO^T into TMEM, P^T = exp2(S^T c - LSE log2 e) and dS^T = P^T ∘
// (dP^T - D) by the elementwise warps, packed back into TMEM over the scores
// they replace, then dV += P^T dO and dK += dS^T Q with A from TMEM.
//
// Work: a fixed grid of CTAs (one per SM) takes the work items — (sample·head,
// key tile) in the heaviest-first order of the plain launch — one at a time
// from a device counter (dot_kernel zeroes it), with no gap between items.
// The producer warp publishes each item (or the end) in a two-slot record
// ring behind mbarriers, merges the item's query list itself (a private
// bitmap, no CTA barrier) and streams its Q, dO, LSE and D stages straight
// after the previous item's; each stage carries its query block, live bits
// and an "item's last tile" mark in a word of shared memory.  K and V are
// double-buffered per item, so the next item's tile loads while the current
// one finishes.
//
// Overlap: the CTA holds all 512 TMEM columns, two S^T / dP^T buffers, so the
// scores of tile n + 2 are issued right after the dV, dK products of tile n
// and are computed while the elementwise warps work on tile n + 1.  Two
// warpgroups split each tile's 64 query columns into halves (measured 0.7 %
// faster over the backward than four warpgroups on quarters).  Two threads
// on different warps issue the MMAs, one for S^T and dV, one for dP^T and dK,
// so each accumulator still sees its products in one fixed order (the result
// is deterministic) while issue, which dominates with one thread sharing its
// scheduler with elementwise warps, runs on two schedulers.  The issuers wait
// for the previous item's epilogue to have read dV and dK before the new
// item's first accumulating product.  Phases follow a tile counter running
// across items.  Every wait is bounded; on a timeout the CTA records an error
// code, drains its loads and products in flight and every role leaves.
// TMEM: buffer b at 128 b (S^T at +0 with P^T packed over the first half of
// each warpgroup's columns, dP^T at +64 with dS^T likewise), dV at 256, dK at
// 320.
#pragma once

namespace gsa {
namespace bwd {

#ifndef GSA_DKVP_STAGES
#define GSA_DKVP_STAGES 7
#endif
// Elementwise warpgroups, each owning 64 / G of a tile's query columns.
#ifndef GSA_DKVP_GROUPS
#define GSA_DKVP_GROUPS 2
#endif

struct DkvPCfg {
    static constexpr int D = 64;
    static constexpr int kStages = GSA_DKVP_STAGES;
    static constexpr int kTileBytes = 128 * D * 2;      // K or V tile (128 key rows)
    static constexpr int kQBytes = kBlk * D * 2;        // one query block of Q or dO
    static constexpr int kVecBytes = kBlk * 4;          // LSE or D of one query block
    static constexpr int kStageBytes = 2 * kQBytes;     // stage: Q, dO (TMA, 1024-aligned)
    static constexpr int kOffKV = 0;                    // [2 items][K, V]
    static constexpr int kOffStage = kOffKV + 4 * kTileBytes;
    static constexpr int kOffVec = kOffStage + kStages * kStageBytes;   // per stage: LSE[64], D[64]
    static constexpr int kOffMeta = kOffVec + kStages * 2 * kVecBytes;  // per stage: block | live << 16 | last << 18
    static constexpr int kOffBar = kOffMeta + ((kStages * 4 + 7) & ~7);
    // full[st], empty[st], kv_full[2], kv_free[2], s_full[2], p_full[2], acc_done, acc_free,
    // item_full[2], rec_free[2], drain
    static constexpr int kNumBars = 2 * kStages + 17;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;              // tmem base, abort, item record[2][2]
    static constexpr int kOffBits = kOffMisc + 32;                       // producer's two bitmaps
    static constexpr int kEnd = kOffBits + 2 * (kListMaxBlocks / 32) * 4;
    static constexpr int kSmemBytes = kEnd + 1024;
    static_assert(kSmemBytes <= 232448 - 1024, "shared memory per CTA");
    static_assert(kStageBytes % 1024 == 0 && kTileBytes % 1024 == 0, "1024-byte alignment");
    static constexpr int kTmemCols = 512;
    static constexpr uint32_t kTmemDV = 256, kTmemDK = 320;
    static constexpr int kGroups = GSA_DKVP_GROUPS;
    static_assert(kGroups == 2 || kGroups == 4, "warpgroups of 32 or 16 query columns");
    static constexpr int kEw = 128 * kGroups;           // elementwise threads (warps 2 .. 1 + 4 G)
    static constexpr int kIssuer2 = 2 + 4 * kGroups;    // the second MMA issuer's warp
    static constexpr int kThreads = 64 + kEw + 32;
};

template <bool K4>   // strided tensors through 4-D maps (see load_rows)
__global__ void __launch_bounds__(DkvPCfg::kThreads, 1)
dkdv_persist_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                     const Params p) {
    using C = DkvPCfg;
    constexpr int D = C::D;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sStage = smem + C::kOffStage;
    uint32_t* meta = reinterpret_cast<uint32_t*>(smem + C::kOffMeta);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::kStages;
    uint64_t* kv_full = bars + 2 * C::kStages;   // [item & 1], phase item >> 1: K, V of the item loaded
    uint64_t* kv_free = kv_full + 2;             // [item & 1], phase item >> 1: its last S^T, dP^T completed
    uint64_t* s_full = kv_free + 2;              // [tile & 1], phase tile >> 1: S^T, dP^T landed
    // [tile & 1], phase tile >> 1: P^T, dS^T in TMEM (512 arrivals).  Two, because the
    // issuer is not one of the arriving threads: the elementwise warps may finish tile
    // n + 1 before the issuer waits for tile n, but not tile n + 2 (its scores are
    // issued after that wait)
    uint64_t* p_full = s_full + 2;
    uint64_t* acc_done = p_full + 2;             // phase per item: its last dV, dK products completed
    uint64_t* acc_free = acc_done + 1;           // phase per item: its epilogue read dV, dK (512 arrivals)
    uint64_t* item_full = acc_free + 1;          // [item & 1], phase item >> 1: the item's record published
    uint64_t* rec_free = item_full + 2;          // [item & 1], phase item >> 1: every elementwise thread read it
    uint64_t* drain = rec_free + 2;              // the MMA thread's products at exit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    // record slot b: rec[2 b] = item (-1: the end), rec[2 b + 1] = ka | (kb + 1) << 16
    int* rec = reinterpret_cast<int*>(smem + C::kOffMisc + 8);
    uint32_t* bitsA = reinterpret_cast<uint32_t*>(smem + C::kOffBits);
    uint32_t* bitsB = bitsA + kListMaxBlocks / 32;
    auto tile_k = [&](int b) { return smem + C::kOffKV + b * 2 * C::kTileBytes; };
    auto tile_v = [&](int b) { return smem + C::kOffKV + b * 2 * C::kTileBytes + C::kTileBytes; };
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
        g = (p.cls[h] == 0 && p.local_implicit) ? -1 : static_cast<int64_t>(s) * 3 + p.cls[h];   // -1: implicit
        const int32_t* ord = g < 0 ? nullptr : p.order + g * nblk;
        ka = order_at(ord, 2 * tile);
        kb = (2 * tile + 1 < nblk) ? order_at(ord, 2 * tile + 1) : -1;
    };

    if (threadIdx.x == 0) {
        // two MMA issuers commit to the barriers of products: empty, kv_free, s_full, acc_done, drain
        for (int st = 0; st < C::kStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 2);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&kv_full[b], 1);
            mbar_init(&kv_free[b], 2);
            mbar_init(&s_full[b], 2);
            mbar_init(&item_full[b], 1);
            mbar_init(&rec_free[b], C::kEw);
        }
        mbar_init(&p_full[0], C::kEw);
        mbar_init(&p_full[1], C::kEw);
        mbar_init(acc_done, 2);
        mbar_init(acc_free, C::kEw);
        mbar_init(drain, 2);
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
        int nload = 0;
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
                const ListRef cols{g < 0 ? nullptr : p.ptr + g * (nblk + 1), p.idx + (g < 0 ? 0 : g) * p.cap, p.w,
                                   nblk, true};
                cols.each(ka, lane, 32, [&](int i) { atomicOr(&bitsA[i >> 5], 1u << (i & 31)); });
                if (kb >= 0) cols.each(kb, lane, 32, [&](int i) { atomicOr(&bitsB[i >> 5], 1u << (i & 31)); });
                __syncwarp();
            }
            const int64_t head_row0 = static_cast<int64_t>(sh) * p.L;
            const int s_ = sh / p.H, h_ = sh - s_ * p.H;   // the 4-D maps' head and sample
            if (lane == 0) {
                // record slot and K / V buffer k & 1 held item k - 2: every elementwise
                // thread has read its record, and its last S^T, dP^T completed
                if (k >= 2 && !(mbar_wait(&rec_free[k & 1], ((k - 2) >> 1) & 1, abort_flag, kErrTimeoutProducer) &&
                                mbar_wait(&kv_free[k & 1], ((k - 2) >> 1) & 1, abort_flag, kErrTimeoutProducer)))
                    ok = false;
                rec[2 * (k & 1)] = (ok && have) ? it : -1;
                rec[2 * (k & 1) + 1] = ka | ((kb + 1) << 16);
                mbar_arrive(&item_full[k & 1]);
                if (ok && have) {
                    ++nload;
                    mbar_arrive_expect_tx(&kv_full[k & 1], (kb >= 0 ? 2 : 1) * 2 * kBlk * D * 2);
                    for (int half = 0; half < 2; ++half) {
                        const int blk = half ? kb : ka;
                        if (blk < 0) continue;
                        const int l0 = blk * kBlk;   // token coordinate in the (sample, head)
                        load_rows<K4>(tile_k(k & 1) + half * (kBlk * 128), &tmK, &kv_full[k & 1], 0, l0, h_, s_,
                                      head_row0);
                        load_rows<K4>(tile_v(k & 1) + half * (kBlk * 128), &tmV, &kv_full[k & 1], 0, l0, h_, s_,
                                      head_row0);
                    }
                }
                int lastw = (ok && have) ? nwords - 1 : -1;
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
                        const int l0 = i * kBlk;
                        const int64_t row64 = head_row0 + l0;
                        load_rows<K4>(stage_q(st), &tmQ, &full[st], 0, l0, h_, s_, head_row0);
                        load_rows<K4>(stage_do(st), &tmDO, &full[st], 0, l0, h_, s_, head_row0);
                        bulk_load(stage_lse(st), p.nlse2 + row64, C::kVecBytes, &full[st]);
                        bulk_load(stage_d(st), p.ndvec + row64, C::kVecBytes, &full[st]);
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
    } else if (warp >= 2 && warp < C::kIssuer2) {
        // ================= elementwise: GSA_DKVP_GROUPS warpgroups, each with 64 / G query columns
        constexpr int kCols = 64 / C::kGroups, kW = 8, kChunks = kCols / kW;
        const int qc = (warp - 2) >> 2;           // query columns [kCols qc, kCols qc + kCols)
        const int c0 = kCols * qc;
        const int quad = warp & 3;
        const int u = quad * 32 + lane;           // key row of the tile = TMEM lane
        const int half = u >> 6;
        const int uu = u & 63;
        const uint32_t tlane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
        // The previous item's epilogue (dV, dK of this thread's row, its kCols columns) runs inside
        // the next item's first tile, after its P^T, dS^T are stored and before they are released:
        // by then the item's last products have long been issued, and the accumulators are read
        // (acc_free) before the next item's first accumulating products, which wait for it.
        struct Pending {
            bool on = false;
            int parity = 0;
            int64_t tok = -1;   // this row's token (-1: no row)
        } pend;
        auto epilogue = [&]() -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait(acc_done, pend.parity, abort_flag, kErrTimeoutSoftmax))) return false;
            tc_fence_after();
            float ov[kCols], ok_[kCols];
#pragma unroll
            for (int cb = 0; cb < kCols; cb += 16) {
                tmem_ld16(tlane + C::kTmemDV + c0 + cb, ov + cb);
                tmem_ld16(tlane + C::kTmemDK + c0 + cb, ok_ + cb);
            }
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(acc_free);   // the accumulators may take the next item's products
            if (pend.tok >= 0) {
                const int64_t off = (K4 ? tok_off(pend.tok, p.L, p.H, p.lq) : pend.tok * D) + c0;
#pragma unroll
                for (int h2 = 0; h2 < kCols / 8; ++h2) {
                    uint4 a, b;
                    a.x = pack_bf16x2(ov[8 * h2 + 0], ov[8 * h2 + 1]);
                    a.y = pack_bf16x2(ov[8 * h2 + 2], ov[8 * h2 + 3]);
                    a.z = pack_bf16x2(ov[8 * h2 + 4], ov[8 * h2 + 5]);
                    a.w = pack_bf16x2(ov[8 * h2 + 6], ov[8 * h2 + 7]);
                    b.x = pack_bf16x2(ok_[8 * h2 + 0] * p.scale, ok_[8 * h2 + 1] * p.scale);
                    b.y = pack_bf16x2(ok_[8 * h2 + 2] * p.scale, ok_[8 * h2 + 3] * p.scale);
                    b.z = pack_bf16x2(ok_[8 * h2 + 4] * p.scale, ok_[8 * h2 + 5] * p.scale);
                    b.w = pack_bf16x2(ok_[8 * h2 + 6] * p.scale, ok_[8 * h2 + 7] * p.scale);
                    *reinterpret_cast<uint4*>(p.out0 + off + 8 * h2) = a;
                    *reinterpret_cast<uint4*>(p.out1 + off + 8 * h2) = b;
                }
            }
            pend.on = false;
            return true;
        };
        bool ok = true;
        int gt = 0;   // tiles done so far, across items
        for (int k = 0; ok; ++k) {
            if (!__all_sync(0xffffffffu, mbar_wait(&item_full[k & 1], (k >> 1) & 1, abort_flag, kErrTimeoutSoftmax))) {
                ok = false;
                break;
            }
            const int it = rec[2 * (k & 1)];
            const int kw = rec[2 * (k & 1) + 1];
            mbar_arrive(&rec_free[k & 1]);   // the slot may take item k + 2
            if (it < 0) {
                if (pend.on && !epilogue()) ok = false;   // the last item's
                break;
            }
            const int sh = it % SH;
            const int my_blk = half ? (kw >> 16) - 1 : (kw & 0xffff);
            const int64_t head_row0 = static_cast<int64_t>(sh) * p.L;
            for (int ti = 0; ok; ++ti, ++gt) {
                const int st = gt % C::kStages;
                const uint32_t tb = tlane + 128 * (gt & 1);   // this tile's S^T / dP^T buffer
                bool w_ok = mbar_wait(&s_full[gt & 1], (gt >> 1) & 1, abort_flag, kErrTimeoutSoftmax);
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
                // the TMEM loads are warp-collective: skip them only when the whole
                // warp's rows start past this column range (the diagonal's first column
                // varies across the warp's lanes; the element mask below covers it)
                if (__all_sync(0xffffffffu, first >= c0 + kCols)) {
#pragma unroll
                    for (int e = 0; e < kCols / 2; ++e) pp[e] = pd[e] = 0u;
                } else {
                    const float4* lse4 = reinterpret_cast<const float4*>(stage_lse(st));
                    const float4* dv4 = reinterpret_cast<const float4*>(stage_d(st));
                    float sv[2][kW], dp[2][kW];
                    tmem_ldw<kW>(tb + c0, sv[0]);
                    tmem_ldw<kW>(tb + 64 + c0, dp[0]);
#pragma unroll
                    for (int ch = 0; ch < kChunks; ++ch) {
                        tmem_wait_ld();
                        if (ch + 1 < kChunks) {
                            tmem_ldw<kW>(tb + c0 + kW * (ch + 1), sv[(ch + 1) & 1]);
                            tmem_ldw<kW>(tb + 64 + c0 + kW * (ch + 1), dp[(ch + 1) & 1]);
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
                            for (int e = 0; e < 4; e += 2) {   // P^T = 2^(S^T c - LSE log2 e), dS^T = P^T (dP^T - D), in pairs
                                const int cc = 4 * c4 + e;
                                float x0, x1;
                                f2_unpack(f2_fma(f2_pack(s_[cc], s_[cc + 1]), sc2, f2_pack(lv[e], lv[e + 1])), x0, x1);
                                float p0 = ex2(x0), p1 = ex2(x1);
                                if (first > cb) {
                                    p0 = cb + cc >= first ? p0 : 0.f;
                                    p1 = cb + cc + 1 >= first ? p1 : 0.f;
                                }
                                s_[cc] = p0;
                                s_[cc + 1] = p1;
                                f2_unpack(f2_mul(f2_pack(p0, p1), f2_add(f2_pack(d_[cc], d_[cc + 1]), f2_pack(dd[e], dd[e + 1]))),
                                          d_[cc], d_[cc + 1]);
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
                tmem_stn<kCols / 2>(tb + c0, pp);
                tmem_stn<kCols / 2>(tb + 64 + c0, pd);
                tmem_wait_st();
                if (pend.on && !epilogue()) {   // the previous item's dV, dK
                    ok = false;
                    break;
                }
                tc_fence_before();
                mbar_arrive(&p_full[gt & 1]);
                if (last) {
                    ++gt;
                    pend.on = true;
                    pend.parity = k & 1;
                    pend.tok = my_blk >= 0 ? head_row0 + static_cast<int64_t>(my_blk) * kBlk + uu : -1;
                    break;
                }
            }
        }
    } else if (warp == 1 || warp == C::kIssuer2) {
        // ================= MMA issuers (warps 1 and kIssuer2, on different SM sub-partitions: a
        // tcgen05.mma takes issue slots its sub-partition's elementwise warps also want).  Each
        // warp runs its loop converged (waits by vote) and one elected lane issues, so the loop
        // state and operands stay warp-uniform.  Warp 1
        // issues S^T = K Q^T and dV += P^T dO, the other dP^T = V dO^T and dK += dS^T Q: each TMEM
        // region (S^T and P^T, dP^T and dS^T, dV, dK) is written and read by one thread's products,
        // in its issue order, so the accumulation order is fixed.  Per tile: dV (dK) of tile n when
        // its P^T, dS^T are in TMEM, then S^T (dP^T) of tile n + 2.
        const bool side_s = warp == 1;
        constexpr uint32_t idesc_s = idesc_bf16(128, kBlk, 0);
        constexpr uint32_t idesc_acc = idesc_bf16(128, D, 1);
        int nx = 0, nx_item = 0;   // next tile (and its item) whose scores to issue
        bool nx_first = true, nx_end = false;
        const auto wait_all = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, kErrTimeoutMma));
        };
        // S^T = K Q^T, dP^T = V dO^T of tile nx into buffer nx & 1 (false: a wait gave up)
        auto issue_next = [&]() -> bool {
            if (nx_end) return true;
            if (nx_first) {
                if (!wait_all(&item_full[nx_item & 1], (nx_item >> 1) & 1)) return false;
                if (rec[2 * (nx_item & 1)] < 0) {
                    nx_end = true;
                    return true;
                }
                if (!wait_all(&kv_full[nx_item & 1], (nx_item >> 1) & 1)) return false;
            }
            const int st = nx % C::kStages;
            if (!wait_all(&full[st], (nx / C::kStages) & 1)) return false;
            tc_fence_after();
            const bool last = (meta[st] >> 18) & 1u;
            // this side's operands: K and Q (S^T) or V and dO (dP^T); descriptors built once per
            // tile and stepped by the K offset (fewer instructions per MMA issue)
            const uint64_t da = sdesc_sw128(smem_u32(side_s ? tile_k(nx_item & 1) : tile_v(nx_item & 1)), 16, 1024);
            const uint64_t db = sdesc_sw128(smem_u32(side_s ? stage_q(st) : stage_do(st)), 16, 1024);
            const uint32_t dst = tmem + 128 * (nx & 1) + (side_s ? 0 : 64);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                umma_bf16_w(dst, sdesc_advance(da, kk * 32), sdesc_advance(db, kk * 32), idesc_s, kk > 0 ? 1u : 0u);
            umma_commit_w(&s_full[nx & 1]);
            if (last) umma_commit_w(&kv_free[nx_item & 1]);   // the item's K, V are no longer read
            ++nx;
            nx_first = last;
            if (last) ++nx_item;
            return true;
        };
        bool ok = issue_next() && issue_next();
        for (int n = 0, k = 0, ti = 0; ok && n < nx; ++n) {
            ok = wait_all(&p_full[n & 1], (n >> 1) & 1);
            // the item's first accumulating products: the previous item's epilogue has read dV and dK
            if (ok && ti == 0 && k >= 1) ok = wait_all(acc_free, (k - 1) & 1);
            if (!ok) break;
            tc_fence_after();
            const int st = n % C::kStages;
            const bool last = (meta[st] >> 18) & 1u;
            // dV += P^T dO or dK += dS^T Q (A from TMEM: the 16 queries of K step kk belong to
            // warpgroup g = 16 kk / kCols, packed at kCols g + (16 kk - kCols g) / 2)
            const uint32_t ab = tmem + 128 * (n & 1) + (side_s ? 0 : 64);
            const uint32_t acc = tmem + (side_s ? C::kTmemDV : C::kTmemDK);
            const uint64_t bb = sdesc_sw128(smem_u32(side_s ? stage_do(st) : stage_q(st)), kBlk * 128, 1024);
#pragma unroll
            for (int kk = 0; kk < kBlk / 16; ++kk)
                umma_bf16_ts_w(acc, ab + (64 / C::kGroups) * ((16 * kk) / (64 / C::kGroups)) +
                                        ((16 * kk) % (64 / C::kGroups)) / 2,
                               sdesc_advance(bb, kk * (16 * 128)), idesc_acc,
                               (ti > 0 || kk > 0) ? 1u : 0u);
            umma_commit_w(&empty[st]);
            if (last) umma_commit_w(acc_done);
            ok = issue_next();   // the scores of tile n + 2 into the buffer this tile's products read
            if (last) {
                ++k;
                ti = 0;
            } else {
                ++ti;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // a role gave up a wait: the loads and products issued must land before
        // shared memory and TMEM go (without one, every one of them was waited for)
        if (warp == 0 && lane == 0) {
            if (loads > 0) mbar_wait_drain(&kv_full[(loads - 1) & 1], ((loads - 1) >> 1) & 1);
            if (loads > 1) mbar_wait_drain(&kv_full[(loads - 2) & 1], ((loads - 2) >> 1) & 1);
            drain_fills(full, C::kStages, fills);
        }
        if (warp == 1 || warp == C::kIssuer2) {
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
