// Forward at d = 64 and d = 128 with persistent CTAs.
//
// Same products as attn_fwd_bf16_kernel<D> — S = Q K^T per key block, an
// online softmax in exp2 with O rescaled only when a running max grows by
// more than 8 (log2 units), P packed to bf16 in TMEM as the A operand of
// O += P V — organised for the short items of the gzip masks (~12 key tiles
// per 128-row query tile):
//   persistent CTAs: a fixed grid (two per SM at d = 64, one at d = 128)
//     takes the work items —
//     (sample·head, query tile of two blocks from the class's pairing
//     order), heaviest tile first — one at a time from a device counter, so
//     set-up, key-list merge, pipeline fill and epilogue overlap the
//     previous item's tiles;
//   column split: two softmax warpgroups, A with key columns 0..31 of every
//     tile and B with columns 32..63, each with its own running max m_h,
//     sum l_h and accumulator O_h = Σ P_h V_h (split-key online softmax), so
//     no value crosses warps per tile; they combine once per item:
//     m = max(m_A, m_B), O = Σ_h O_h 2^(m_h - m) / Σ_h l_h 2^(m_h - m).
//     Each thread reads its 32 scores from TMEM once and writes its packed
//     P over its own, already-read score columns.
// Roles:
//   warp 0   producer: takes an item, merges its two CSR rows (private
//            bitmaps), publishes it in a two-slot record ring, loads its Q
//            into one of two Q buffers, then streams its key blocks' K and V
//            into the stage ring straight after the previous item's, each
//            stage carrying its block, live bit per half and an "item's last
//            tile" mark in a metadata word;
//   warp 1   TMEM owner; issues QK^T and P V in tile order across items,
//            event-driven: the warp runs the loop converged, one elected
//            lane issues.  tcgen05 products of one thread run in
//            issue order, so the QK^T of tile n + 2 goes into the S buffer of
//            tile n right after the P V products that read its P;
//   warps 2-9 softmax warpgroups.  An item's epilogue (O / l and the LSE)
//            runs inside the next item's first tile, between storing its P
//            and releasing it: the wait for the previous tile's P V, taken
//            every tile, has by then shown the item's last product complete,
//            and O is read before the P V that overwrites it is issued.  The
//            item's query blocks come with its record, from shared memory.
// The counter is one of a ring of device-global slots picked per launch; the
// launch's last CTA to leave returns its slot to zero.  An item without a
// live key block (no mask built here has one: every row holds its diagonal
// block) gets O = 0 and LSE = -inf from the producer.  Every wait is bounded;
// on a timeout the CTA records an error code, drains its loads and products
// in flight and every role leaves.
// TMEM: S[b] at 64 b (P_A packed over its columns 0..15, P_B over 32..47),
// O_A at 128, O_B at 128 + d (256 columns a CTA at d = 64, 512 at d = 128).
// Shared memory holds d in 64-column atoms of the 128-byte swizzle: a Q
// buffer is [d / 64][128 rows][64], a K or V stage [d / 64][64 rows][64].
#pragma once

namespace gsa {
namespace bf16 {

#ifndef GSA_FWDP_STAGES
#define GSA_FWDP_STAGES 4
#endif

template <int D_>
struct FwdPCfg {
    static constexpr int D = D_;
    static constexpr int kAtoms = D / 64;               // 64-column atoms of a row
    static constexpr int kCtasPerSm = D == 64 ? 2 : 1;
    static constexpr int kStages = GSA_FWDP_STAGES;
    static constexpr int kQBytes = 128 * D * 2;         // Q tile (two query blocks)
    static constexpr int kKVBytes = kBlk * D * 2;       // one key block of K or V
    static constexpr int kStageBytes = 2 * kKVBytes;    // stage: K, V (1024-aligned)
    static constexpr int kOffQ = 0;                     // [2 items]
    static constexpr int kOffStage = kOffQ + 2 * kQBytes;
    static constexpr int kOffMeta = kOffStage + kStages * kStageBytes;   // per stage: block | live << 16 | last << 18
    static constexpr int kOffBar = kOffMeta + ((kStages * 4 + 7) & ~7);
    // full[st], empty[st], q_full[2], q_free[2], s_full[2], p_full[2], item_full[2], rec_free[2],
    // drain, ml_full[4]
    static constexpr int kNumBars = 2 * kStages + 17;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;   // tmem base, abort, item record[2][2]
    static constexpr int kOffBits = kOffMisc + 32;            // producer's two bitmaps
    // [item parity][2 halves][m, l][128 rows]: a warp writes a buffer again only after
    // the next item's exchange phase, which the other warp joins after its reads
    static constexpr int kOffMl = kOffBits + 2 * (kListMaxBlocks / 32) * 4;
    static constexpr int kEnd = kOffMl + 2 * 2 * 2 * 128 * 4;
    static constexpr int kSmemBytes = kEnd + 1024;
    static_assert(kSmemBytes <= 232448 / kCtasPerSm - 1024, "shared memory per SM");
    static_assert(kQBytes % 1024 == 0 && kStageBytes % 1024 == 0, "1024-byte alignment");
    static constexpr int kTmemCols = D == 64 ? 256 : 512;
    static constexpr uint32_t kTmemS = 0, kTmemO = 128;   // O_h at 128 + D h
    static constexpr int kSoftmax = 256;                  // two warpgroups
    static constexpr int kThreads = 64 + kSoftmax;
};

template <int DH, bool K4>   // head dimension; strided tensors through 4-D maps (see load_rows)
__global__ void __launch_bounds__(FwdPCfg<DH>::kThreads, FwdPCfg<DH>::kCtasPerSm)
attn_fwd_persist_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using C = FwdPCfg<DH>;
    constexpr int D = C::D;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sStage = smem + C::kOffStage;
    uint32_t* meta = reinterpret_cast<uint32_t*>(smem + C::kOffMeta);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::kStages;        // P V of the stage's tile completed (also: O quiescent)
    uint64_t* q_full = bars + 2 * C::kStages;   // [2] Q of item k in buffer k & 1 loaded (phase k >> 1)
    uint64_t* q_free = q_full + 2;              // [2] item k's last QK^T completed (phase k >> 1)
    uint64_t* s_full = q_free + 2;              // [2] QK^T of tile n landed in S[n & 1] (phase n >> 1)
    uint64_t* p_full = s_full + 2;              // [2] P of tile n over S[n & 1] (256 arrivals, phase n >> 1)
    // [2] item k's record (or the end) published in slot k & 1 (phase k >> 1);
    // the slot is written again once the softmax threads read it (rec_free)
    // and the MMA thread issued the item's last QK^T (q_free)
    uint64_t* item_full = p_full + 2;
    uint64_t* rec_free = item_full + 2;
    uint64_t* drain = rec_free + 2;             // the MMA thread's products at exit
    // [quadrant] both halves' (m, l) of an item's rows are in shared memory (64 arrivals: the
    // quadrant's two softmax warps; phase per item)
    uint64_t* ml_full = drain + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    // record slot b: rec[2 b] = item (-1: the end), rec[2 b + 1] = qa | (qb + 1) << 16
    int* rec = reinterpret_cast<int*>(smem + C::kOffMisc + 8);
    uint32_t* bitsA = reinterpret_cast<uint32_t*>(smem + C::kOffBits);
    uint32_t* bitsB = bitsA + kListMaxBlocks / 32;
    auto q_buf = [&](int b) { return smem + C::kOffQ + b * C::kQBytes; };
    auto stage_k = [&](int st) { return sStage + st * C::kStageBytes; };
    auto stage_v = [&](int st) { return sStage + st * C::kStageBytes + C::kKVBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nblk = p.nblk;
    const int SH = p.S * p.H;
    const int items = SH * ((nblk + 1) / 2);
    // item it: query tile it / SH (heaviest first), sample-head it % SH
    // (g < 0: a local class with implicit lists)
    auto item_keys = [&](int it, int& sh, int& qa, int& qb, int64_t& g) {
        sh = it % SH;
        const int tile = it / SH;
        const int s = sh / p.H, h = sh % p.H;
        g = (p.cls[h] == 0 && p.local_implicit) ? -1 : static_cast<int64_t>(s) * 3 + p.cls[h];
        const int32_t* ord = g < 0 ? nullptr : p.q_order + g * nblk;
        qa = order_at(ord, 2 * tile);
        qb = (2 * tile + 1 < nblk) ? order_at(ord, 2 * tile + 1) : -1;
    };

    if (threadIdx.x == 0) {
        for (int st = 0; st < C::kStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_full[b], 1);
            mbar_init(&q_free[b], 1);
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], C::kSoftmax);
            mbar_init(&item_full[b], 1);
            mbar_init(&rec_free[b], C::kSoftmax);
        }
        mbar_init(drain, 1);
        for (int q = 0; q < 4; ++q) mbar_init(&ml_full[q], 64);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
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

    int fills = 0, loads = 0;   // producer (lane 0): stages and Q tiles issued
    if (warp == 0) {
        // ================= producer
        const int nwords = (nblk + 31) >> 5;
        int gt = 0;      // stages issued so far, across items
        int k = 0;       // items published
        bool ok = true;
        while (ok) {
            int it = 0;
            if (lane == 0) it = atomicAdd(p.ticket, 1);
            it = __shfl_sync(0xffffffffu, it, 0);
            const bool have = it < items;
            int sh = 0, qa = 0, qb = -1;
            int64_t g = 0;
            bool any = false;
            if (have) {
                item_keys(it, sh, qa, qb, g);
                // union of the two CSR rows, ascending, with a live bit per query half
                for (int w = lane; w < nwords; w += 32) {
                    bitsA[w] = 0u;
                    bitsB[w] = 0u;
                }
                __syncwarp();
                const ListRef rows{g < 0 ? nullptr : p.row_ptr + g * (nblk + 1), p.col_idx + (g < 0 ? 0 : g) * p.cap,
                                   p.w, nblk, false};
                rows.each(qa, lane, 32, [&](int j) { atomicOr(&bitsA[j >> 5], 1u << (j & 31)); });
                if (qb >= 0) rows.each(qb, lane, 32, [&](int j) { atomicOr(&bitsB[j >> 5], 1u << (j & 31)); });
                __syncwarp();
                uint32_t u = 0u;
                for (int w = lane; w < nwords; w += 32) u |= bitsA[w] | bitsB[w];
                any = __any_sync(0xffffffffu, u != 0u);
            }
            const int64_t head_row0 = static_cast<int64_t>(sh) * p.L;
            if (have && !any) {
                // no live key block: the softmax over an empty set
                for (int half = 0; half < 2; ++half) {
                    const int blk = half ? qb : qa;
                    if (blk < 0) continue;
                    for (int rr = lane; rr < kBlk; rr += 32) {
                        const int64_t tok = head_row0 + static_cast<int64_t>(blk) * kBlk + rr;
                        uint4* orow = reinterpret_cast<uint4*>(p.o + (K4 ? tok_off(tok, p.L, p.H, p.lo) : tok * D));
#pragma unroll
                        for (int e = 0; e < D * 2 / 16; ++e) orow[e] = make_uint4(0u, 0u, 0u, 0u);
                        p.lse[tok] = -INFINITY;
                    }
                }
                __syncwarp();   // the bitmaps are rewritten for the next item
                continue;
            }
            const int s_ = sh / p.H, h_ = sh - s_ * p.H;   // the 4-D maps' head and sample
            if (lane == 0) {
                // slot k & 1 and Q buffer k & 1 held item k - 2
                if (k >= 2) {
                    ok = mbar_wait(&rec_free[k & 1], ((k - 2) >> 1) & 1, abort_flag, kErrTimeoutProducer) &&
                         mbar_wait(&q_free[k & 1], ((k - 2) >> 1) & 1, abort_flag, kErrTimeoutProducer);
                }
                rec[2 * (k & 1)] = (ok && have) ? it : -1;
                rec[2 * (k & 1) + 1] = qa | ((qb + 1) << 16);
                mbar_arrive(&item_full[k & 1]);
                if (ok && have) {
                    mbar_arrive_expect_tx(&q_full[k & 1], (qb >= 0 ? 2 : 1) * kBlk * D * 2);
                    for (int half = 0; half < 2; ++half) {
                        const int blk = half ? qb : qa;
                        if (blk < 0) continue;
#pragma unroll
                        for (int at = 0; at < C::kAtoms; ++at)
                            load_rows<K4>(q_buf(k & 1) + at * (128 * 128) + half * (kBlk * 128), &tmQ, &q_full[k & 1],
                                          64 * at, blk * kBlk, h_, s_, head_row0);
                    }
                    ++loads;
                }
                int lastw = (ok && have) ? nwords - 1 : -1;
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
#pragma unroll
                        for (int at = 0; at < C::kAtoms; ++at) {
                            load_rows<K4>(stage_k(st) + at * (kBlk * 128), &tmK, &full[st], 64 * at, j * kBlk, h_, s_,
                                          head_row0);
                            load_rows<K4>(stage_v(st) + at * (kBlk * 128), &tmV, &full[st], 64 * at, j * kBlk, h_, s_,
                                          head_row0);
                        }
                        ++gt;
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            gt = __shfl_sync(0xffffffffu, gt, 0);
            ++k;
            __syncwarp();   // the bitmaps are rewritten for the next item
            if (!have) break;
        }
        fills = gt;
    } else if (warp == 1) {
        // ================= MMA issuer: QK^T of tile ns and P V of tile na, in tile order across
        // items.  The whole warp runs the loop converged (decisions by vote), one elected lane
        // issues: the loop state and every operand stay warp-uniform.
        constexpr uint32_t idesc_qk = idesc_bf16(128, kBlk, 0);
        constexpr uint32_t idesc_pv = idesc_bf16(128, D, 1);
        const auto all = [](bool b) { return __all_sync(0xffffffffu, b); };
        int ns = 0, kq = 0;     // QK^T: tiles issued, item of tile ns
        int na = 0, ta = 0;     // P V: tiles issued, tile index of na within its item
        bool item_open = false, qk_end = false, q_ready = false, ok = true;
        PollGuard guard;
        while (ok && !(qk_end && na == ns)) {
            bool moved = false;
            if (!qk_end) {
                if (!item_open) {
                    if (all(mbar_test(&item_full[kq & 1], (kq >> 1) & 1))) {
                        if (rec[2 * (kq & 1)] < 0) qk_end = true;
                        else item_open = true;
                        q_ready = false;
                        moved = true;
                    }
                } else {
                    const int st = ns % C::kStages, sb = ns & 1;
                    // S[sb] held tile ns - 2: its P V products are issued (in order before this QK^T)
                    if (!q_ready) q_ready = all(mbar_test(&q_full[kq & 1], (kq >> 1) & 1));
                    if (ns < na + 2 && q_ready && all(mbar_test(&full[st], (ns / C::kStages) & 1))) {
                        tc_fence_after();
                        const uint64_t da = sdesc_sw128(smem_u32(q_buf(kq & 1)), 16, 1024);
                        const uint64_t db = sdesc_sw128(smem_u32(stage_k(st)), 16, 1024);
                        // K step kk: 32 bytes into atom kk / 4 (Q atoms 16 KB apart, K atoms 8 KB)
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            umma_bf16_w(tmem + C::kTmemS + 64 * sb,
                                        sdesc_advance(da, (kk >> 2) * (128 * 128) + (kk & 3) * 32),
                                        sdesc_advance(db, (kk >> 2) * (kBlk * 128) + (kk & 3) * 32), idesc_qk,
                                        kk > 0 ? 1u : 0u);
                        umma_commit_w(&s_full[sb]);
                        if ((meta[st] >> 18) & 1u) {   // the item's Q is no longer read
                            umma_commit_w(&q_free[kq & 1]);
                            ++kq;
                            item_open = false;
                        }
                        ++ns;
                        moved = true;
                    }
                }
            }
            // with no QK^T issuable before it, block on the next P (the hardware suspends the
            // warp until the phase completes or a time limit passes)
            const bool only_pv = qk_end || ns >= na + 2;
            if (na < ns && all(only_pv ? mbar_try_wait(&p_full[na & 1], (na >> 1) & 1)
                                       : mbar_test(&p_full[na & 1], (na >> 1) & 1))) {
                tc_fence_after();
                const int st = na % C::kStages;
                const bool last = (meta[st] >> 18) & 1u;
                const uint64_t bv = sdesc_sw128(smem_u32(stage_v(st)), kBlk * 128, 1024);
                // O_h += P_h V[32 h .. 32 h + 31]: key chunk kk (16 keys) of half kk / 2 sits at
                // packed column 32 (kk / 2) + 8 (kk % 2) of the S buffer; V's d spans its atoms
                // (the descriptor's leading offset: 8 KB apart)
                const uint32_t ap = tmem + C::kTmemS + 64 * (na & 1);
#pragma unroll
                for (int kk = 0; kk < kBlk / 16; ++kk)
                    umma_bf16_ts_w(tmem + C::kTmemO + D * (kk >> 1), ap + 32 * (kk >> 1) + 8 * (kk & 1),
                                   sdesc_advance(bv, kk * (16 * 128)), idesc_pv, (ta > 0 || (kk & 1)) ? 1u : 0u);
                umma_commit_w(&empty[st]);
                ta = last ? 0 : ta + 1;
                ++na;
                moved = true;
            }
            if (moved) {
                guard.progress();
            } else {
                bool stop = false;
                if (lane == 0) stop = guard.stalled(abort_flag, kErrTimeoutMma);
                if (__shfl_sync(0xffffffffu, stop ? 1 : 0, 0)) ok = false;
            }
        }
    } else {
        // ================= softmax warpgroups (warps 2..9): one thread per query row and column half
        const int hc = (warp - 2) >> 2;          // key columns [32 hc, 32 hc + 32), accumulator O_hc
        const int c0 = 32 * hc;
        const int quad = warp & 3;               // TMEM lane quadrant this warp may access
        const int r = quad * 32 + lane;          // query row in the tile = TMEM lane
        const int half = r >> 6;
        const int rr = r & 63;
        const uint32_t tl = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const uint32_t tO = tl + C::kTmemO + D * hc;
        float* ml = reinterpret_cast<float*>(smem + C::kOffMl);
        // the previous item's epilogue, run once its last P V completed: combine the halves'
        // (m, l) through shared memory (double-buffered by item parity: a warp writes a buffer
        // again only after the next item's exchange phase, which the other warp joins after its
        // reads; a bounded mbarrier wait, so a partner that gave up cannot hang it), then O / l
        // for this thread's 32 output columns and the LSE.  False: a wait gave up.
        struct Pending {
            bool on = false;
            int parity = 0;
            int64_t tok = -1;   // this row's token (-1: no row)
            float m = 0.f, l = 0.f;
        } pend;
        auto epilogue = [&]() -> bool {
            float* mlk = ml + pend.parity * (4 * 128);
            mlk[(hc * 2 + 0) * 128 + r] = pend.m;
            mlk[(hc * 2 + 1) * 128 + r] = pend.l;
            mbar_arrive(&ml_full[quad]);
            if (!__all_sync(0xffffffffu, mbar_wait(&ml_full[quad], pend.parity, abort_flag, kErrTimeoutSoftmax)))
                return false;
            const float mA = mlk[0 * 128 + r], lA = mlk[1 * 128 + r];
            const float mB = mlk[2 * 128 + r], lB = mlk[3 * 128 + r];
            const float mm = fmaxf(mA, mB);
            const float wA = mA == -INFINITY ? 0.f : ex2(mA - mm);
            const float wB = mB == -INFINITY ? 0.f : ex2(mB - mm);
            const float lt = lA * wA + lB * wB;
            const float rl = rcp_approx(lt);
            // this thread's D / 2 output columns, 32 at a time
#pragma unroll
            for (int cb = 0; cb < D / 2; cb += 32) {
                const int col = hc * (D / 2) + cb;
                float a[32], b2[32];
                tmem_ld32(tl + C::kTmemO + col, a);
                tmem_ld32(tl + C::kTmemO + D + col, b2);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) a[e] = fmaf(b2[e], wB, a[e] * wA);
                if (pend.tok >= 0) {
                    __nv_bfloat16* orow = p.o + (K4 ? tok_off(pend.tok, p.L, p.H, p.lo) : pend.tok * D);
                    store_scaled_bf16(orow + col, a, rl);
                }
            }
            if (pend.tok >= 0 && hc == 0) p.lse[pend.tok] = (mm + lg2_approx(lt)) * 0.69314718055994531f;
            pend.on = false;
            return true;
        };
        bool ok = true;
        int n = 0;   // tiles done so far, across items
        for (int k = 0; ok; ++k) {
            if (!__all_sync(0xffffffffu, mbar_wait(&item_full[k & 1], (k >> 1) & 1, abort_flag, kErrTimeoutSoftmax))) {
                ok = false;
                break;
            }
            const int it = rec[2 * (k & 1)];
            const int qw = rec[2 * (k & 1) + 1];
            mbar_arrive(&rec_free[k & 1]);
            if (it < 0) {
                // the last item's epilogue: its last P V (tile n - 1) completes the stage's phase
                if (pend.on) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&empty[(n - 1) % C::kStages], ((n - 1) / C::kStages) & 1,
                                                           abort_flag, kErrTimeoutSoftmax))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (!epilogue()) ok = false;
                }
                break;
            }
            const int sh = it % SH;
            const int my_blk = half ? (qw >> 16) - 1 : (qw & 0xffff);
            float m = -INFINITY, l = 0.f;   // running max (log2 units) and sum of this row's half
            for (;; ++n) {
                const int sb = n & 1, st = n % C::kStages;
                const uint32_t tS = tl + C::kTmemS + 64 * sb + c0;
                bool w_ok = mbar_wait(&s_full[sb], (n >> 1) & 1, abort_flag, kErrTimeoutSoftmax);
                // the stage's metadata came with its loads
                w_ok = w_ok && mbar_wait(&full[st], (n / C::kStages) & 1, abort_flag, kErrTimeoutSoftmax);
                if (!__all_sync(0xffffffffu, w_ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t mt = meta[st];
                const int j = static_cast<int>(mt & 0xffffu);
                const bool is_live = (mt >> (16 + half)) & 1u;
                const bool last_tile = (mt >> 18) & 1u;
                // visible columns of this half: 0 .. lim (none below 0)
                const int lim = (!is_live ? -1 : (j == my_blk ? rr : kBlk - 1)) - c0;
                float v[32];
                tmem_ld32(tS, v);
                tmem_wait_ld();
                if (lim < 31) {
#pragma unroll
                    for (int cc = 0; cc < 32; ++cc) v[cc] = cc <= lim ? v[cc] : -INFINITY;
                }
                // raw-score maximum (the scale is positive), then p = 2^(s * scale * log2 e - m)
                const float mx = max_reduce3_32(v) * p.scale_log2;
                const float m_new = fmaxf(m, mx);
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
                const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nm2 = f2_pack(-msafe, -msafe);
#pragma unroll
                for (int e = 0; e < 16; ++e) {   // masked: 2^-inf = 0
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(v[2 * e], v[2 * e + 1]), sc2, nm2), x0, x1);
                    v[2 * e] = ex2(x0);
                    v[2 * e + 1] = ex2(x1);
                }
                l = l * alpha + sum_reduce2_32(v);
                m = m_use;
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
                // P over this thread's own, already-read score columns
                tmem_st16u(tS, pk);
                // O_hc was last written by the P V products of the previous tile, which complete
                // the phase of its stage's empty barrier (one phase per use of the stage; this
                // wait, taken every tile, keeps the softmax at most one phase behind)
                if (n >= 1 && !__all_sync(0xffffffffu, mbar_wait(&empty[(n - 1) % C::kStages],
                                                                 ((n - 1) / C::kStages) & 1, abort_flag,
                                                                 kErrTimeoutSoftmax))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // the previous item's O: read before this tile's P V overwrites it
                if (pend.on && !epilogue()) {
                    ok = false;
                    break;
                }
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
                mbar_arrive(&p_full[sb]);
                if (last_tile) {
                    ++n;
                    pend.on = true;
                    pend.parity = k & 1;
                    pend.tok = my_blk >= 0 ? static_cast<int64_t>(sh) * p.L + static_cast<int64_t>(my_blk) * kBlk + rr
                                           : -1;
                    pend.m = m;
                    pend.l = l;
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
            for (int b = 0; b < 2; ++b) {
                const int kl = loads - 1 - ((loads - 1 - b) & 1);   // last item loaded into buffer b
                if (loads > b) mbar_wait_drain(&q_full[b], (kl >> 1) & 1);
            }
            drain_fills(full, C::kStages, fills);
        }
        if (warp == 1) {
            umma_commit_w(drain);   // the lane that issued the products
            if (lane == 0) mbar_wait_drain(drain, 0);
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
    if (threadIdx.x == 0) {
        // the launch's last CTA returns the counter slot to zero (its producer
        // took its last ticket before this point, like every other CTA's)
        __threadfence();
        if (atomicAdd(p.ticket + 1, 1) == static_cast<int>(gridDim.x) - 1) {
            atomicExch(p.ticket, 0);
            atomicExch(p.ticket + 1, 0);
            __threadfence();
        }
    }
}

}  // namespace bf16
}  // namespace gsa
