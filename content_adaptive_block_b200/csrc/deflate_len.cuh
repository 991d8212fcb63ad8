// Per-block gzip level-1 compressed length, one warp per block.
//
// Gzip-guided Sparse Attention (daiwk.github.io reproduction of arXiv
// 2607.21752), section "核心公式", r_i equation: the information signal of
// block i is |gzip(x_{ib:(i+1)b})|, each block compressed alone at gzip
// level 1 (flowchart: "gzip level-1 per block").  The length is that of
// Python's gzip.compress(block, 1): 18 framing bytes plus the raw DEFLATE
// stream (RFC 1951) that zlib's level 1 writes.  No stream is produced here;
// the warp walks the same decisions and sums the bits.
//
// Level 1 is a greedy parse over hash chains of 3-byte strings: at each
// position the (at most 4) most recent earlier positions with the same
// 15-bit hash ((x0 << 10) ^ (x1 << 5) ^ x2) are tried, most recent first,
// keeping the first longest match and stopping at 8 bytes ("nice" length);
// a match needs 3 bytes.  Position 0 is never a source.  A match of at most
// 4 bytes enters its inner positions into the chains; a longer one skips
// them.  Here the chains are bitmasks: each lane owns the positions
// lane + 32k, holds their hashes, and one ballot per word finds every
// inserted earlier position with the current hash; the 4 most significant
// set bits are the chain.  One more ballot compares 8 bytes of each of the 4
// candidates at once (lane = 8 * candidate + byte).
//
// The block is one final DEFLATE block of the cheapest kind by zlib's rule:
// stored (b + 5 bytes) when b + 4 <= min(fixed, dynamic) bytes, else fixed
// when it is no larger than dynamic, else dynamic.  The dynamic cost needs
// the exact code lengths zlib would pick, so the Huffman trees are built
// with zlib's heap discipline (order by frequency, then subtree depth; ties
// resolved by heap position, with the right child preferred and the moving
// node kept on ties), its dummy codes for alphabets of fewer than two
// symbols, and its repair when a code would exceed 15 bits (7 for the
// code-length code).  The code-length run-length coding is counted in closed
// form per maximal run of equal lengths (see count_runs).
#pragma once

#include "common.cuh"

namespace gsa {
namespace deflate {

constexpr int kMaxB = 128;              // largest block handled (bytes)
constexpr int kWords = kMaxB / 32;      // position bitmask words
constexpr int kWarps = 4;               // warps (blocks) per CTA of the one-launch mask stage
// Warps (blocks) per CTA of the lengths kernel: a CTA's shared memory stays
// held until its slowest block is done, and block costs vary widely (stored,
// fixed or dynamic blocks), so small CTAs keep more blocks in flight.
#ifndef GSA_LEN_WARPS
#define GSA_LEN_WARPS 1
#endif
constexpr int kLenWarps = GSA_LEN_WARPS;
constexpr int kLitLeaves = kMaxB + 4;   // distinct literal/length symbols + end of block + dummies
constexpr int kDistLeaves = 32;

template <int NL>
struct Tree {
    uint32_t key[2 * NL];       // frequency << 16 | subtree depth
    uint16_t up[2 * NL];        // parent node
    uint16_t heap[2 * NL + 2];  // 1-based binary heap of node ids
    uint16_t order[2 * NL];     // nodes in the order they left the heap
    uint16_t sym[NL];           // leaf -> symbol
    uint8_t bits[2 * NL];
    uint16_t count[16];         // leaves per code length
    int nleaf;
    int max_code;
};

struct WarpSmem {
    uint8_t x[kMaxB + 16];
    uint16_t lfreq[288];
    uint16_t dfreq[32];
    uint32_t blfreq[20];
    uint8_t llen[288];
    uint8_t dlen[32];
    uint8_t bllen[20];
    Tree<kLitLeaves> lt;        // literal/length tree, then the code-length tree
    Tree<kDistLeaves> dt;
};

// ------------------------------------------------ RFC 1951 code mapping

// Order in which the code-length code lengths are sent (section 3.2.7).
__constant__ uint8_t kBlOrder[19] = {16, 17, 18, 0, 8, 7, 9, 6, 10, 5, 11, 4, 12, 3, 13, 2, 14, 1, 15};

// Length 3..258 -> code - 257 (0..28) and its extra bits.
__device__ __forceinline__ void length_code(int len, int& code, int& extra) {
    if (len == 258) { code = 28; extra = 0; return; }
    const int v = len - 3;
    if (v < 8) { code = v; extra = 0; return; }
    const int e = (31 - __clz(v)) - 2;
    code = 4 * e + 4 + ((v >> e) - 4);
    extra = e;
}

// Distance 1..32768 -> code 0..29 and its extra bits.
__device__ __forceinline__ void dist_code(int dist, int& code, int& extra) {
    const int v = dist - 1;
    if (v < 4) { code = v; extra = 0; return; }
    const int e = (31 - __clz(v)) - 1;
    code = 2 * e + 2 + ((v >> e) & 1);
    extra = e;
}

// Fixed-code length of a literal/length symbol (RFC 1951 section 3.2.6).
__device__ __forceinline__ int fixed_len(int s) { return s < 144 ? 8 : (s < 256 ? 9 : (s < 280 ? 7 : 8)); }

__device__ __forceinline__ uint32_t hash3(uint32_t a, uint32_t b, uint32_t c) {
    return ((a << 10) ^ (b << 5) ^ c) & 0x7fffu;
}

// ------------------------------------------------ the greedy parse

// Fills lfreq / dfreq (end of block included) and returns the total number
// of extra bits of the length and distance codes.  Whole warp.
__device__ int parse_block(WarpSmem& ws, int n, int lane) {
    constexpr unsigned kAll = 0xffffffffu;
    for (int i = lane; i < 288; i += 32) ws.lfreq[i] = 0;
    if (lane < 32) ws.dfreq[lane] = 0;

    uint32_t hq[kWords];
#pragma unroll
    for (int k = 0; k < kWords; ++k) {
        const int q = lane + 32 * k;
        hq[k] = (q + 2 < n) ? hash3(ws.x[q], ws.x[q + 1], ws.x[q + 2]) : 0xffffffffu;
    }
    uint32_t ins[kWords];
#pragma unroll
    for (int k = 0; k < kWords; ++k) ins[k] = 0;
    const int nw = (n + 31) >> 5;
    __syncwarp();

    int extra_bits = 0;
    int p = 0;
    while (p < n) {
        const int rem = n - p;
        int mlen = 0, mpos = 0;
        if (rem >= 3) {
            const int pw = p >> 5;
            uint32_t hsel = 0;
#pragma unroll
            for (int k = 0; k < kWords; ++k)
                if (k == pw) hsel = hq[k];
            const uint32_t hp = __shfl_sync(kAll, hsel, p & 31);
            // candidates: inserted positions q in (0, p) with hash(q) == hash(p)
            uint32_t cw[kWords];
#pragma unroll
            for (int k = 0; k < kWords; ++k) {
                const int q = lane + 32 * k;
                const bool c = k < nw && q > 0 && q < p && ((ins[k] >> lane) & 1u) && hq[k] == hp;
                cw[k] = __ballot_sync(kAll, c);
            }
#pragma unroll
            for (int k = 0; k < kWords; ++k)
                if (k == pw) ins[k] |= 1u << (p & 31);
            // the (up to) 4 most recent candidates, newest first
            int c0 = 0, c1 = 0, c2 = 0, c3 = 0, nc = 0;
#pragma unroll
            for (int k = kWords - 1; k >= 0; --k) {
                uint32_t m = cw[k];
                while (m != 0u && nc < 4) {
                    const int bit = 31 - __clz(m);
                    m &= ~(1u << bit);
                    const int pos = 32 * k + bit;
                    if (nc == 0) c0 = pos;
                    else if (nc == 1) c1 = pos;
                    else if (nc == 2) c2 = pos;
                    else c3 = pos;
                    ++nc;
                }
            }
            if (nc > 0) {
                const int nice = rem < 8 ? rem : 8;
                const int ci = lane >> 3, kk = lane & 7;
                const int cpos = ci == 0 ? c0 : (ci == 1 ? c1 : (ci == 2 ? c2 : c3));
                const bool eq = ci < nc && kk < nice && ws.x[cpos + kk] == ws.x[p + kk];
                const uint32_t bal = __ballot_sync(kAll, eq);
                int best = 2, bpos = 0;
                for (int c = 0; c < nc; ++c) {
                    const uint32_t m8 = (bal >> (8 * c)) & 0xffu;
                    const int len = __ffs(~m8) - 1;   // leading equal bytes, at most nice
                    if (len > best) {
                        best = len;
                        bpos = c == 0 ? c0 : (c == 1 ? c1 : (c == 2 ? c2 : c3));
                        if (len >= nice) break;
                    }
                }
                if (best >= 8 && rem > 8) {
                    // extend the winning match up to min(258, rem) bytes
                    const int lim = rem < 258 ? rem : 258;
                    for (int k0 = 8;; k0 += 32) {
                        const int k = k0 + lane;
                        const bool mis = k < lim && ws.x[bpos + k] != ws.x[p + k];
                        const uint32_t mm = __ballot_sync(kAll, mis);
                        if (mm != 0u) { best = k0 + __ffs(mm) - 1; break; }
                        if (k0 + 32 >= lim) { best = lim; break; }
                    }
                }
                if (best >= 3) {
                    mlen = best < rem ? best : rem;
                    mpos = bpos;
                }
            }
        }
        if (mlen >= 3) {
            int lc, le, dc, de;
            length_code(mlen, lc, le);
            dist_code(p - mpos, dc, de);
            if (lane == 0) {
                ws.lfreq[257 + lc] += 1;
                ws.dfreq[dc] += 1;
            }
            extra_bits += le + de;
            if (mlen <= 4 && rem - mlen >= 3) {
                for (int q = p + 1; q < p + mlen; ++q) {
#pragma unroll
                    for (int k = 0; k < kWords; ++k)
                        if (k == (q >> 5)) ins[k] |= 1u << (q & 31);
                }
            }
            p += mlen;
        } else {
            if (lane == 0) ws.lfreq[ws.x[p]] += 1;
            p += 1;
        }
    }
    if (lane == 0) ws.lfreq[256] = 1;
    __syncwarp();
    return extra_bits;
}

// ------------------------------------------------ Huffman trees

// Whole warp: list the symbols with nonzero frequency, in increasing symbol
// order, as the tree's leaves (their heap insertion order).
template <int NL, typename F>
__device__ void gather_leaves(Tree<NL>& t, const F* freq, int nsym, uint8_t* lens, int lane) {
    int nleaf = 0, max_code = -1;
    for (int base = 0; base < nsym; base += 32) {
        const int s = base + lane;
        const uint32_t f = s < nsym ? freq[s] : 0u;
        if (s < nsym) lens[s] = 0;
        const uint32_t m = __ballot_sync(0xffffffffu, f != 0u);
        if (f != 0u) {
            const int pos = nleaf + __popc(m & ((1u << lane) - 1u));
            t.sym[pos] = static_cast<uint16_t>(s);
            t.key[pos] = f << 16;
            t.heap[pos + 1] = static_cast<uint16_t>(pos);
        }
        if (m != 0u) max_code = base + 31 - __clz(m);
        nleaf += __popc(m);
    }
    if (lane == 0) {
        t.nleaf = nleaf;
        t.max_code = max_code;
    }
    __syncwarp();
}

template <int NL>
__device__ __forceinline__ void sift_down(Tree<NL>& t, int heap_len, int k) {
    const uint16_t v = t.heap[k];
    const uint32_t kv = t.key[v];
    int j = k << 1;
    while (j <= heap_len) {
        uint16_t cj = t.heap[j];
        uint32_t kj = t.key[cj];
        if (j < heap_len) {
            const uint16_t cr = t.heap[j + 1];
            const uint32_t kr = t.key[cr];
            if (kr <= kj) { ++j; cj = cr; kj = kr; }
        }
        if (kv <= kj) break;
        t.heap[k] = cj;
        k = j;
        j <<= 1;
    }
    t.heap[k] = v;
}

// One thread: build the tree over the gathered leaves and write the code
// length of every leaf symbol (dummies included) into lens.  Returns the
// largest code the header sends (dummies included).
template <int NL>
__device__ int build_tree(Tree<NL>& t, int max_bits, uint8_t* lens) {
    int nleaf = t.nleaf;
    int max_code = t.max_code;
    while (nleaf < 2) {   // dummy codes of frequency 1
        const int s = max_code < 2 ? ++max_code : 0;
        t.sym[nleaf] = static_cast<uint16_t>(s);
        t.key[nleaf] = 1u << 16;
        t.heap[nleaf + 1] = static_cast<uint16_t>(nleaf);
        ++nleaf;
    }
    int heap_len = nleaf;
    for (int k = heap_len / 2; k >= 1; --k) sift_down(t, heap_len, k);
    int next = nleaf, no = 0;
    do {
        const uint16_t a = t.heap[1];
        t.heap[1] = t.heap[heap_len--];
        sift_down(t, heap_len, 1);
        const uint16_t b = t.heap[1];
        t.order[no++] = a;
        t.order[no++] = b;
        const uint32_t ka = t.key[a], kb = t.key[b];
        const uint32_t da = ka & 0xffffu, db = kb & 0xffffu;
        t.key[next] = (((ka >> 16) + (kb >> 16)) << 16) | ((da > db ? da : db) + 1u);
        t.up[a] = t.up[b] = static_cast<uint16_t>(next);
        t.heap[1] = static_cast<uint16_t>(next++);
        sift_down(t, heap_len, 1);
    } while (heap_len >= 2);
    t.order[no++] = t.heap[1];

    for (int i = 0; i < 16; ++i) t.count[i] = 0;
    t.bits[t.order[no - 1]] = 0;
    int overflow = 0;
    for (int r = no - 2; r >= 0; --r) {
        const int nd = t.order[r];
        int d = t.bits[t.up[nd]] + 1;
        if (d > max_bits) { d = max_bits; ++overflow; }
        t.bits[nd] = static_cast<uint8_t>(d);
        if (nd < nleaf) t.count[d] += 1;
    }
    if (overflow > 0) {
        do {
            int d = max_bits - 1;
            while (t.count[d] == 0) --d;
            t.count[d] -= 1;
            t.count[d + 1] += 2;
            t.count[max_bits] -= 1;
            overflow -= 2;
        } while (overflow > 0);
        int r = 0;
        for (int d = max_bits; d != 0; --d) {
            int c = t.count[d];
            while (c != 0) {
                const int nd = t.order[r++];
                if (nd >= nleaf) continue;
                t.bits[nd] = static_cast<uint8_t>(d);
                --c;
            }
        }
    }
    for (int i = 0; i < nleaf; ++i) lens[t.sym[i]] = t.bits[i];
    return max_code;
}

// ------------------------------------------------ code-length run counting
//
// RFC 1951 section 3.2.7 sends the literal/length and the distance code
// lengths (each array separately) as code-length symbols, with zlib's run
// rules.  They split into independent maximal runs of equal lengths:
//   * a run of R zeros: floor(R/138) symbols 18, then for the rest r:
//     r >= 11 one 18, 3 <= r <= 10 one 17, r < 3 r symbols 0;
//   * a run of R copies of v > 0: R < 4 sends v R times; otherwise v once
//     and one 16 for the next min(R, 7) - 1 copies, then for the remaining
//     R - 7 (when R > 7) one 16 per 6 copies and, for the rest r, one 16 if
//     r >= 3 else r more symbols v.
// Whole warp; adds into blfreq (shared) and returns the extra bits
// (2 per 16, 3 per 17, 7 per 18).
__device__ int count_runs(const uint8_t* len, int max_code, uint32_t* blfreq, int lane) {
    int extra = 0;
    for (int base = 0; base <= max_code; base += 32) {
        const int n = base + lane;
        const bool valid = n <= max_code;
        const int v = valid ? len[n] : -1;
        const int vprev = (valid && n > 0) ? len[n - 1] : -2;
        const bool start = valid && (n == 0 || v != vprev);
        const uint32_t starts = __ballot_sync(0xffffffffu, start);
        // run end (exclusive) of a run starting at n: the next start, or the
        // first start of a later chunk, or max_code + 1
        if (start) {
            const uint32_t later = lane == 31 ? 0u : (starts & ~((2u << lane) - 1u));
            int end;
            if (later != 0u) {
                end = base + __ffs(later) - 1;
            } else {
                end = n + 1;
                while (end <= max_code && len[end] == v) ++end;
            }
            const int R = end - n;
            if (v == 0) {
                const int full = R / 138, r = R % 138;
                int n18 = full, n17 = 0, n0 = 0;
                if (r >= 11) ++n18;
                else if (r >= 3) ++n17;
                else n0 = r;
                if (n18) atomicAdd(&blfreq[18], static_cast<uint32_t>(n18));
                if (n17) atomicAdd(&blfreq[17], static_cast<uint32_t>(n17));
                if (n0) atomicAdd(&blfreq[0], static_cast<uint32_t>(n0));
                extra += 7 * n18 + 3 * n17;
            } else {
                int nv, n16;
                if (R < 4) {
                    nv = R;
                    n16 = 0;
                } else {
                    nv = 1;
                    n16 = 1;
                    if (R > 7) {
                        const int rest = R - 7;
                        n16 += rest / 6;
                        const int r = rest % 6;
                        if (r >= 3) ++n16;
                        else nv += r;
                    }
                }
                atomicAdd(&blfreq[v], static_cast<uint32_t>(nv));
                if (n16) atomicAdd(&blfreq[16], static_cast<uint32_t>(n16));
                extra += 2 * n16;
            }
        }
    }
    // warp total of extra bits
    for (int o = 16; o > 0; o >>= 1) extra += __shfl_xor_sync(0xffffffffu, extra, o);
    return extra;
}

__device__ __forceinline__ int warp_sum(int v) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ------------------------------------------------ the kernel

// gzip length (18 + raw DEFLATE bytes) of the b bytes at src; the whole
// warp calls it, the result is valid on every lane.
__device__ int block_length_warp(WarpSmem& ws, const uint8_t* __restrict__ src, int b, int lane) {
    for (int k = lane; k < b + 16; k += 32) ws.x[k] = k < b ? src[k] : 0;
    __syncwarp();

    const int n = b;
    const int extra = parse_block(ws, n, lane);

    // literal/length and distance trees: leaves by the warp, heaps by lanes 0 and 1
    gather_leaves(ws.lt, ws.lfreq, 286, ws.llen, lane);
    gather_leaves(ws.dt, ws.dfreq, 30, ws.dlen, lane);
    if (lane == 0) ws.lt.max_code = build_tree(ws.lt, 15, ws.llen);
    if (lane == 1) ws.dt.max_code = build_tree(ws.dt, 15, ws.dlen);
    __syncwarp();
    const int lmax = ws.lt.max_code, dmax = ws.dt.max_code;

    // data bits, dynamic and fixed
    int dyn = 0, fix = 0;
    for (int sym = lane; sym < 286; sym += 32) {
        const int f = ws.lfreq[sym];
        dyn += f * ws.llen[sym];
        fix += f * fixed_len(sym);
    }
    if (lane < 30) {
        const int f = ws.dfreq[lane];
        dyn += f * ws.dlen[lane];
        fix += f * 5;
    }
    dyn = warp_sum(dyn) + extra;
    fix = warp_sum(fix) + extra;

    // code-length code
    if (lane < 20) ws.blfreq[lane] = 0;
    __syncwarp();
    int blx = count_runs(ws.llen, lmax, ws.blfreq, lane);
    __syncwarp();
    blx += count_runs(ws.dlen, dmax, ws.blfreq, lane);
    __syncwarp();
    gather_leaves(ws.lt, ws.blfreq, 19, ws.bllen, lane);
    if (lane == 0) build_tree(ws.lt, 7, ws.bllen);
    __syncwarp();
    int blbits = lane < 19 ? ws.blfreq[lane] * ws.bllen[lane] : 0;
    blbits = warp_sum(blbits) + blx;
    // number of code-length code lengths sent: RFC order, trailing zeros trimmed, at least 4
    const bool nz = lane < 19 && ws.bllen[kBlOrder[lane < 19 ? lane : 0]] != 0;
    const uint32_t nzm = __ballot_sync(0xffffffffu, nz);
    int hclen = nzm ? 32 - __clz(nzm) : 0;
    if (hclen < 4) hclen = 4;
    dyn += blbits + 5 + 5 + 4 + 3 * hclen;

    int opt = (dyn + 3 + 7) >> 3;
    const int stat = (fix + 3 + 7) >> 3;
    if (stat <= opt) opt = stat;
    const int raw = (n + 4 <= opt) ? n + 5 : opt;
    return raw + 18;
}

__global__ void __launch_bounds__(32 * kLenWarps)
block_lengths_kernel(const uint8_t* __restrict__ bytes, int64_t L, int b, int64_t nblocks_total,
                     int32_t* __restrict__ lengths) {
    extern __shared__ __align__(16) uint8_t dsmem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WarpSmem& ws = reinterpret_cast<WarpSmem*>(dsmem)[warp];
    const int64_t task = static_cast<int64_t>(blockIdx.x) * kLenWarps + warp;
    if (task >= nblocks_total) return;   // warp-uniform
    const int64_t nblk = L / b;
    const int64_t s = task / nblk, i = task % nblk;
    const int len = block_length_warp(ws, bytes + s * L + i * b, b, lane);
    if (lane == 0) lengths[task] = len;
}

constexpr size_t kSmemBytes = sizeof(WarpSmem) * kWarps;         // one-launch mask stage
constexpr size_t kLenSmemBytes = sizeof(WarpSmem) * kLenWarps;   // lengths kernel

}  // namespace deflate
}  // namespace gsa
