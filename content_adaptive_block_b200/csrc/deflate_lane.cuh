// Per-block gzip level-1 compressed length, one block per lane.
//
// Gzip-guided Sparse Attention (daiwk.github.io reproduction of arXiv
// 2607.21752), section "核心公式", r_i equation: the information signal of
// block i is |gzip(x_{ib:(i+1)b})|, each block compressed alone at gzip
// level 1.  The length is that of Python's gzip.compress(block, 1): 18
// framing bytes plus the raw DEFLATE stream (RFC 1951) zlib's level 1
// writes.  No stream is produced; each lane walks the decisions zlib makes
// for its block and sums the bits.
//
// Why one block per lane.  The work per block is a chain of small
// data-dependent steps (a greedy parse, three heap-ordered Huffman builds),
// so a warp per block leaves most lanes idle: here the 32 lanes of a warp
// take 32 consecutive blocks and run the same steps side by side.  Each lane
// keeps its block's state in shared memory as 32-bit words at
// [word][lane], so lane l always hits bank l whatever word it reads: no
// bank conflicts although the lanes' indices differ.
//
// The decisions (the same as zlib level 1):
//  * parse: at each position with >= 3 bytes left, the earlier positions
//    with the same 15-bit hash ((x0 << 10) ^ (x1 << 5) ^ x2) that were
//    entered into the hash chains are tried, most recent first, at most 4;
//    the first longest match wins (strictly longer than the best so far,
//    starting from 2) and the search stops at 8 bytes (or the bytes left);
//    a match of 8 extends up to 258 (or the bytes left).  Position 0 is
//    never a source (zlib's empty-slot sentinel).  The current position is
//    entered before the next one is looked at; after a match of at most 4
//    bytes that leaves >= 3 bytes, its inner positions are entered too,
//    after a longer one they are skipped.  The chains here are short bucket
//    lists (one bucket per position of the largest block, on the hash's low bits) filtered by the full hash,
//    which visits exactly zlib's chain in the same order.
//  * trees: the literal/length and distance codes are Huffman codes built
//    with zlib's heap discipline: leaves in increasing symbol order, a
//    1-based binary min-heap on (frequency, subtree depth), ties left to the
//    heap's own order (right child taken on equality, the moving node kept
//    on equality), a parent one deeper than its deeper child; an alphabet of
//    fewer than two symbols gets dummy symbols of frequency 1.  With at most
//    129 symbols of total frequency <= 129 no code can exceed 15 bits (a
//    Huffman code of depth 16 needs a total frequency of at least the 18th
//    Fibonacci number), so only the code-length code (limit 7) can overflow;
//    it gets zlib's repair (leaves moved down to the deepest level that is
//    not full, then lengths dealt out again in the order the nodes left the
//    heap).
//  * header: the code lengths of each alphabet are run-length coded
//    separately with zlib's run rules, counted in closed form per maximal
//    run of equal lengths (see add_run).
//  * block kind (zlib >= 1.2.12): stored (b + 5 bytes) when b + 4 <=
//    min(fixed, dynamic) bytes, else fixed when it is no larger than
//    dynamic, else dynamic.
#pragma once

#include "common.cuh"

namespace gsa {
namespace deflate_lane {


// Per-lane word layout in shared memory (offsets in words; word i of lane l
// is at smem[i * 32 + l] of the warp's region).  The literal counts are made
// after the parse, over the position words it no longer needs; the counts of
// the length codes (and end of block) and of the distance codes are made
// during the parse, in words of their own.
template <int MAXB>
struct Layout {
    // Blocks of at most 64 bytes build their (rare) Huffman trees in local
    // memory and keep only the parse's words here; larger blocks need the
    // trees often enough that they keep them here too, over words dead by then.
    static constexpr bool kSharedTrees = MAXB > 64;
    static constexpr int kMaxLeaves = MAXB + 2;
    static constexpr int kXb = 0;                          // block bytes, 4 per word, zero padded
    static constexpr int kXw = MAXB / 4 + 3;
    static constexpr int kPos = kXb + kXw;                 // per position: hash | previous bucket-mate << 15
    static constexpr int kBuckets = MAXB;                  // hash buckets (the hash's low bits), one per position
    static constexpr int kHeads = kPos + MAXB;             // bucket heads, 4 positions per word
    static constexpr int kPhaseA = kHeads + kBuckets / 4;
    // literal counts (bytes 0..255, 4 per word): over the position words,
    // made after the parse; with shared trees, in words of their own above
    // the nodes the leaves take
    static constexpr int kLcnt = kSharedTrees ? (kPhaseA > kMaxLeaves ? kPhaseA : kMaxLeaves) : kPos;
    // symbols 256..287 (end of block, length codes), 4 per word, then the distance codes
    static constexpr int kMcnt = kSharedTrees ? kLcnt + 64 : kPos + (MAXB + kBuckets / 4 > 64 ? MAXB + kBuckets / 4 : 64);
    // with shared trees the distance counts must outlive the literal/length tree
    static constexpr int kDcnt = kSharedTrees ? ((kMcnt + 8 > 3 * kMaxLeaves + 1) ? kMcnt + 8 : 3 * kMaxLeaves + 1)
                                              : kMcnt + 8;
    static constexpr int kWords = kSharedTrees ? ((kDcnt + 8 > 2 * kMaxLeaves + 64) ? kDcnt + 8 : 2 * kMaxLeaves + 64)
                                               : kMcnt + 16;
};

// Words of the Huffman builds: in local memory (blocks <= 64 bytes, whose
// lower bound below rarely fails) or in the lane's shared words (larger).
template <int MAXB>
struct TreeLayout {
    static constexpr bool kShared = Layout<MAXB>::kSharedTrees;
    static constexpr int kMaxLeaves = MAXB + 2;            // symbols of one tree (+ dummies)
    static constexpr int kNode = 0;                        // parent | symbol << 9 | freq << 18 | bits << 27
    static constexpr int kHeap = 2 * kMaxLeaves;           // (freq << 8 | depth) << 9 | node, 1-based
    // code-length tree (<= 19 leaves, 37 nodes, 20 heap entries): its nodes in
    // heap-exit order, above its heap entries (shared: over words dead by then)
    static constexpr int kOrder = kShared ? kHeap + 24 : kHeap + kMaxLeaves + 1;
    static constexpr int kWords = kOrder + 40;
    static_assert(!kShared || kOrder + 40 <= Layout<MAXB>::kWords, "the heap-exit order fits");
    static_assert(!kShared || kHeap + kMaxLeaves + 1 <= Layout<MAXB>::kDcnt, "distance counts outlive the heap");
    static_assert(!kShared || Layout<MAXB>::kLcnt >= kMaxLeaves, "leaves gathered below the literal counts");
};

// Word holding the count of literal/length symbol s (0..287) or, with dist,
// of distance code s (0..29).
template <int MAXB>
__device__ __forceinline__ int cnt_word(int s, bool dist = false) {
    using Y = Layout<MAXB>;
    if (dist) return Y::kDcnt + (s >> 2);
    return s < 256 ? Y::kLcnt + (s >> 2) : Y::kMcnt + ((s - 256) >> 2);
}

// The 19 code-length symbol counts (each < 512) in three registers, 9 bits
// apiece: symbol s in word s / 7 at bit 9 (s % 7).
struct ClCounts {
    uint64_t w[3] = {0, 0, 0};
    __device__ __forceinline__ void add(int s, int n) {
        const uint64_t d = static_cast<uint64_t>(n) << (9 * (s % 7));
        const int k = s / 7;
        if (k == 0) w[0] += d;
        else if (k == 1) w[1] += d;
        else w[2] += d;
    }
    __device__ __forceinline__ int get(int s) const {
        const int k = s / 7;
        const uint64_t x = k == 0 ? w[0] : (k == 1 ? w[1] : w[2]);
        return static_cast<int>((x >> (9 * (s % 7))) & 511u);
    }
};

// Fixed-code length of a literal/length symbol (RFC 1951 section 3.2.6).
__device__ __forceinline__ int fixed_len(int s) { return s < 144 ? 8 : (s < 256 ? 9 : (s < 280 ? 7 : 8)); }

// Length 3..258 -> code - 257 (0..28) and its extra bits.
__device__ __forceinline__ void length_code(int len, int& code, int& extra) {
    if (len == 258) {
        code = 28;
        extra = 0;
        return;
    }
    const int v = len - 3;
    if (v < 8) {
        code = v;
        extra = 0;
        return;
    }
    const int e = (31 - __clz(v)) - 2;
    code = 4 * e + 4 + ((v >> e) - 4);
    extra = e;
}

// Distance 1..32768 -> code 0..29 and its extra bits.
__device__ __forceinline__ void dist_code(int dist, int& code, int& extra) {
    const int v = dist - 1;
    if (v < 4) {
        code = v;
        extra = 0;
        return;
    }
    const int e = (31 - __clz(v)) - 1;
    code = 2 * e + 2 + ((v >> e) & 1);
    extra = e;
}

// One lane's view of its words.
struct LaneMem {
    uint32_t* p;   // warp region + lane
    __device__ __forceinline__ uint32_t ld(int i) const { return p[i * 32]; }
    __device__ __forceinline__ void st(int i, uint32_t v) const { p[i * 32] = v; }
};

// One thread's local-memory words.
struct LocalMem {
    uint32_t* p;
    __device__ __forceinline__ uint32_t ld(int i) const { return p[i]; }
    __device__ __forceinline__ void st(int i, uint32_t v) const { p[i] = v; }
};

// 4 bytes of the block starting at byte k (little endian; k + 4 within the padded words).
template <int MAXB>
__device__ __forceinline__ uint32_t load4(const LaneMem& m, int k) {
    const int w = Layout<MAXB>::kXb + (k >> 2);
    return __funnelshift_r(m.ld(w), m.ld(w + 1), (k & 3) * 8);
}

// Leading equal bytes of a and b (as loaded by load4), 0..4.
__device__ __forceinline__ int equal_bytes(uint32_t a, uint32_t b) {
    const uint32_t d = a ^ b;
    return d ? (__ffs(d) - 1) >> 3 : 4;
}

// Sift the heap entry at k down (zlib's heap discipline; comparisons on the
// key bits above the node id).
template <int MAXB, typename M>
__device__ __forceinline__ void sift_down(const M& m, int len, int k) {
    constexpr int H = TreeLayout<MAXB>::kHeap;
    const uint32_t v = m.ld(H + k);
    const uint32_t kv = v | 511u;
    int j = k << 1;
    while (j <= len) {
        uint32_t cj = m.ld(H + j);
        if (j < len) {
            const uint32_t cr = m.ld(H + j + 1);
            if ((cr | 511u) <= (cj | 511u)) {
                ++j;
                cj = cr;
            }
        }
        if (kv <= (cj | 511u)) break;
        m.st(H + k, cj);
        k = j;
        j <<= 1;
    }
    m.st(H + k, v);
}

// Huffman tree over the nleaf leaves in node words 0 .. nleaf-1 (symbol and
// frequency set, parent 0).  Writes each node's parent and, for every node,
// its code length (bits 27..31).  track: record the heap-exit order at
// kOrder (needed for the repair of a length-limited tree).  Returns the
// number of nodes.
template <int MAXB, typename M>
__device__ int build_tree(const M& m, int nleaf, bool track) {
    using Y = TreeLayout<MAXB>;
    for (int i = 0; i < nleaf; ++i) m.st(Y::kHeap + 1 + i, ((m.ld(Y::kNode + i) >> 18 & 511u) << 17) | i);
    int len = nleaf;
    for (int k = len >> 1; k >= 1; --k) sift_down<MAXB, M>(m, len, k);
    int next = nleaf, no = 0;
    do {
        const uint32_t a = m.ld(Y::kHeap + 1);
        m.st(Y::kHeap + 1, m.ld(Y::kHeap + len));
        --len;
        sift_down<MAXB, M>(m, len, 1);
        const uint32_t b = m.ld(Y::kHeap + 1);
        const int na = a & 511u, nb = b & 511u;
        m.st(Y::kNode + na, m.ld(Y::kNode + na) | next);
        m.st(Y::kNode + nb, m.ld(Y::kNode + nb) | next);
        if (track) {
            m.st(Y::kOrder + no, na);
            m.st(Y::kOrder + no + 1, nb);
            no += 2;
        }
        const uint32_t ka = a >> 9, kb = b >> 9;
        const uint32_t da = ka & 255u, db = kb & 255u;
        const uint32_t key = (((ka >> 8) + (kb >> 8)) << 8) | ((da > db ? da : db) + 1u);
        m.st(Y::kNode + next, 0u);
        m.st(Y::kHeap + 1, (key << 9) | next);
        ++next;
        sift_down<MAXB, M>(m, len, 1);
    } while (len >= 2);
    if (track) m.st(Y::kOrder + no, m.ld(Y::kHeap + 1) & 511u);
    // lengths, parents before children (a parent's id is above its children's)
    for (int id = next - 2; id >= 0; --id) {
        const uint32_t w = m.ld(Y::kNode + id);
        const uint32_t pb = m.ld(Y::kNode + (w & 511u)) >> 27;
        m.st(Y::kNode + id, (w & 0x07ffffffu) | ((pb + 1u) << 27));
    }
    return next;
}

// Code-length symbols of a maximal run of R copies of length v (zlib's run
// rules with the run starting after a different length or an array start):
// counts into cl, returns the extra bits.
__device__ __forceinline__ int add_run(ClCounts& cl, int v, int R) {
    if (R <= 0) return 0;
    if (v == 0) {
        int n18 = R / 138;
        const int r = R - 138 * n18;
        int x = 0;
        if (r >= 11) ++n18;
        else if (r >= 3) {
            cl.add(17, 1);
            x += 3;
        } else if (r > 0) cl.add(0, r);
        if (n18) cl.add(18, n18);
        return x + 7 * n18;
    }
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
    cl.add(v, nv);
    if (n16) cl.add(16, n16);
    return 2 * n16;
}

// x (< 2^23) as a float with one integer OR and one subtraction (the
// float 2^23 + x minus 2^23), leaving the conversion unit alone.
__device__ __forceinline__ float small_int_float(uint32_t x) {
    return __uint_as_float(0x4B000000u | x) - 8388608.f;
}

// Huffman cost (sum of frequency x code length) of at most four symbol
// counts, zeros ignored; a lone symbol costs one bit per occurrence (zlib
// gives it a dummy sibling).  Closed forms on the sorted counts
// v0 <= v1 <= v2 <= v3: four symbols merge v0 + v1 first, then the two
// smallest of (v0 + v1, v2, v3).
__device__ __forceinline__ int huffman_cost4(int a, int b, int c, int d) {
    int v0 = a, v1 = b, v2 = c, v3 = d, t;
#define GSA_CX(x, y) \
    t = min(x, y);   \
    y = max(x, y);   \
    x = t;
    GSA_CX(v0, v1) GSA_CX(v2, v3) GSA_CX(v0, v2) GSA_CX(v1, v3) GSA_CX(v1, v2)
#undef GSA_CX
    const int total = v0 + v1 + v2 + v3;
    if (v0 > 0) {
        const int m1 = v0 + v1;
        return m1 + min(m1, v3) + v2 + total;
    }
    if (v1 > 0) return 2 * (v1 + v2) + v3;
    if (v2 > 0) return v2 + v3;
    return v3;
}

// Lowest position in RFC 1951's code-length order (16 17 18 0 8 7 9 6 10 5
// 11 4 12 3 13 2 14 1 15) of a code length that a Huffman code over U >= 2
// symbols must use, taken as the larger of two facts: some length is at
// most floor(log2 U), some length is at least ceil(log2 U) (Kraft).  The
// header sends the code-length code lengths up to the last nonzero one in
// that order, so it sends at least this position + 1 of them.
__device__ __forceinline__ int min_order_pos(int U) {
    const int fl = 31 - __clz(U);                  // floor(log2 U)
    const int cl = fl + ((U & (U - 1)) ? 1 : 0);   // ceil(log2 U)
    // best (lowest) position among lengths <= fl: 8 -> 4, 7 -> 5, 6 -> 7, 5 -> 9, 4 -> 11, 3 -> 13, 2 -> 15, 1 -> 17
    const int lo = fl >= 8 ? 4 : (fl == 7 ? 5 : (fl == 6 ? 7 : 9 + 2 * (5 - (fl < 1 ? 1 : fl))));
    // lowest position among lengths >= cl: 8 -> 4 while cl <= 8; 9 -> 6, 10 -> 8, 11 -> 10, ...
    const int hi = cl <= 8 ? 4 : 2 * cl - 12;
    return lo > hi ? lo : hi;
}

// Code-length symbols of a zero run of R >= 1 (zlib's rules), as counts
// of symbols 0, 17, 18 and their extra bits.
__device__ __forceinline__ void zero_run_counts(int R, int& z0, int& z17, int& z18, int& ext) {
    int n18 = R / 138;
    const int r = R - 138 * n18;
    if (r >= 11) ++n18;
    else if (r >= 3) {
        ++z17;
        ext += 3;
    } else z0 += r;
    z18 += n18;
    ext += 7 * n18;
}

// Code-length symbols of the zero runs between used symbols of an
// alphabet (its used-symbol bitmask, NWD words), and a lower bound on those
// of its used symbols: islands of m consecutive used symbols send each
// length alone when m <= 3 and at least two symbols (a length, a repeat)
// otherwise.  Zero runs after the last used symbol are not sent.
template <int NWD>
__device__ __forceinline__ void run_counts(const uint32_t (&um)[NWD], int& z0, int& z17, int& z18, int& zext,
                                           int& nz) {
    bool ones = false;
    int run = 0;   // length of the current run (of ones or zeros)
#pragma unroll
    for (int k = 0; k < NWD; ++k) {
        const uint32_t w = um[k];
        int i = 0;
        while (i < 32) {
            const uint32_t x = ones ? ~w : w;   // the next bit that ends the current run
            const uint32_t rest = x >> i;
            const int len = rest ? __ffs(rest) - 1 : 32 - i;
            run += len;
            i += len;
            if (i < 32) {   // run ends at bit i
                if (ones) nz += run <= 3 ? run : 2;
                else if (run > 0) zero_run_counts(run, z0, z17, z18, zext);
                ones = !ones;
                run = 0;
            }
        }
    }
    if (ones) nz += run <= 3 ? run : 2;
}

// The exact size, with zlib's trees: the literal/length, distance and
// code-length Huffman codes built as the header says, their run-length
// coded lengths, and zlib's choice of block kind.  m: the lane's counts;
// t: the words of the trees (see TreeLayout).
template <int MAXB, typename TM>
__device__ int exact_length(const LaneMem& m, const TM& t, int n, int extra, int stat) {
    using TY = TreeLayout<MAXB>;
    // ---- literal/length tree: leaves in symbol order (never fewer than two:
    // end of block and at least one literal)
    int nleaf = 0;
    for (int wd = 0; wd < 72; ++wd) {
        uint32_t v = m.ld(cnt_word<MAXB>(4 * wd));
        while (v) {
            const int j = (__ffs(v) - 1) >> 3;
            const uint32_t f = (v >> (8 * j)) & 255u;
            v &= ~(255u << (8 * j));
            t.st(TY::kNode + nleaf, (static_cast<uint32_t>(4 * wd + j) << 9) | (f << 18));
            ++nleaf;
        }
    }
    ClCounts cl;
    build_tree<MAXB>(t, nleaf, false);
    int dyn = extra;
    int blx = 0;   // extra bits of the code-length symbols
    {
        // data bits, and the run-length coding of lengths 0 .. max symbol
        int prev = -1, rv = -1, rl = 0;
        for (int i = 0; i < nleaf; ++i) {
            const uint32_t w = t.ld(TY::kNode + i);
            const int sy = (w >> 9) & 511u, v = w >> 27;
            dyn += static_cast<int>((w >> 18) & 511u) * v;
            const int gap = sy - prev - 1;
            if (gap > 0 || v != rv) {
                blx += add_run(cl, rv, rl);
                blx += add_run(cl, 0, gap);
                rv = v;
                rl = 1;
            } else {
                ++rl;
            }
            prev = sy;
        }
        blx += add_run(cl, rv, rl);
    }

    // ---- distance tree (dummies for fewer than two codes)
    {
        nleaf = 0;
        int max_code = -1;
        for (int wd = 0; wd < 8; ++wd) {
            uint32_t v = m.ld(cnt_word<MAXB>(4 * wd, true));
            while (v) {
                const int j = (__ffs(v) - 1) >> 3;
                const uint32_t f = (v >> (8 * j)) & 255u;
                v &= ~(255u << (8 * j));
                t.st(TY::kNode + nleaf, (static_cast<uint32_t>(4 * wd + j) << 9) | (f << 18));
                max_code = 4 * wd + j;
                ++nleaf;
            }
        }
        const int nreal = nleaf;
        while (nleaf < 2) {
            const int sd = max_code < 2 ? ++max_code : 0;
            t.st(TY::kNode + nleaf, (static_cast<uint32_t>(sd) << 9) | (1u << 18));
            ++nleaf;
        }
        build_tree<MAXB>(t, nleaf, false);
        // lengths by code, 4 bits each (codes 0 .. 29), dummies included; data bits of real codes
        uint64_t dlo = 0, dhi = 0;
        for (int i = 0; i < nleaf; ++i) {
            const uint32_t w = t.ld(TY::kNode + i);
            const int sd = (w >> 9) & 511u;
            const uint64_t v = w >> 27;
            if (sd < 16) dlo |= v << (4 * sd);
            else dhi |= v << (4 * (sd - 16));
            if (i < nreal) dyn += static_cast<int>((w >> 18) & 511u) * static_cast<int>(v);
        }
        int rv = -1, rl = 0;
        for (int sd = 0; sd <= max_code; ++sd) {
            const int v = static_cast<int>(((sd < 16 ? dlo >> (4 * sd) : dhi >> (4 * (sd - 16)))) & 15u);
            if (v == rv) {
                ++rl;
            } else {
                blx += add_run(cl, rv, rl);
                rv = v;
                rl = 1;
            }
        }
        blx += add_run(cl, rv, rl);
    }

    // ---- code-length tree (limit 7 bits, with zlib's repair)
    uint64_t bllen = 0;   // 3 bits per code-length symbol
    int blbits = blx;
    {
        nleaf = 0;
        int max_code = -1;
        for (int sy = 0; sy < 19; ++sy) {
            const int f = cl.get(sy);
            if (f) {
                t.st(TY::kNode + nleaf, (static_cast<uint32_t>(sy) << 9) | (static_cast<uint32_t>(f) << 18));
                max_code = sy;
                ++nleaf;
            }
        }
        const int nreal = nleaf;
        while (nleaf < 2) {
            const int sy = max_code < 2 ? ++max_code : 0;
            t.st(TY::kNode + nleaf, (static_cast<uint32_t>(sy) << 9) | (1u << 18));
            ++nleaf;
        }
        const int nodes = build_tree<MAXB>(t, nleaf, true);
        // overflow: nodes whose length passed 7 (each clamped in turn from its clamped parent)
        int overflow = 0;
        uint64_t count = 0;   // leaves per length 0..7, 8 bits each
        for (int id = nodes - 1; id >= 0; --id) {
            const uint32_t w = t.ld(TY::kNode + id);
            int d = static_cast<int>(w >> 27);
            if (id < nodes - 1) {
                const int pdp = static_cast<int>(t.ld(TY::kNode + (w & 511u)) >> 27);
                d = pdp + 1;
                if (d > 7) {
                    d = 7;
                    ++overflow;
                }
                t.st(TY::kNode + id, (w & 0x07ffffffu) | (static_cast<uint32_t>(d) << 27));
            }
            if (id < nleaf) count += uint64_t(1) << (8 * d);
        }
        if (overflow > 0) {
            do {
                int d = 6;
                while (((count >> (8 * d)) & 255u) == 0) --d;
                count -= uint64_t(1) << (8 * d);
                count += uint64_t(2) << (8 * (d + 1));
                count -= uint64_t(1) << 56;
                overflow -= 2;
            } while (overflow > 0);
            int r = 0;
            for (int d = 7; d != 0; --d) {
                int c = static_cast<int>((count >> (8 * d)) & 255u);
                while (c != 0) {
                    const int nd = static_cast<int>(t.ld(TY::kOrder + r));
                    ++r;
                    if (nd >= nleaf) continue;
                    t.st(TY::kNode + nd, (t.ld(TY::kNode + nd) & 0x07ffffffu) | (static_cast<uint32_t>(d) << 27));
                    --c;
                }
            }
        }
        for (int i = 0; i < nleaf; ++i) {
            const uint32_t w = t.ld(TY::kNode + i);
            const int sy = (w >> 9) & 511u;
            bllen |= static_cast<uint64_t>(w >> 27) << (3 * sy);
            if (i < nreal) blbits += static_cast<int>((w >> 18) & 511u) * static_cast<int>(w >> 27);
        }
    }
    // code-length code lengths sent: RFC order, trailing zeros trimmed, at least 4
    constexpr uint64_t kOrderNibbles = 0xF1E2D3C4B5A69780ull;   // order positions 3..18: 0 8 7 9 6 10 5 11 4 12 3 13 2 14 1 15
    int hclen = 4;
    for (int i = 18; i >= 4; --i) {
        const int sy = static_cast<int>((kOrderNibbles >> (4 * (i - 3))) & 15u);
        if ((bllen >> (3 * sy)) & 7u) {
            hclen = i + 1;
            break;
        }
    }
    dyn += blbits + 5 + 5 + 4 + 3 * hclen;

    int opt = (dyn + 3 + 7) >> 3;
    if (stat <= opt) opt = stat;
    const int raw = (n + 4 <= opt) ? n + 5 : opt;
    return raw + 18;
}

// gzip length (18 + raw DEFLATE bytes) of the lane's block of n bytes, whose
// bytes are already in its words (zero padded).  lanes: the warp's lanes
// that hold a block (all of them call this together).
template <int MAXB>
__device__ int lane_block_length(const LaneMem& m, int n, unsigned lanes) {
    using Y = Layout<MAXB>;
    constexpr int NW = MAXB / 32;   // words of the per-position bitmasks
    // ---- prepass, the same steps on every lane: each position with >= 3
    // bytes left gets its hash and its previous bucket-mate (Layout::kBuckets buckets on the
    // hash's low bits; 0 ends a list, as position 0 is never a match source)
    for (int i = 0; i < Y::kBuckets / 4; ++i) m.st(Y::kHeads + i, 0u);
    for (int i = 0; i < 8; ++i) {
        m.st(Y::kMcnt + i, 0u);
        m.st(Y::kDcnt + i, 0u);
    }
    {
        uint32_t h = 0;
        for (int q = 0; q + 2 < n; ++q) {
            const uint32_t x2 = (m.ld(Y::kXb + ((q + 2) >> 2)) >> (((q + 2) & 3) * 8)) & 255u;
            if (q == 0) {
                const uint32_t w0 = m.ld(Y::kXb);
                h = ((w0 & 255u) << 10) ^ (((w0 >> 8) & 255u) << 5) ^ x2;
            } else {
                h = (h << 5) ^ x2;
            }
            h &= 0x7fffu;
            const uint32_t bk = h & (Y::kBuckets - 1);
            const int hw = Y::kHeads + (bk >> 2);
            const uint32_t sh = (bk & 3u) * 8u;
            const uint32_t heads = m.ld(hw);
            m.st(Y::kPos + q, h | (((heads >> sh) & 255u) << 15));
            m.st(hw, (heads & ~(255u << sh)) | (static_cast<uint32_t>(q) << sh));
        }
    }

    // ---- greedy parse.  Candidates for p: its earlier bucket-mates with the
    // same hash that were entered into the chains (a bitmask in registers),
    // newest first.  Literal positions are marked and counted afterwards.
    uint32_t ins[NW], lit[NW];
#pragma unroll
    for (int k = 0; k < NW; ++k) ins[k] = lit[k] = 0u;
    auto bit = [&](const uint32_t (&a)[NW], uint32_t q) -> bool {
        uint32_t w = 0;
#pragma unroll
        for (int k = 0; k < NW; ++k)
            if (k == static_cast<int>(q >> 5)) w = a[k];
        return (w >> (q & 31u)) & 1u;
    };
    auto set = [&](uint32_t (&a)[NW], int q) {
#pragma unroll
        for (int k = 0; k < NW; ++k)
            if (k == (q >> 5)) a[k] |= 1u << (q & 31);
    };
    int fix = 7;       // fixed-code bits (end of block included), extra bits included
    int extra = 0;     // extra bits of the length and distance codes
    int p = 0;
    while (p < n) {
        const int rem = n - p;
        int mlen = 0, mpos = 0;
        if (rem >= 3) {
            const uint32_t wp = m.ld(Y::kPos + p);
            const uint32_t h = wp & 0x7fffu;
            uint32_t q = (wp >> 15) & 127u;
            set(ins, p);
            if (q != 0u) {
                const int nice = rem < 8 ? rem : 8;
                const uint32_t p0 = load4<MAXB>(m, p), p1 = load4<MAXB>(m, p + 4);
                int best = 2, nc = 0;
                while (q != 0u && nc < 4) {
                    const uint32_t wq = m.ld(Y::kPos + q);
                    if ((wq & 0x7fffu) == h && bit(ins, q)) {
                        ++nc;
                        const uint32_t q0 = load4<MAXB>(m, q), q1 = load4<MAXB>(m, q + 4);
                        int len = equal_bytes(q0, p0);
                        if (len == 4) len += equal_bytes(q1, p1);
                        if (len > nice) len = nice;
                        if (len > best) {
                            best = len;
                            mpos = static_cast<int>(q);
                            if (len >= nice) break;
                        }
                    }
                    q = (wq >> 15) & 127u;
                }
                if (best >= 8 && rem > 8) {
                    const int lim = rem < 258 ? rem : 258;
                    int k = 8;
                    while (k < lim) {   // 8 bytes per step
                        const uint32_t a0 = load4<MAXB>(m, mpos + k), b0 = load4<MAXB>(m, p + k);
                        const uint32_t a1 = load4<MAXB>(m, mpos + k + 4), b1 = load4<MAXB>(m, p + k + 4);
                        int e = equal_bytes(a0, b0);
                        if (e == 4) e += equal_bytes(a1, b1);
                        k += e;
                        if (e < 8) break;
                    }
                    best = k < lim ? k : lim;
                }
                if (best >= 3) mlen = best < rem ? best : rem;
            }
        }
        if (mlen >= 3) {
            int lc, le, dc, de;
            length_code(mlen, lc, le);
            dist_code(p - mpos, dc, de);
            const int sym = 257 + lc;
            const int ws = cnt_word<MAXB>(sym), wd = cnt_word<MAXB>(dc, true);
            m.st(ws, m.ld(ws) + (1u << ((sym & 3) * 8)));
            m.st(wd, m.ld(wd) + (1u << ((dc & 3) * 8)));
            extra += le + de;
            fix += fixed_len(sym) + 5 + le + de;
            if (mlen <= 4 && rem - mlen >= 3)
                for (int q = p + 1; q < p + mlen; ++q) set(ins, q);
            p += mlen;
        } else {
            set(lit, p);
            p += 1;
        }
    }
    // literal counts, the same steps on every lane, over the position words
    for (int i = 0; i < 64; ++i) m.st(Y::kLcnt + i, 0u);
    for (int q = 0; q < n; ++q) {
        if (bit(lit, q)) {
            const uint32_t xq = (m.ld(Y::kXb + (q >> 2)) >> ((q & 3) * 8)) & 255u;
            m.st(Y::kLcnt + (xq >> 2), m.ld(Y::kLcnt + (xq >> 2)) + (1u << ((xq & 3) * 8)));
            fix += xq < 144 ? 8 : 9;
        }
    }
    // end of block
    m.st(Y::kMcnt, m.ld(Y::kMcnt) + 1u);
    const int stat = (fix + 3 + 7) >> 3;

    // ---- a lower bound on the dynamic block's bits, from the counts alone:
    //  * data: at least the entropy of each alphabet's symbol counts (a lone
    //    distance code costs exactly one bit per use);
    //  * header: 5 + 5 + 4 bits, 3 bits per code-length code length sent
    //    (at least min_order_pos + 1 of them), and the code-length symbols:
    //    those of the zero runs between used symbols are known exactly
    //    (symbols 0, 17, 18 and their extra bits), the islands of used
    //    symbols need at least the counts run_counts gives, and coding all
    //    of them costs at least the Huffman cost of those four counts
    //    (merging symbols and lowering counts never raise a Huffman cost).
    // When the bound shows fixed (or stored) coding no larger than dynamic,
    // zlib's choice follows without building any tree.
    int result = -1;
    {
        uint32_t um[9];   // used literal/length symbols 0 .. 287
        float slog = 0.f;
        int T = 0;
#pragma unroll
        for (int k = 0; k < 9; ++k) um[k] = 0u;
#pragma unroll
        for (int wd = 0; wd < 72; ++wd) {
            const uint32_t v = m.ld(cnt_word<MAXB>(4 * wd));
            if (v) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t f = (v >> (8 * j)) & 255u;
                    T += static_cast<int>(f);
                    const float ff = small_int_float(f);
                    slog += ff * lg2_approx(f > 1u ? ff : 1.f);
                }
            }
            // bytes that are nonzero -> 4 bits (positions 21..24 of the product)
            uint32_t t = v | (v >> 4);
            t |= t >> 2;
            t |= t >> 1;
            t &= 0x01010101u;
            um[wd >> 3] |= ((t * 0x204081u) >> 21 & 15u) << (4 * (wd & 7));
        }
        int U = 0;
#pragma unroll
        for (int k = 0; k < 9; ++k) U += __popc(um[k]);
        int z0 = 0, z17 = 0, z18 = 0, zext = 0, nz = 0;
        run_counts<9>(um, z0, z17, z18, zext, nz);
        float data = static_cast<float>(T) * lg2_approx(static_cast<float>(T)) - slog;   // U >= 2 always
        // distance codes, with zlib's dummies for fewer than two codes
        int Td = 0, dmax = -1;
        float slogd = 0.f;
        uint32_t ud[1] = {0u};
#pragma unroll
        for (int wd = 0; wd < 8; ++wd) {
            const uint32_t v = m.ld(cnt_word<MAXB>(4 * wd, true));
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t f = (v >> (8 * j)) & 255u;
                Td += static_cast<int>(f);
                const float ff = small_int_float(f);
                slogd += ff * lg2_approx(f > 1u ? ff : 1.f);
                if (f) ud[0] |= 1u << (4 * wd + j);
            }
        }
        const int Ud = __popc(ud[0]);
        if (ud[0]) dmax = 31 - __clz(ud[0]);
        int dbits_int = 0;
        if (Ud >= 2) data += static_cast<float>(Td) * lg2_approx(static_cast<float>(Td)) - slogd;
        else dbits_int = Td;   // zero or one code: one bit per use
        for (int u = Ud; u < 2; ++u) {
            const int sd = dmax < 2 ? ++dmax : 0;
            ud[0] |= 1u << sd;
        }
        run_counts<1>(ud, z0, z17, z18, zext, nz);
        int pos = min_order_pos(U);
        const int pd = min_order_pos(Ud > 2 ? Ud : 2);
        if (pd > pos) pos = pd;
        const int hclen_lb = pos + 1 > 4 ? pos + 1 : 4;
        // data bits rounded down with half a bit to spare for the approximate logarithms
        const int data_lb = static_cast<int>(floorf(data - 0.5f)) + dbits_int;
        const int lb = data_lb + extra + 5 + 5 + 4 + 3 * hclen_lb + huffman_cost4(z0, z17, z18, nz) + zext;
        if (lb >= fix) result = (n + 4 <= stat) ? n + 5 : stat;   // fixed no larger than dynamic
        else if (((lb + 3 + 7) >> 3) >= n + 4 && stat >= n + 4) result = n + 5;   // stored
    }
    if (__all_sync(lanes, result >= 0)) return result + 18;
    if (result >= 0) return result + 18;   // this lane waits while the others build their trees

    if constexpr (Layout<MAXB>::kSharedTrees) {
        return exact_length<MAXB>(m, m, n, extra, stat);
    } else {
        uint32_t tree_words[TreeLayout<MAXB>::kWords];
        return exact_length<MAXB>(m, LocalMem{tree_words}, n, extra, stat);
    }
}

// Per-lane words a warp needs, and warps per CTA, for blocks of at most MAXB bytes.
template <int MAXB>
struct KernelShape {
    static constexpr int kWarpBytes = Layout<MAXB>::kWords * 32 * 4;
    static constexpr int kWarps = 1;
    static constexpr int kSmemBytes = kWarpBytes * kWarps;
    // CTAs (warps) resident per SM by shared memory (1 KB reserved per CTA)
    static constexpr int kResident = 227 * 1024 / (kSmemBytes + 1024) < 32 ? 227 * 1024 / (kSmemBytes + 1024) : 32;
};

// Blocks per warp (one per lane) for a batch of total blocks on fill
// resident warps: the fewest of 1, 2, 4, ..., 32 that still run every block in
// one wave.  A warp's time is its slowest lane's block plus the steps where
// its lanes diverge, so when the batch leaves warps to spare, fewer blocks per
// warp finish sooner (measured at 1024 blocks of 64 bytes: 66 us at one block
// per warp against 83 us at eight).
inline int blocks_per_warp(int64_t total, int64_t fill) {
    int bpw = 1;
    while (bpw < 32 && total > bpw * fill) bpw *= 2;
    return bpw;
}

// Lengths of the nb (<= 32) blocks task0 .. task0 + nb - 1 of the batch, one
// per lane, into lengths[task0 ..]: the warp stages its blocks (contiguous
// bytes) into the lanes' words of region with coalesced loads, then each lane
// runs its block.  Whole warp.
template <int MAXB>
__device__ __forceinline__ void warp_block_lengths(uint32_t* region, const uint8_t* __restrict__ bytes, int b,
                                                   int64_t task0, int nb, int32_t* __restrict__ lengths, int lane) {
    using Y = Layout<MAXB>;
    for (int i = 0; i < Y::kXw; ++i) region[(Y::kXb + i) * 32 + lane] = 0u;
    __syncwarp();
    const uint8_t* src = bytes + task0 * b;
    uint8_t* r8 = reinterpret_cast<uint8_t*>(region);
    for (int j = lane; j < nb * b; j += 32) {
        const int blk = j / b, k = j - blk * b;
        r8[((Y::kXb + (k >> 2)) * 32 + blk) * 4 + (k & 3)] = src[j];
    }
    __syncwarp();
    if (lane < nb) {
        const LaneMem m{region + lane};
        const unsigned lanes = nb >= 32 ? 0xffffffffu : ((1u << nb) - 1u);
        lengths[task0 + lane] = lane_block_length<MAXB>(m, b, lanes);
    }
    __syncwarp();   // the region may be restaged next
}

// Lengths of blocks task0 .. task0 + 31 of the batch, one per lane (see
// warp_block_lengths), one warp per CTA.
template <int MAXB>
__global__ void __launch_bounds__(32 * KernelShape<MAXB>::kWarps)
block_lengths_lane_kernel(const uint8_t* __restrict__ bytes, int b, int64_t nblocks_total, int bpw,
                          int32_t* __restrict__ lengths) {
    using Y = Layout<MAXB>;
    extern __shared__ __align__(16) uint32_t lsmem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t* region = lsmem + static_cast<size_t>(warp) * Y::kWords * 32;
    // bpw (1 .. 32) blocks per warp: fewer when the batch is small, so that
    // more warps share the blocks and each warp's lanes diverge less
    const int64_t task0 = (static_cast<int64_t>(blockIdx.x) * KernelShape<MAXB>::kWarps + warp) * bpw;
    if (task0 >= nblocks_total) return;   // warp-uniform
    const int nb = nblocks_total - task0 < bpw ? static_cast<int>(nblocks_total - task0) : bpw;
    warp_block_lengths<MAXB>(region, bytes, b, task0, nb, lengths, lane);
}

}  // namespace deflate_lane
}  // namespace gsa
