/*
 * ORACLE — test infrastructure only.  Nothing on the product path may link,
 * load or call this file; only the tests, the bench's CPU-baseline leg and
 * the package smoke check do.
 *
 * A plain, slow, from-scratch DEFLATE compressor at "gzip level 1", written to
 * define the per-block compressed length that gzip-guided sparse attention
 * uses as its information-density signal:
 *
 *   Gzip-guided Sparse Attention (daiwk.github.io reproduction of arXiv
 *   2607.21752), section "核心公式", the r_i equation: r_i = |gzip(x_{ib:(i+1)b})| / b,
 *   each block compressed on its own ("背景与主要改动" and the flowchart node
 *   "gzip level-1 per block").
 *
 * Reading taken (the pages name no implementation): "gzip level 1" is what
 * Python's gzip.compress(x, compresslevel=1) produces, i.e. a 10-byte gzip
 * header, a raw DEFLATE stream (RFC 1951) made by the zlib library at level 1
 * with its default window (15 bits), memory level (8) and strategy, and an
 * 8-byte CRC32/ISIZE trailer.  |gzip(x)| = 18 + raw DEFLATE bytes.
 *
 * The compressor follows RFC 1951 for the format and zlib's documented level-1
 * behaviour for the choices the format leaves open:
 *   - parse: greedy ("fast") matching over hash chains of 3-byte strings,
 *     hash = ((x0 << 10) ^ (x1 << 5) ^ x2) & 0x7fff, at most 4 chain
 *     candidates, stop early at a match of 8 ("nice" length), minimum match 3;
 *     short matches (<= 4) have their inner positions inserted into the hash
 *     chains, longer ones do not; position 0 marks an empty chain and can
 *     never be a match source; bytes past the end of input read as zero;
 *   - one final block; its type (stored / fixed / dynamic Huffman) is the
 *     cheapest by zlib's rule, and the dynamic trees are built with zlib's
 *     heap-based Huffman construction (frequency, then subtree depth) and its
 *     length-limiting repair.
 * The whole stream is emitted, so the tests can compare it byte for byte
 * with the host zlib and inflate it back.
 *
 * Blocks up to 16383 bytes are supported (a single DEFLATE block); longer
 * inputs return -2.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <pthread.h>

#define NLIT 286          /* literal/length alphabet used by zlib: 0..285 */
#define NDIST 30
#define NBL 19
#define MAX_INPUT 16383
#define MAX_MATCH 258

/* ---------------- RFC 1951 section 3.2.5 code tables, built from their rules */

static int len_extra[29], len_base[29];     /* codes 257..285 */
static int dist_extra[30], dist_base[30];   /* codes 0..29 */
static int tables_ready = 0;
static pthread_mutex_t tables_lock = PTHREAD_MUTEX_INITIALIZER;

static void build_tables(void)
{
    pthread_mutex_lock(&tables_lock);
    if (!tables_ready) {
        /* length codes 257..284: extra bits 0 for the first 8, then one more
         * extra bit every 4 codes; lengths are consecutive from 3.  Code 285
         * is length 258 with no extra bits. */
        int base = 3;
        for (int k = 0; k < 28; ++k) {
            len_extra[k] = k < 8 ? 0 : (k - 4) / 4;
            len_base[k] = base;
            base += 1 << len_extra[k];
        }
        len_extra[28] = 0;
        len_base[28] = 258;
        /* distance codes 0..29: extra bits 0,0,0,0,1,1,2,2,...,13,13; distances
         * consecutive from 1. */
        base = 1;
        for (int k = 0; k < 30; ++k) {
            dist_extra[k] = k < 4 ? 0 : k / 2 - 1;
            dist_base[k] = base;
            base += 1 << dist_extra[k];
        }
        tables_ready = 1;
    }
    pthread_mutex_unlock(&tables_lock);
}

static int length_code_index(int len)   /* returns 0..28 (code - 257) */
{
    if (len == 258) return 28;
    for (int k = 27; k >= 0; --k)
        if (len >= len_base[k]) return k;
    return -1;
}

static int dist_code(int dist)
{
    for (int k = 29; k >= 0; --k)
        if (dist >= dist_base[k]) return k;
    return -1;
}

/* Fixed Huffman code lengths, RFC 1951 section 3.2.6. */
static int fixed_lit_len(int sym)
{
    if (sym <= 143) return 8;
    if (sym <= 255) return 9;
    if (sym <= 279) return 7;
    return 8;
}

/* ---------------- the parse ---------------------------------------------- */

typedef struct {
    int len;     /* 0 for a literal */
    int dist;    /* match distance */
    int lit;     /* literal byte */
} symbol_t;

static unsigned hash3(const uint8_t *w, int p)
{
    return ((unsigned)(w[p] << 10) ^ (unsigned)(w[p + 1] << 5) ^ (unsigned)w[p + 2]) & 0x7fffu;
}

/* Number of equal leading bytes of the strings at a and p (a < p), at most
 * MAX_MATCH, reading zero past the end of the input (w is zero padded). */
static int common_prefix(const uint8_t *w, int a, int p)
{
    int k = 0;
    while (k < MAX_MATCH && w[a + k] == w[p + k]) ++k;
    return k;
}

/* Greedy level-1 parse.  Returns the number of symbols written to syms. */
static int parse_level1(const uint8_t *w, int n, symbol_t *syms)
{
    /* head[h]: most recent inserted position with hash h (0 = empty);
     * prev[p]: the position head[h] held when p was inserted. */
    static const int max_chain = 4, nice_length = 8, max_insert = 4;
    int *head = (int *)calloc(1u << 15, sizeof(int));
    int *prev = (int *)calloc((size_t)n + 1, sizeof(int));
    int nsym = 0;
    int p = 0;
    while (p < n) {
        int remaining = n - p;
        int match_len = 0, match_dist = 0;
        if (remaining >= 3) {
            unsigned h = hash3(w, p);
            int cand = head[h];
            prev[p] = head[h];
            head[h] = p;
            if (cand != 0) {
                int nice = nice_length < remaining ? nice_length : remaining;
                int best = 2, best_pos = 0, chain = max_chain;
                for (;;) {
                    int l = common_prefix(w, cand, p);
                    if (l > best) {
                        best = l;
                        best_pos = cand;
                        if (l >= nice) break;
                    }
                    cand = prev[cand];
                    if (cand == 0 || --chain == 0) break;
                }
                if (best > remaining) best = remaining;
                if (best >= 3) {
                    match_len = best;
                    match_dist = p - best_pos;
                }
            }
        }
        if (match_len >= 3) {
            syms[nsym].len = match_len;
            syms[nsym].dist = match_dist;
            syms[nsym].lit = 0;
            ++nsym;
            if (match_len <= max_insert && remaining - match_len >= 3) {
                for (int q = p + 1; q < p + match_len; ++q) {
                    unsigned h = hash3(w, q);
                    prev[q] = head[h];
                    head[h] = q;
                }
            }
            p += match_len;
        } else {
            syms[nsym].len = 0;
            syms[nsym].dist = 0;
            syms[nsym].lit = w[p];
            ++nsym;
            p += 1;
        }
    }
    free(head);
    free(prev);
    return nsym;
}

/* ---------------- Huffman tree construction ------------------------------ */

/* Node store for one tree: leaves are the symbols 0..nelems-1, internal nodes
 * follow.  The priority of a node is its frequency, then its subtree depth;
 * nodes that are equal on both are ordered by their place in the heap. */
typedef struct {
    int freq[2 * NLIT + 1];
    int depth[2 * NLIT + 1];
    int parent[2 * NLIT + 1];
    int bits[2 * NLIT + 1];
    int heap[2 * NLIT + 2];   /* 1-based binary min-heap of node ids */
    int heap_len;
    int order[2 * NLIT + 1];  /* nodes in the order they left the heap */
    int norder;
} tree_work_t;

static int node_le(const tree_work_t *t, int a, int b)
{
    return t->freq[a] < t->freq[b] ||
           (t->freq[a] == t->freq[b] && t->depth[a] <= t->depth[b]);
}

/* Restore the heap property below slot k: walk down, at each level taking the
 * second child when it is not larger than the first, and stop as soon as the
 * moving node is not larger than that child. */
static void sift_down(tree_work_t *t, int k)
{
    int v = t->heap[k];
    int j = 2 * k;
    while (j <= t->heap_len) {
        if (j < t->heap_len && node_le(t, t->heap[j + 1], t->heap[j])) j++;
        if (node_le(t, v, t->heap[j])) break;
        t->heap[k] = t->heap[j];
        k = j;
        j = 2 * k;
    }
    t->heap[k] = v;
}

/*
 * Build the code lengths for one alphabet.  freq[0..nelems-1] in, lens out.
 * Returns the largest code that has a length (dummy codes included): the
 * header sends codes 0..max_code.
 */
static int build_lengths(const int *freq_in, int nelems, int max_bits, int *lens,
                         int *unclamped_depth)
{
    tree_work_t *t = (tree_work_t *)calloc(1, sizeof(tree_work_t));
    int max_code = -1;
    t->heap_len = 0;
    for (int s = 0; s < nelems; ++s) {
        lens[s] = 0;
        t->freq[s] = freq_in[s];
        t->depth[s] = 0;
        if (freq_in[s] != 0) {
            t->heap[++t->heap_len] = s;
            max_code = s;
        }
    }
    /* A code needs at least two symbols: add dummies of frequency 1, taking the
     * code just above the largest while that is below 2, else code 0.  Their
     * cost is never counted (the caller sums over real symbols only). */
    while (t->heap_len < 2) {
        int node = max_code < 2 ? ++max_code : 0;
        t->heap[++t->heap_len] = node;
        t->freq[node] = 1;
        t->depth[node] = 0;
    }
    for (int k = t->heap_len / 2; k >= 1; --k) sift_down(t, k);

    int next = nelems;
    t->norder = 0;
    do {
        int a = t->heap[1];
        t->heap[1] = t->heap[t->heap_len--];
        sift_down(t, 1);
        int b = t->heap[1];
        t->order[t->norder++] = a;
        t->order[t->norder++] = b;
        t->freq[next] = t->freq[a] + t->freq[b];
        t->depth[next] = (t->depth[a] >= t->depth[b] ? t->depth[a] : t->depth[b]) + 1;
        t->parent[a] = t->parent[b] = next;
        t->heap[1] = next++;
        sift_down(t, 1);
    } while (t->heap_len >= 2);
    t->order[t->norder++] = t->heap[1];      /* the root */

    /* Depths from the root down (reverse of the removal order), clamped at
     * max_bits; every node pushed past the limit, leaf or not, is counted. */
    int overflow = 0;
    int count[16] = {0};
    int root = t->order[t->norder - 1];
    t->bits[root] = 0;
    if (unclamped_depth) {
        /* statistics for the tests: the deepest leaf before clamping */
        int *ud = (int *)calloc(2 * NLIT + 1, sizeof(int));
        int deepest = 0;
        for (int r = t->norder - 2; r >= 0; --r) {
            int node = t->order[r];
            ud[node] = ud[t->parent[node]] + 1;
            if (node < nelems && ud[node] > deepest) deepest = ud[node];
        }
        *unclamped_depth = deepest;
        free(ud);
    }
    for (int r = t->norder - 2; r >= 0; --r) {
        int node = t->order[r];
        int d = t->bits[t->parent[node]] + 1;
        if (d > max_bits) { d = max_bits; overflow++; }
        t->bits[node] = d;
        if (node < nelems) count[d]++;
    }
    if (overflow > 0) {
        /* Each round moves one leaf from the deepest non-full level down one
         * level, pairing it with a leaf taken from the max_bits level. */
        do {
            int d = max_bits - 1;
            while (count[d] == 0) d--;
            count[d]--;
            count[d + 1] += 2;
            count[max_bits]--;
            overflow -= 2;
        } while (overflow > 0);
        /* Hand the lengths back out, longest first, to the leaves in the order
         * they left the heap (least frequent first). */
        int r = 0;
        for (int d = max_bits; d != 0; --d) {
            int c = count[d];
            while (c != 0) {
                int node = t->order[r++];
                if (node >= nelems) continue;
                t->bits[node] = d;
                c--;
            }
        }
    }
    for (int s = 0; s <= max_code; ++s)
        if (t->freq[s] != 0) lens[s] = t->bits[s];
    free(t);
    return max_code;
}

/* RFC 1951 section 3.2.2: canonical codes from code lengths. */
static void canonical_codes(const int *lens, int n, unsigned *codes)
{
    int bl_count[16] = {0};
    unsigned next_code[16] = {0};
    for (int s = 0; s < n; ++s) if (lens[s]) bl_count[lens[s]]++;
    unsigned code = 0;
    for (int bits = 1; bits <= 15; ++bits) {
        code = (code + bl_count[bits - 1]) << 1;
        next_code[bits] = code;
    }
    for (int s = 0; s < n; ++s) {
        codes[s] = 0;
        if (lens[s]) codes[s] = next_code[lens[s]]++;
    }
}

/* ---------------- code-length run-length coding (RFC 1951 section 3.2.7) - */

typedef struct { int sym; int extra_bits; int extra_val; } clsym_t;

/* Run-length code one code-length array lens[0..max_code]; appends to out.
 * Runs: a nonzero length repeated 4+ times is sent once and then as code 16
 * (3..6 repeats) — or only as code 16 when it equals the length sent just
 * before; zeros use code 17 (3..10) or 18 (11..138); shorter runs are sent
 * one by one. */
static int rle_lengths(const int *lens, int max_code, clsym_t *out, int nout)
{
    int prevlen = -1;
    int nextlen = lens[0];
    int count = 0;
    int max_count = 7, min_count = 4;
    if (nextlen == 0) { max_count = 138; min_count = 3; }
    for (int s = 0; s <= max_code; ++s) {
        int curlen = nextlen;
        nextlen = s + 1 <= max_code ? lens[s + 1] : -1;  /* -1: end of array */
        if (++count < max_count && curlen == nextlen) continue;
        if (count < min_count) {
            for (int k = 0; k < count; ++k) out[nout++] = (clsym_t){curlen, 0, 0};
        } else if (curlen != 0) {
            if (curlen != prevlen) {
                out[nout++] = (clsym_t){curlen, 0, 0};
                count--;
            }
            out[nout++] = (clsym_t){16, 2, count - 3};
        } else if (count <= 10) {
            out[nout++] = (clsym_t){17, 3, count - 3};
        } else {
            out[nout++] = (clsym_t){18, 7, count - 11};
        }
        count = 0;
        prevlen = curlen;
        if (nextlen == 0) { max_count = 138; min_count = 3; }
        else if (curlen == nextlen) { max_count = 6; min_count = 3; }
        else { max_count = 7; min_count = 4; }
    }
    return nout;
}

/* ---------------- bit output -------------------------------------------- */

typedef struct {
    uint8_t *out;
    long cap;
    long pos;
    uint32_t acc;
    int nbits;
    int overflow;
} bitwriter_t;

static void put_bits(bitwriter_t *bw, unsigned value, int nbits)
{
    for (int k = 0; k < nbits; ++k) {
        bw->acc |= ((value >> k) & 1u) << bw->nbits;
        if (++bw->nbits == 8) {
            if (bw->pos < bw->cap) bw->out[bw->pos] = (uint8_t)bw->acc;
            else bw->overflow = 1;
            bw->pos++;
            bw->acc = 0;
            bw->nbits = 0;
        }
    }
}

/* Huffman codes are sent most significant bit first. */
static void put_code(bitwriter_t *bw, unsigned code, int len)
{
    for (int k = len - 1; k >= 0; --k) put_bits(bw, (code >> k) & 1u, 1);
}

static void flush_to_byte(bitwriter_t *bw)
{
    if (bw->nbits > 0) put_bits(bw, 0, 8 - bw->nbits);
}

static void put_symbols(bitwriter_t *bw, const symbol_t *syms, int nsym,
                        const int *llen, const unsigned *lcode,
                        const int *dlen, const unsigned *dcode)
{
    for (int k = 0; k < nsym; ++k) {
        if (syms[k].len == 0) {
            put_code(bw, lcode[syms[k].lit], llen[syms[k].lit]);
        } else {
            int li = length_code_index(syms[k].len);
            put_code(bw, lcode[257 + li], llen[257 + li]);
            put_bits(bw, (unsigned)(syms[k].len - len_base[li]), len_extra[li]);
            int dc = dist_code(syms[k].dist);
            put_code(bw, dcode[dc], dlen[dc]);
            put_bits(bw, (unsigned)(syms[k].dist - dist_base[dc]), dist_extra[dc]);
        }
    }
    put_code(bw, lcode[256], llen[256]);
}

/* ---------------- the compressor ---------------------------------------- */

/*
 * Compress in[0..n) as one final DEFLATE block.  Writes the raw stream to
 * out (capacity cap) and returns its length in bytes, or a negative value:
 * -1 out of capacity, -2 n outside [0, 16383].
 * If out is NULL only the length is returned.
 * kind (optional) receives the block type: 0 stored, 1 fixed, 2 dynamic.
 */
static long deflate1(const uint8_t *in, long n, uint8_t *out, long cap, int *kind, int *depths)
{
    if (n < 0 || n > MAX_INPUT) return -2;
    build_tables();
    uint8_t *w = (uint8_t *)calloc((size_t)n + MAX_MATCH + 8, 1);
    if (n) memcpy(w, in, (size_t)n);
    symbol_t *syms = (symbol_t *)malloc(sizeof(symbol_t) * ((size_t)n + 1));
    int nsym = parse_level1(w, (int)n, syms);

    int lfreq[NLIT] = {0}, dfreq[NDIST] = {0};
    for (int k = 0; k < nsym; ++k) {
        if (syms[k].len == 0) lfreq[syms[k].lit]++;
        else {
            lfreq[257 + length_code_index(syms[k].len)]++;
            dfreq[dist_code(syms[k].dist)]++;
        }
    }
    lfreq[256] = 1;   /* end of block */

    int llen[NLIT + 2] = {0}, dlen[NDIST + 2] = {0};
    int lmax = build_lengths(lfreq, NLIT, 15, llen, depths ? &depths[0] : NULL);
    int dmax = build_lengths(dfreq, NDIST, 15, dlen, depths ? &depths[1] : NULL);

    clsym_t *cl = (clsym_t *)malloc(sizeof(clsym_t) * (NLIT + NDIST + 4));
    int ncl = rle_lengths(llen, lmax, cl, 0);
    ncl = rle_lengths(dlen, dmax, cl, ncl);
    int blfreq[NBL] = {0};
    for (int k = 0; k < ncl; ++k) blfreq[cl[k].sym]++;
    int bllen[NBL + 2] = {0};
    build_lengths(blfreq, NBL, 7, bllen, depths ? &depths[2] : NULL);
    static const int bl_order[NBL] = {16, 17, 18, 0, 8, 7, 9, 6, 10, 5, 11, 4, 12, 3, 13, 2, 14, 1, 15};
    int hclen = NBL;
    while (hclen > 4 && bllen[bl_order[hclen - 1]] == 0) hclen--;

    /* Costs in bits (without the 3 block-header bits). */
    long dyn_bits = 5 + 5 + 4 + 3L * hclen;
    long fix_bits = 0;
    for (int s = 0; s < NLIT; ++s) {
        if (!lfreq[s]) continue;
        int extra = s >= 257 ? len_extra[s - 257] : 0;
        dyn_bits += (long)lfreq[s] * (llen[s] + extra);
        fix_bits += (long)lfreq[s] * (fixed_lit_len(s) + extra);
    }
    for (int s = 0; s < NDIST; ++s) {
        if (!dfreq[s]) continue;
        dyn_bits += (long)dfreq[s] * (dlen[s] + dist_extra[s]);
        fix_bits += (long)dfreq[s] * (5 + dist_extra[s]);
    }
    static const int cl_extra[NBL] = {0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 2, 3, 7};
    for (int s = 0; s < NBL; ++s) dyn_bits += (long)blfreq[s] * (bllen[s] + cl_extra[s]);

    long opt_bytes = (dyn_bits + 3 + 7) / 8;
    long fix_bytes = (fix_bits + 3 + 7) / 8;
    if (fix_bytes <= opt_bytes) opt_bytes = fix_bytes;
    int type;
    if (n + 4 <= opt_bytes) type = 0;
    else if (fix_bytes == opt_bytes) type = 1;
    else type = 2;
    if (kind) *kind = type;

    uint8_t dummy[1];
    bitwriter_t bw = {out ? out : dummy, out ? cap : 0, 0, 0, 0, 0};
    put_bits(&bw, (unsigned)(type << 1) | 1u, 3);   /* BFINAL = 1, BTYPE */
    if (type == 0) {
        flush_to_byte(&bw);
        put_bits(&bw, (unsigned)n & 0xffffu, 16);
        put_bits(&bw, (~(unsigned)n) & 0xffffu, 16);
        for (long k = 0; k < n; ++k) put_bits(&bw, in[k], 8);
    } else if (type == 1) {
        int fl[288], fd[30];
        unsigned fcl[288], fcd[30];
        for (int s = 0; s < 288; ++s) fl[s] = fixed_lit_len(s);
        for (int s = 0; s < 30; ++s) fd[s] = 5;
        canonical_codes(fl, 288, fcl);
        canonical_codes(fd, 30, fcd);
        put_symbols(&bw, syms, nsym, fl, fcl, fd, fcd);
    } else {
        unsigned lcode[NLIT + 2], dcode[NDIST + 2], blcode[NBL + 2];
        canonical_codes(llen, NLIT, lcode);
        canonical_codes(dlen, NDIST, dcode);
        canonical_codes(bllen, NBL, blcode);
        put_bits(&bw, (unsigned)(lmax + 1 - 257), 5);
        put_bits(&bw, (unsigned)(dmax + 1 - 1), 5);
        put_bits(&bw, (unsigned)(hclen - 4), 4);
        for (int k = 0; k < hclen; ++k) put_bits(&bw, (unsigned)bllen[bl_order[k]], 3);
        for (int k = 0; k < ncl; ++k) {
            put_code(&bw, blcode[cl[k].sym], bllen[cl[k].sym]);
            if (cl[k].extra_bits) put_bits(&bw, (unsigned)cl[k].extra_val, cl[k].extra_bits);
        }
        put_symbols(&bw, syms, nsym, llen, lcode, dlen, dcode);
    }
    flush_to_byte(&bw);

    free(cl);
    free(syms);
    free(w);
    if (out && bw.overflow) return -1;
    return bw.pos;
}

long oracle_deflate1_raw(const uint8_t *in, long n, uint8_t *out, long cap, int *kind)
{
    return deflate1(in, n, out, cap, kind, NULL);
}

/* Deepest leaf of the literal/length, distance and code-length trees before
 * the length limits (15, 15, 7) are applied.  A value above the limit means
 * the length-limiting repair ran.  Returns the raw stream length. */
long oracle_deflate1_tree_depths(const uint8_t *in, long n, int *depths3)
{
    return deflate1(in, n, NULL, 0, NULL, depths3);
}

/* |gzip(x)| at level 1: 10-byte header + raw stream + 8-byte trailer. */
long oracle_gzip1_len(const uint8_t *in, long n)
{
    long raw = oracle_deflate1_raw(in, n, NULL, 0, NULL);
    return raw < 0 ? raw : raw + 18;
}

/* ---------------- batch driver over blocks ------------------------------ */

typedef struct {
    const uint8_t *bytes;
    long nblocks_total, b;
    int32_t *lengths;
    long first, last;
} job_t;

static void *run_job(void *arg)
{
    job_t *j = (job_t *)arg;
    for (long k = j->first; k < j->last; ++k)
        j->lengths[k] = (int32_t)oracle_gzip1_len(j->bytes + k * j->b, j->b);
    return NULL;
}

/*
 * lengths[s*N + i] = |gzip level 1 of block i of sample s|, for a row-major
 * [S][L] byte array split into N = L/b blocks.  Blocks are independent; the
 * loop over them is split over nthreads POSIX threads.  Returns 0, or -2 on
 * bad sizes.
 */
int oracle_gzip1_block_lengths(const uint8_t *bytes, long S, long L, long b,
                               int32_t *lengths, int nthreads)
{
    if (S < 0 || L < 0 || b <= 0 || b > MAX_INPUT || L % b != 0) return -2;
    build_tables();
    long total = S * (L / b);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (total < nthreads) nthreads = total > 0 ? (int)total : 1;
    pthread_t th[256];
    job_t jobs[256];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].bytes = bytes;
        jobs[t].nblocks_total = total;
        jobs[t].b = b;
        jobs[t].lengths = lengths;
        jobs[t].first = total * t / nthreads;
        jobs[t].last = total * (t + 1) / nthreads;
    }
    for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, run_job, &jobs[t]);
    run_job(&jobs[0]);
    for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
    return 0;
}
