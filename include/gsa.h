/*
 * gsa.h — C ABI of the gzip-guided sparse attention hot path on B200 (sm_100a).
 *
 * The method (Gzip-guided Sparse Attention, daiwk.github.io reproduction of
 * arXiv 2607.21752; abstract page "Parameter-free Adaptive Sparse Attention
 * via Compression-Based Content Selection"):
 *
 *   raw bytes -> fixed-size blocks -> gzip level-1 length of each block
 *   -> literal flags l_i = 1[r_i > mean r] -> per-head-class causal block
 *   mask M = M_lit ∪ M_local ∪ I -> block-sparse causal attention (forward,
 *   and the backward pass for training).
 *
 * Conventions for every call
 *   - Pointers are DEVICE pointers unless marked "host".  The caller owns all
 *     memory; the library allocates nothing on the device and keeps no state
 *     between calls (apart from the device error word of gsa_device_error).
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Work is only enqueued on that stream; no call synchronises it.
 *   - Arguments are checked on the host before anything is launched; a bad
 *     argument returns an error code and launches nothing.
 *   - Calls are thread-safe (no shared mutable host state).
 *   - Samples are called "B" in the argument lists below (batch size); the
 *     pages' own "B" (blocks per sample) is called nblk here.
 */
#ifndef GSA_H
#define GSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GSA_OK = 0,
    GSA_ERR_INVALID_ARGUMENT = 1, /* null pointer, bad size, inconsistent shapes */
    GSA_ERR_UNSUPPORTED = 2,      /* valid request outside what the kernels implement */
    GSA_ERR_CAPACITY = 3,         /* caller-provided buffer too small */
    GSA_ERR_CUDA = 4,             /* a CUDA launch or query failed */
    GSA_ERR_TIMEOUT = 5           /* a kernel gave up a bounded wait (gsa_device_error) */
} gsa_status;

typedef enum {
    GSA_HEAD_LOCAL = 0,   /* local window only:        M_local ∩ causal        */
    GSA_HEAD_LITERAL = 1, /* literal long-range + self: (M_lit ∪ I) ∩ causal   */
    GSA_HEAD_HYBRID = 2   /* union:        (M_lit ∪ M_local ∪ I) ∩ causal       */
} gsa_head_class;

typedef enum { GSA_F32 = 0, GSA_BF16 = 1 } gsa_dtype;

/* Largest block size (bytes) gsa_block_lengths accepts. */
#define GSA_MAX_BLOCK_BYTES 128
/* Largest number of heads an attention call accepts. */
#define GSA_MAX_HEADS 256
/* Largest number of blocks per sample the bf16 attention accepts. */
#define GSA_MAX_BLOCKS_BF16 2048

/*
 * gsa_block_lengths — per-block gzip level-1 compressed size.
 *
 * Gzip-guided Sparse Attention, section "核心公式", r_i equation:
 * r_i = |gzip(x_{ib:(i+1)b})| / b, each block compressed on its own at gzip
 * level 1.  This call returns |gzip(block)| in bytes: the size of the stream
 * Python's gzip.compress(block, compresslevel=1) produces — a 10-byte header,
 * the raw DEFLATE stream of zlib level 1 (window 15 bits, memory level 8,
 * default strategy), and an 8-byte trailer.  Exact, integer.
 *
 *   bytes    [B][L] uint8, row-major (sample s, byte t at s*L + t)
 *   B        samples, >= 1
 *   L        bytes per sample, a multiple of b, >= b
 *   b        block size in bytes, 1 <= b <= GSA_MAX_BLOCK_BYTES
 *   lengths  [B][L/b] int32 out: lengths[s*(L/b) + i] for block i of sample s
 * Errors: GSA_ERR_INVALID_ARGUMENT for null pointers or bad sizes.
 */
gsa_status gsa_block_lengths(const uint8_t* bytes, int32_t B, int64_t L, int32_t b,
                             int32_t* lengths, void* stream);

/*
 * gsa_literal_flags — the literal flag of every block.
 *
 * Section "核心公式": l_i = 1[r_i > r̄], r̄ the mean of r_j over the nblk
 * blocks of the same sample ("背景与主要改动": above the sample mean).  With
 * r_i = len_i / b this is exactly len_i * nblk > Σ_j len_j, which the kernel
 * evaluates in 64-bit integers.  Ties are not literal (strict >).
 *
 *   lengths  [B][nblk] int32 (as written by gsa_block_lengths; any values)
 *   flags    [B][nblk] uint8 out, 0 or 1
 * Errors: GSA_ERR_INVALID_ARGUMENT for null pointers, B < 1 or nblk < 1.
 */
gsa_status gsa_literal_flags(const int32_t* lengths, int32_t B, int32_t nblk, uint8_t* flags,
                             void* stream);

/*
 * Block lists of the mask, per sample s and head class c (0 local, 1 literal,
 * 2 hybrid), at block granularity.  Section "核心公式", mask equation:
 * M = M_lit ∪ M_local ∪ I with M_lit_ij = 1[l_i = l_j = 1],
 * M_local_ij = 1[|i - j| <= w], intersected with the causal mask; section
 * "背景与主要改动": local heads see M_local, literal heads M_lit ∪ I (each block
 * keeps itself), hybrid heads all of M.  The causal cut inside the diagonal
 * block is token-level and applied by the attention calls.
 *
 * All arrays are device memory the caller allocates; g = s*3 + c:
 *   row_ptr [B][3][nblk+1]  CSR: the key blocks of query block i are
 *   col_idx [B][3][capacity]     col_idx[g*capacity + row_ptr[g*(nblk+1) + i] ..
 *                                        g*capacity + row_ptr[g*(nblk+1) + i+1] - 1],
 *                                ascending.  row_ptr[g*(nblk+1) + nblk] = live pairs.
 *   col_ptr [B][3][nblk+1]  CSC: the query blocks that see key block j,
 *   row_idx [B][3][capacity]     ascending, same indexing.
 *   q_order [B][3][nblk]    query blocks in the order the attention pairs them
 *                           into 128-row tiles (entries 2t and 2t+1 form tile
 *                           t): literal blocks together, heaviest first.
 *   k_order [B][3][nblk]    key blocks in the order the backward pass pairs
 *                           them into 128-row key tiles.
 * capacity must be >= gsa_csr_capacity(nblk) (the dense causal count).
 * Every list holds its own block (i in row i, j in column j), as the mask
 * equation's I term guarantees; the attention backward at d = 64 relies on
 * it, and a list given to it without its own block ends in a bounded wait
 * that sets the device error (gsa_device_error: GSA_ERR_TIMEOUT).
 */
typedef struct {
    int32_t B;
    int32_t nblk;
    int32_t w;          /* set by gsa_build_block_csr */
    int32_t classes;    /* bit c set: the lists of head class c were built; bit 3: the local
                           class's lists are implicit — not stored: the attention calls derive
                           row i = key blocks max(0, i - w) .. i from (nblk, w) (set by the
                           builders: gsa_mask_pipeline sets it when the local class is in use) */
    int64_t capacity;   /* entries per (sample, class) in col_idx and row_idx */
    int32_t* row_ptr;
    int32_t* col_idx;
    int32_t* col_ptr;
    int32_t* row_idx;
    int32_t* q_order;
    int32_t* k_order;
} gsa_block_csr;

/*
 * gsa_build_fixed_csr — the same lists for a fixed, content-blind block mask,
 * so that the attention calls run the masks the method is compared with.
 * Background paragraph of section "核心公式" and the arXiv abstract name
 * BigBird and Longformer as those baselines; the pages do not define them,
 * so their published patterns are taken at block granularity, causal:
 *   GSA_FIXED_LONGFORMER: live(i, j) = j <= i and (i - j <= w or j < g or i < g)
 *     (a sliding window of w blocks each side, the first g blocks global);
 *   GSA_FIXED_BIGBIRD: the same, or j = u_ik mod (i + 1) for some k < r
 *     (r random key blocks per query block, drawn causally).
 *   rnd  device uint32 [csr->B][csr->nblk][r]: the random words u_ik (the
 *        caller draws them); BigBird with r > 0 only, else ignored (may be NULL).
 * All three class slots of each sample receive the same lists, so every
 * head, whatever its class, attends with the fixed mask.  Lists ascend;
 * q_order is nblk-1 .. 0 (heaviest query blocks first), k_order 0 .. nblk-1.
 * Errors: GSA_ERR_INVALID_ARGUMENT (unknown kind, w, g or r < 0, null
 * pointers), GSA_ERR_UNSUPPORTED (nblk > GSA_MAX_FIXED_BLOCKS or
 * r > GSA_MAX_RANDOM_BLOCKS), GSA_ERR_CAPACITY (capacity <
 * gsa_csr_capacity(nblk)).
 */
#define GSA_FIXED_LONGFORMER 0
#define GSA_FIXED_BIGBIRD 1
#define GSA_MAX_FIXED_BLOCKS 8192
#define GSA_MAX_RANDOM_BLOCKS 8
gsa_status gsa_build_fixed_csr(int32_t kind, int32_t w, int32_t g, int32_t r, const uint32_t* rnd,
                               gsa_block_csr* csr, void* stream);

/* Worst-case live pairs of one (sample, class): nblk*(nblk+1)/2. */
int64_t gsa_csr_capacity(int32_t nblk);

/*
 * gsa_build_block_csr — the lists above from the literal flags, for the head
 * classes the heads use.
 *
 *   flags         [csr->B][csr->nblk] uint8 (nonzero = literal)
 *   w             local window in blocks, >= 0
 *   head_classes  host [H], each 0, 1 or 2 (gsa_head_class): the lists are
 *                 built only for the classes that appear (a class's slots of
 *                 the arrays are left untouched otherwise); NULL builds all
 *                 three (H is then ignored)
 *   H             heads, 1 .. GSA_MAX_HEADS (when head_classes is given)
 *   csr           host struct; its B, nblk, capacity and device pointers are
 *                 read, w and classes (the bitmask of classes built) are written.
 * The attention calls reject a head whose class's lists were not built.
 * Errors: GSA_ERR_INVALID_ARGUMENT (null pointers, sizes < 1, w < 0, H out of
 *         range, a class outside 0..2), GSA_ERR_CAPACITY (capacity <
 *         gsa_csr_capacity(nblk)).
 */
gsa_status gsa_build_block_csr(const uint8_t* flags, int32_t w, const uint8_t* head_classes, int32_t H,
                               gsa_block_csr* csr, void* stream);

/*
 * gsa_mask_pipeline — gsa_block_lengths, gsa_literal_flags and
 * gsa_build_block_csr in one launch.
 *
 * The flowchart of the pages (gzip level-1 per block -> r_i > r̄ -> mask per
 * head class) as one pass: a cooperative launch whose CTAs first compute all
 * lengths, meet at a grid barrier, then share out the (sample, class) list
 * jobs, each of which computes its sample's flags.  The local class's lists
 * depend only on (nblk, w) (the mask equation's window intersected with
 * causality): they are not written at all, csr->classes gets bit 3
 * (value 8) to say so, and the attention calls derive them.  Lengths, flags
 * and the other classes' lists are those of the three calls, bit for bit,
 * and attention on these lists gives the three calls' results bit for bit.
 *
 *   bytes, B, L, b   as for gsa_block_lengths; L / b = nblk <= GSA_MAX_PIPELINE_BLOCKS
 *   w                local window in blocks, >= 0
 *   head_classes, H  as for gsa_build_block_csr (NULL: all three classes)
 *   lengths          [B][nblk] int32 out
 *   flags            [B][nblk] uint8 out
 *   csr              as for gsa_build_block_csr (csr->B == B, csr->nblk == nblk)
 *   counter          one int32 of device scratch owned by the caller (the
 *                    grid barrier's counter): zero before the first call;
 *                    every completed call leaves it zero.  Two calls in
 *                    flight at once must not share it.  After a call whose
 *                    barrier timed out (a device error code is recorded) it
 *                    must be zeroed again.
 * Errors: GSA_ERR_INVALID_ARGUMENT (null pointers, bad sizes, csr shape, H or
 *         a class out of range), GSA_ERR_UNSUPPORTED (nblk >
 *         GSA_MAX_PIPELINE_BLOCKS: use the three calls), GSA_ERR_CAPACITY
 *         (capacity < gsa_csr_capacity(nblk)), GSA_ERR_CUDA (the cooperative
 *         launch was refused).
 */
#define GSA_MAX_PIPELINE_BLOCKS 1024
gsa_status gsa_mask_pipeline(const uint8_t* bytes, int32_t B, int64_t L, int32_t b, int32_t w,
                             const uint8_t* head_classes, int32_t H, int32_t* lengths, uint8_t* flags,
                             gsa_block_csr* csr, int32_t* counter, void* stream);

/*
 * Attention problem description (host struct).
 *   q, k, v, o, dq, dk, dv: [B][H][L][d] contiguous, element type dtype.
 *   lse: [B][H][L] float32, natural log of the softmax denominator,
 *        lse_t = ln Σ_{u visible} exp(scale * q_t·k_u).
 *   head_classes: host [H], each 0, 1 or 2 (gsa_head_class).
 *   scale: softmax scale; 0 means 1/sqrt(d).
 * Kernels: dtype GSA_F32 runs a CUDA-core float32 forward (any b in 1..128,
 * d in {16, 32, 64, 128}); GSA_BF16 runs the tcgen05 tensor-core path
 * (b = 64, d in {64, 128}, nblk <= GSA_MAX_BLOCKS_BF16) with float32
 * accumulation and softmax.
 */
/*
 * Layout of the attention tensors, in elements (bf16 calls only).  Element
 * (sample s, head h, token l, e) of q, k, v, dq, dk and dv is at
 * s*qkv_s + h*qkv_h + l*qkv_l + e from its base pointer; of o and dO at
 * s*o_s + h*o_h + l*o_l + e.  Every stride is a positive multiple of 8
 * (16 bytes, the TMA rule) and the token strides are >= d; the caller keeps
 * the written tensors (o, dq, dk, dv) free of overlaps.  Example: with one
 * token-major projection output qkv [B][L][3][H][d], q = qkv, k = qkv + H*d,
 * v = qkv + 2*H*d and qkv_s = 3*L*H*d, qkv_h = d, qkv_l = 3*H*d.
 */
typedef struct {
    int64_t qkv_s, qkv_h, qkv_l;
    int64_t o_s, o_h, o_l;
} gsa_attn_layout;

typedef struct {
    int32_t B, H;
    int64_t L;          /* tokens (bytes) per sample = nblk * b */
    int32_t d;          /* head dimension */
    int32_t b;          /* block size in tokens */
    int32_t dtype;      /* gsa_dtype */
    float scale;
    const uint8_t* head_classes;
    const gsa_attn_layout* layout;   /* host; NULL: dense [B][H][L][d] for every tensor */
} gsa_attn_desc;

/*
 * gsa_attn_fwd — block-sparse causal attention forward.
 *
 * Section "复现边界": the reproduction forms softmax(Q K^T / sqrt(d) + mask) V
 * densely and masks it.  This call computes the same output visiting only
 * live blocks: for sample s, head h of class c = head_classes[h] and query
 * token t in block i,
 *   o_t = Σ_{u in A(t)} softmax_u(scale * q_t·k_u) v_u,
 *   A(t) = { u <= t : block(u) in the CSR row i of (s, c) }.
 *   o [B][H][L][d] out (or desc->layout's strides), lse [B][H][L] float32 out
 *   (dense always; may be NULL for GSA_F32).
 * bf16 at d = 64 runs persistent CTAs that draw work items from a counter in
 * the library's device memory: one of 256 slots, taken in turn per call and
 * returned to zero by the call's last CTA, so up to 256 such calls may be in
 * flight at once (on any streams) on one device.  The slot is chosen on the
 * host when the call is made: a call captured into a CUDA graph keeps its
 * slot for every replay, so replays of that graph must not overlap one
 * another, nor run beside 256 or more later eager calls (which wrap round
 * onto the same slot); overlapping users of one slot skip or repeat work
 * items without any error being reported.  Every query row needs at
 * least one live key, as in every mask built by this library (each block
 * sees itself); a row without one has no defined output.
 * Errors: GSA_ERR_INVALID_ARGUMENT (null pointers, L != nblk*b, shapes that
 * disagree with csr, a class outside 0..2, bf16 tensors not 16-byte aligned,
 * a layout breaking its rules), GSA_ERR_UNSUPPORTED (dtype / b / d outside the
 * kernels above, a layout with GSA_F32), GSA_ERR_CUDA.
 */
gsa_status gsa_attn_fwd(const void* q, const void* k, const void* v, const gsa_block_csr* csr,
                        const gsa_attn_desc* desc, void* o, float* lse, void* stream);

/*
 * gsa_attn_bwd — gradients of the forward above (training; section
 * "论文离线与线上效果" trains the model for 20K steps).  With P the softmax,
 * D_t = Σ_e dO_te O_te:
 *   dV = P^T dO,  dS = P ∘ (dO V^T − D),  dQ = scale · dS K,  dK = scale · dS^T Q,
 * every sum over live pairs only.  o and lse are the forward's outputs.
 *   workspace: device scratch of at least gsa_attn_bwd_workspace(desc) bytes
 *              (holds -D and -LSE log2(e), float32 [B][H][L] each, then two
 *              work counters); its contents need no init.
 * dq, dk, dv are written (not accumulated).  Deterministic: each output row
 * is summed by one CTA in a fixed order (the only atomic hands out work
 * items).
 * Errors: as gsa_attn_fwd, plus GSA_ERR_CAPACITY when ws_bytes is too small.
 * Only GSA_BF16 is implemented.
 */
gsa_status gsa_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dO, const gsa_block_csr* csr,
                        const gsa_attn_desc* desc, void* dq, void* dk, void* dv,
                        void* workspace, size_t ws_bytes, void* stream);

size_t gsa_attn_bwd_workspace(const gsa_attn_desc* desc);

/*
 * gsa_attn_bwd_noalloc — gsa_attn_bwd for callers that cannot allocate
 * device memory.  The paper has no counterpart: this is a deployment
 * variant.  Some callers own no allocator of their own (a host framework
 * that hands out every device byte from its pool and forbids other
 * allocations) or cannot afford cudaMalloc's implicit device
 * synchronisation in their loop.  This call needs no workspace argument: its
 * float32 scratch (D_t and LSE_t log2(e), two values per query row) is a fixed array compiled
 * into the library, at most gsa_attn_bwd_noalloc_max_rows() rows
 * (2^21 = B*H*L; 16 MiB, held on every GPU that loads the library until the
 * process exits).  The caller still passes all inputs and outputs, exactly as
 * for gsa_attn_bwd; results are identical.
 *   - Allocates nothing: no cudaMalloc / cudaFree, no allocating library call.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls share the one array, which keeps the last call's contents
 *     (every call overwrites the rows it uses before reading them, so nothing
 *     needs clearing).  Calls that overlap on the GPU (other streams, other
 *     threads) race on it: serialise them.
 * Errors: as gsa_attn_bwd; GSA_ERR_CAPACITY when B*H*L exceeds the maximum.
 */
gsa_status gsa_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dO, const gsa_block_csr* csr,
                                const gsa_attn_desc* desc, void* dq, void* dk, void* dv, void* stream);

/* Rows (B*H*L) gsa_attn_bwd_noalloc can take. */
int64_t gsa_attn_bwd_noalloc_max_rows(void);

/*
 * gsa_device_error — read (and optionally clear) the library's device error
 * word.  Kernels that give up a bounded wait record a nonzero code there
 * instead of hanging.  Synchronises the device.  *code receives the word
 * (0 = none); returns GSA_ERR_TIMEOUT when it is nonzero, GSA_OK otherwise.
 */
gsa_status gsa_device_error(int32_t* code, int32_t clear);

const char* gsa_status_string(gsa_status status);

#ifdef __cplusplus
}
#endif

#endif /* GSA_H */
