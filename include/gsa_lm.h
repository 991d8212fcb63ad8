/*
 * gsa_lm.h — one ByteLM transformer block around the attention of gsa.h
 * (forward and backward), so the attention can be timed in the model it
 * trains.
 *
 * Gzip-guided Sparse Attention (daiwk.github.io): the fidelity line ("训练同参数
 * ByteLM") and section "论文离线与线上效果" train a byte-level LM of 92M
 * parameters at 8K bytes with the adaptive mask; the arXiv abstract states
 * the same.  The pages give no block layout; the one taken here:
 *
 *   x0 = E[bytes]                              (learned byte embedding, no positions)
 *   x1 = x0 + Attn(LN1(x0)) W_o^T              (Q, K, V = LN1(x0) W_qkv^T split
 *                                               into H heads of 64; block-sparse
 *                                               causal attention of gsa_attn_fwd,
 *                                               scale 1/8, one class per head)
 *   y  = x1 + GELU(LN2(x1) W_1^T) W_2^T        (tanh-form GELU, applied to the
 *                                               float32 product)
 *
 * LayerNorm: (x - mean) / sqrt(var + eps) * gain + bias, biased variance.
 * Linear layers have no bias.  D = 768, H = 12, F = 3072 is the width of a
 * 12-block, ~85M-weight model, the paper's size class.
 *
 * Conventions as in gsa.h (device pointers, caller-owned memory, stream as
 * void*, host-side argument checks before any launch, nothing synchronises);
 * every pointer passed to these calls must be 16-byte aligned.
 * The projections run on this library's tcgen05 GEMM (bf16 operands,
 * float32 accumulation in TMEM, the residual additions, the GELU and its
 * derivative in its epilogue; the long-K weight gradients split K and sum
 * the parts in a fixed order, so results repeat bit for bit).  Every kernel
 * of the block is this library's own.
 */
#ifndef GSA_LM_H
#define GSA_LM_H

#include "gsa.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int32_t B;                      /* samples */
    int32_t L;                      /* bytes (tokens) per sample, a multiple of b */
    int32_t D;                      /* model width = 64 * H, a multiple of 256, <= 2048 */
    int32_t H;                      /* heads (head dimension 64) */
    int32_t F;                      /* MLP width, a multiple of 256 */
    int32_t b;                      /* mask block size in bytes: 64 */
    const uint8_t* head_classes;    /* host [H]: gsa_head_class of each head */
    float ln_eps;                   /* LayerNorm epsilon (> 0) */
} gsa_lm_desc;

/* Weights, device, row-major: a linear layer's matrix is [out][in]. */
typedef struct {
    const void* emb;     /* bf16 [256][D] */
    const float* ln1_g;  /* float32 [D] */
    const float* ln1_b;  /* float32 [D] */
    const void* w_qkv;   /* bf16 [3D][D]: rows Q (heads of 64 in order), then K, then V */
    const void* w_o;     /* bf16 [D][D] */
    const float* ln2_g;  /* float32 [D] */
    const float* ln2_b;  /* float32 [D] */
    const void* w_1;     /* bf16 [F][D] */
    const void* w_2;     /* bf16 [D][F] */
} gsa_lm_weights;

/* Gradients of <y, dy> (float32, same shapes; written, not accumulated). */
typedef struct {
    float* emb;
    float* ln1_g;
    float* ln1_b;
    float* w_qkv;
    float* w_o;
    float* ln2_g;
    float* ln2_b;
    float* w_1;
    float* w_2;
} gsa_lm_grads;

/*
 * Bytes of device workspace the two calls below need (0 for an invalid
 * desc): the activations the forward saves for the backward (about
 * B*L*(10 D + 4 F) bytes), the backward's scratch (about B*L*(12 D + 2 F)),
 * the attention backward's workspace and the float32 scratch of the K-split
 * weight-gradient products (a few times D F float32).
 */
size_t gsa_lm_block_workspace(const gsa_lm_desc* desc);

/*
 * gsa_lm_block_fwd — y (bf16 [B][L][D]) of the block for the bytes
 * (uint8 [B][L]) under the block lists csr (from gsa_build_block_csr,
 * gsa_mask_pipeline or gsa_build_fixed_csr for the same B and L / b).
 * The workspace keeps the activations gsa_lm_block_bwd reads: pass the same
 * workspace, unchanged, to the backward of this forward.
 * Errors: GSA_ERR_INVALID_ARGUMENT (null or unaligned pointers, D != 64 H, b != 64,
 * L % b, a class outside 0..2, F % 8), GSA_ERR_UNSUPPORTED (D % 256, F % 256,
 * D > 2048, L / b > GSA_MAX_BLOCKS_BF16),
 * GSA_ERR_CAPACITY (ws_bytes too small), GSA_ERR_CUDA, and the attention's
 * errors.
 */
gsa_status gsa_lm_block_fwd(const uint8_t* bytes, const gsa_lm_weights* w, const gsa_block_csr* csr,
                            const gsa_lm_desc* desc, void* y, void* workspace, size_t ws_bytes, void* stream);

/*
 * gsa_lm_block_bwd — gradients of <y, dy> for every weight of the forward
 * that last used this workspace (dy bf16 [B][L][D]).  The weight gradients
 * are float32 GEMM outputs; the gain / bias and embedding gradients are
 * summed in a fixed order, so repeated calls give identical results.
 * Errors: as gsa_lm_block_fwd.
 */
gsa_status gsa_lm_block_bwd(const uint8_t* bytes, const gsa_lm_weights* w, const gsa_block_csr* csr,
                            const gsa_lm_desc* desc, const void* dy, const gsa_lm_grads* g, void* workspace,
                            size_t ws_bytes, void* stream);

/*
 * gsa_lm_gemm — the block's projection primitive on its own: row-major
 * D[M][N] = op(A)[M][K] op(B)[K][N] on the tcgen05 tensor cores, bf16
 * operands, float32 accumulation, then
 *   epi 0: D = acc + beta C     (C, D bf16; or, with out32, D float32 and beta 0)
 *   epi 1: D = GELU(acc), aux = acc          (tanh form; D, aux bf16)
 *   epi 2: D = acc * GELU'(aux)              (aux bf16 in)
 *   ta: A stored [K][M] (else [M][K]); tb: B stored [N][K] (else [K][N]).
 * Leading dimensions in elements; every row 16-byte aligned.  N a multiple
 * of 256, K of 64, M of 128 when ta.  A float32 product with too few output
 * tiles to fill the device splits K, sums the parts in a fixed order and
 * needs gsa_lm_gemm_workspace bytes of device scratch (0 otherwise).
 * Errors: GSA_ERR_INVALID_ARGUMENT (null pointers, misaligned leading
 * dimensions), GSA_ERR_UNSUPPORTED (shapes above, out32 with an epilogue or
 * beta), GSA_ERR_CAPACITY (workspace too small), GSA_ERR_CUDA.
 */
gsa_status gsa_lm_gemm(int32_t ta, int32_t tb, int32_t M, int32_t N, int32_t K, const void* A, int64_t lda,
                       const void* B, int64_t ldb, float beta, const void* C, int64_t ldc, void* D, int64_t ldd,
                       int32_t out32, int32_t epi, void* aux, int64_t aux_ld, void* workspace, size_t ws_bytes,
                       void* stream);
size_t gsa_lm_gemm_workspace(int32_t M, int32_t N, int32_t K, int32_t out32);

#ifdef __cplusplus
}
#endif

#endif /* GSA_LM_H */
