// The library's dense GEMM, called by the ByteLM block (lm_block.cu) for its
// projections and weight gradients; defined with the tcgen05 kernels in the
// main translation unit (gemm.cuh).  Host-side declaration only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gsa.h"

namespace gsa {
namespace gemm {

// Epilogue on the float32 accumulator acc = op(A) op(B):
//   kNone:    D = acc + beta C                        (C, D bf16; or D float32 with beta 0)
//   kGeluAux: D = GELU(acc), aux = acc                (tanh form; D, aux bf16)
//   kDGelu:   D = acc * GELU'(aux)                    (aux bf16 in)
enum Epi { kNone = 0, kGeluAux = 1, kDGelu = 2 };

// Row-major D[M][N] = op(A)[M][K] op(B)[K][N] (+ epilogue).  ta: A is stored
// [K][M] (else [M][K]); tb: B is stored [N][K] (else [K][N]).  Leading
// dimensions in elements, 16-byte aligned rows.  N a multiple of 256, K of
// 64, M of 128 when A is stored [K][M] (any M otherwise); out32: D is float32
// (kNone, beta 0 only).  split_ws / split_ws_bytes: float32 scratch for a
// K split of a long-K float32 product (gemm_split_ws_bytes); may be null when
// none is needed.  Launches on st; never synchronises.
gsa_status run(bool ta, bool tb, int M, int N, int K, const __nv_bfloat16* A, int64_t lda,
               const __nv_bfloat16* B, int64_t ldb, float beta, const __nv_bfloat16* C, int64_t ldc, void* D,
               int64_t ldd, bool out32, Epi epi, __nv_bfloat16* aux, int64_t aux_ld, float* split_ws,
               size_t split_ws_bytes, cudaStream_t st);

// Scratch bytes run() needs for an M x N float32 product over K.
size_t split_ws_bytes(int M, int N, int K);

}  // namespace gemm
}  // namespace gsa
