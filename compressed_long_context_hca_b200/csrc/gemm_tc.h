// gemm_tc.h -- the tcgen05 GEMM of gemm_tc.cu (host side, not exported).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace hca {

// One bf16 operand of C = A . B^T. The array is row-major [rows, cols] with row stride ld
// elements (a multiple of 8; the base 16-byte aligned). K-major: cols run along K and rows
// along M (or N); MN-major: cols run along M (or N) and rows along K. The product element
// (mn, k) of batch z sits at array row shift + z * bstride + (K-major ? mn : k).
struct GemmOperand {
  const void* ptr;
  int64_t rows, cols, ld;
  bool mn_major;
  int32_t shift, bstride;
};

// float32 output: product row m of batch z goes to row shift + (z / zdiv) * bstride + m of
// a row-major array with row stride ld; rows outside [0, rows) are not written. atomic:
// C += alpha * A . B^T with float32 atomics (beta ignored), for batches that write the same
// rows (split-K, overlapping bands); the sum order is then not fixed.
// sigmoid_bf16: C = bf16(sigmoid(alpha * A . B^T)) into a bf16 array (ptr then points at
// bf16; beta and atomic unused).
struct GemmOutput {
  float* ptr;
  int64_t ld;
  int32_t shift, bstride, rows;
  int32_t zdiv;
  bool atomic;
  bool sigmoid_bf16;
};

// C = alpha * (A + A_lo) . B^T + beta * C for `batch` products of M x N over K (bf16 in,
// f32 out). A_lo (optional, may be nullptr): the low part of a bf16 pair, laid out as A
// (same rows, cols, major, shift, bstride); its product accumulates with A's in one pass.
cudaError_t gemm_tc(const GemmOperand& A, const GemmOperand* A_lo, const GemmOperand& B,
                    const GemmOutput& C, int M, int N, int K, int batch, float alpha, float beta,
                    int32_t* err_word, cudaStream_t s);

}  // namespace hca
