// Tensor-core (tcgen05 / TMEM / TMA) contraction for the batched FFN.
#pragma once

#include "common.cuh"

namespace tp {

enum TcEpi {
  TC_EPI_STORE_F32 = 0,    // out[seg][m][n] = acc                       (float32)
  TC_EPI_RELU_BF16 = 1,    // out[m][n] = bf16(max(acc, 0))
  TC_EPI_SWIGLU_BF16 = 2,  // out[m][n] = bf16(silu(acc_W1) * acc_W3)   (B = W1, B2 = W3)
};

// D[seg, m, n] = sum_{k < K} A[m, seg*K + k] * B[n, seg*K + k]
// A [M, lda] and B [N, ldb] are bf16 row-major (contraction dimension contiguous).
struct TcGemm {
  const void* A;
  int64_t lda;
  const void* B;
  int64_t ldb;
  const void* B2;   // second B operand (SwiGLU gate), same shape as B
  int M, N, K;      // K = contraction length of one segment
  int nseg;
  int epi;
  void* out;
  int64_t ldo;
  int64_t out_seg;  // elements between segment planes (TC_EPI_STORE_F32)
  int* err;         // device flag set to 1 when a pipeline wait gives up (nullable: not reported)
};

int launch_tc_gemm(const TcGemm& g, cudaStream_t s);

}  // namespace tp
