// Launchers of the partitioned-FFN kernels.
#pragma once

#include "common.cuh"

namespace tp {

enum { ACT_NONE = 0, ACT_RELU = 1, ACT_SWIGLU = 2 };

struct FfnMergeArgs {
  const float* P1;      // [nseg, M, N] partials of the first (or only) product
  const float* P3;      // [nseg, M, N] partials of the gate product (SwiGLU) or nullptr
  int64_t seg_stride;   // elements between segments
  int nseg, M, N;
  int quant;            // Q8 round trip of each partial before summing
  int act;              // ACT_NONE / ACT_RELU / ACT_SWIGLU
  const float* residual;  // optional [M, N] added after the activation
  float* out_f32;       // optional [M, N]
  uint16_t* out_bf16;   // optional [M, N], or hi/lo pairs [2M, N] when bf16_split
  int bf16_split;
};

int launch_gemm_simt(int dtype, const void* A, int64_t lda, const void* B, int64_t ldb, float* P,
                     int M, int N, int Ks, int nseg, cudaStream_t s);
int launch_ffn_merge(const FfnMergeArgs& a, cudaStream_t s);

}  // namespace tp
