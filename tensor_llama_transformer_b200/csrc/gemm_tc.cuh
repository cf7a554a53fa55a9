// Tensor-core (tcgen05 / TMEM / TMA) contraction: the batched FFN and the
// batched decode slice products.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace tp {

enum TcEpi {
  TC_EPI_STORE_F32 = 0,    // out[seg][m][n] = acc                        (float32)
  TC_EPI_RELU_BF16 = 1,    // out[m][n] = bf16(max(acc, 0))
  TC_EPI_SWIGLU_BF16 = 2,  // out[m][n] = bf16(silu(acc_W1) * acc_W3)    (B = W1, B2 = W3)
  TC_EPI_STORE_T_F32 = 3,  // out[seg][n][row_off(matrix) + m] = acc     (transposed float32)
  TC_EPI_STORE_T_PAIRS_F32 = 4,  // as 3 with B rows in hi/lo pairs: out[seg][n/2][..] = acc_2j + acc_2j+1
  // out[m][n] = sum over seg = 0, 1, ... of sync(acc_seg[m][n]), in segment order, float32:
  // each segment's partial is formed on its own (a fresh accumulator) and, with g.quant,
  // passes the Q8 round trip (blocks of 32 columns) before it is added
  TC_EPI_SEGSUM_F32 = 5,
  TC_EPI_SEGSUM_RELU_BF16 = 6,  // as 5, then out[m][n] = bf16(max(sum, 0))
};

// D[seg, m, n] = sum_{k < K} A[m, seg*K + k] * B[n, seg*K + k]
// A and B are bf16 row-major with the contraction dimension contiguous. Up to
// three A matrices (same K and leading dimension) may be given; their rows are
// concatenated, which TC_EPI_STORE_T_F32 reproduces in its output rows. The FFN
// uses A = activations [tokens, K], B = weights [features, K]; batched decode
// uses A = weights [rows, K], B = activations [batch, K] (N <= 128) with the
// transposed store, so that each partial plane is [batch, rows]; with the
// activations given as hi/lo bf16 row pairs (N = 2 x batch) the pair-folding
// store adds the two columns of each batch row.
struct TcGemm {
  const void* A[3];
  int Am[3];        // rows of each A matrix
  int nA;           // 1..3
  int64_t lda;
  const void* B;
  int64_t ldb;
  const void* B2;   // second B operand (SwiGLU gate), same shape as B
  int N, K;         // K = contraction length of one segment
  int nseg;
  int epi;
  void* out;
  int64_t ldo;
  int64_t out_seg;  // elements between segment planes (float32 stores)
  int quant;        // TC_EPI_SEGSUM_*: Q8 round trip of every segment's partial
  int* err;         // device flag set to 1 when a pipeline wait gives up (nullable: not reported)
  // Operands that no kernel before this one writes (TC_INDEP_A / TC_INDEP_B, e.g. the
  // weights): under programmatic dependent launch the producer loads their tiles for
  // the first ring stages before waiting for the previous kernel, the others after.
  int indep;
};
enum { TC_INDEP_A = 1, TC_INDEP_B = 2 };

int launch_tc_gemm(const TcGemm& g, cudaStream_t s);

// 2D TMA map over a bf16 row-major matrix [rows, cols] with row stride `ld`
// elements: box box_cols x box_rows, 128-byte swizzle, zero fill past the edges.
bool make_tensor_map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                        uint64_t ld, int box_cols, int box_rows);
// 3D map over a row-major matrix [rows, ld] of esize-byte elements (2: bf16, 1: int8)
// viewed as {chunk, ld / chunk, rows} (no swizzle): a box of box_rows consecutive rows
// of nchunk * chunk columns lands in shared memory row-major. ld % chunk == 0; chunk,
// nchunk, box_rows <= 256; chunk * esize a multiple of 16.
bool make_tensor_map_rows(CUtensorMap* m, const void* base, uint64_t rows, uint64_t ld, int chunk,
                          int nchunk, int box_rows, int esize);

}  // namespace tp
