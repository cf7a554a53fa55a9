// Partitioned FFN building blocks on CUDA cores: a segmented contraction for
// float32 operands and the cross-slice merge with the activation.
//
//   P[seg, m, n] = sum_{k in K_seg} A[m, k] * B[n, k]        (A [M, lda], B [N, ldb])
//   out[m, n]    = act( sum_seg sync(P1[seg, m, n]) [, sum_seg sync(P3[seg, m, n])] )
//
// The segments are the slices of a row split (aiterms.tw "Tensor Parallelism",
// Linear2 split by rows; Pope et al. demo1 2D stage sums). The merge sums them
// in slice order in float32 with the optional Q8 round trip of each partial,
// i.e. the all-reduce as the receiving side sees it.
#include "ffn.cuh"

namespace tp {

namespace {

constexpr int TBM = 64, TBN = 64, TBK = 16;

template <typename T>
TP_DEV float ld_val(const T* p);
template <>
TP_DEV float ld_val<float>(const float* p) { return *p; }
template <>
TP_DEV float ld_val<uint16_t>(const uint16_t* p) { return __uint_as_float(((uint32_t)*p) << 16); }

// 64x64 output tile per CTA, 256 threads, 4x4 outputs per thread.
template <typename T>
__global__ void __launch_bounds__(256) k_gemm_simt(const T* __restrict__ A, int64_t lda,
                                                   const T* __restrict__ B, int64_t ldb,
                                                   float* __restrict__ P, int M, int N, int Ks,
                                                   int64_t seg_stride) {
  __shared__ float As[TBK][TBM + 4];
  __shared__ float Bs[TBK][TBN + 4];
  const int seg = blockIdx.z;
  const int m0 = blockIdx.y * TBM, n0 = blockIdx.x * TBN;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const size_t k0 = (size_t)seg * Ks;
  float acc[4][4] = {};
  for (int kk = 0; kk < Ks; kk += TBK) {
    for (int i = threadIdx.x; i < TBM * TBK; i += 256) {
      const int r = i / TBK, k = i - r * TBK;
      const int gm = m0 + r, gn = n0 + r, gk = kk + k;
      As[k][r] = (gm < M && gk < Ks) ? ld_val(A + (size_t)gm * lda + k0 + gk) : 0.f;
      Bs[k][r] = (gn < N && gk < Ks) ? ld_val(B + (size_t)gn * ldb + k0 + gk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < TBK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn < N) P[(size_t)seg * seg_stride + (size_t)gm * N + gn] = acc[i][j];
    }
  }
}

// Merge + activation. Each thread handles 4 consecutive outputs of one row;
// 8 consecutive lanes cover one 32-value Q8 block (N % 32 == 0).
__global__ void k_ffn_merge(FfnMergeArgs a) {
  const int64_t n4 = (int64_t)a.M * a.N / 4;
  const int64_t n4r = (n4 + 31) & ~(int64_t)31;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i4 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i4 < n4r; i4 += stride) {
    const bool in = i4 < n4;
    float4 s1 = make_float4(0.f, 0.f, 0.f, 0.f), s3 = s1;
    for (int s = 0; s < a.nseg; ++s) {
      float4 p = in ? reinterpret_cast<const float4*>(a.P1 + (size_t)s * a.seg_stride)[i4]
                    : make_float4(0.f, 0.f, 0.f, 0.f);
      if (a.quant) q8_roundtrip4(p);
      s1.x += p.x; s1.y += p.y; s1.z += p.z; s1.w += p.w;
      if (a.act == ACT_SWIGLU) {
        float4 q = in ? reinterpret_cast<const float4*>(a.P3 + (size_t)s * a.seg_stride)[i4]
                      : make_float4(0.f, 0.f, 0.f, 0.f);
        if (a.quant) q8_roundtrip4(q);
        s3.x += q.x; s3.y += q.y; s3.z += q.z; s3.w += q.w;
      }
    }
    if (!in) continue;
    float r[4] = {s1.x, s1.y, s1.z, s1.w};
    const float u[4] = {s3.x, s3.y, s3.z, s3.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (a.act == ACT_RELU) r[j] = fmaxf(r[j], 0.f);
      else if (a.act == ACT_SWIGLU) r[j] = r[j] / (1.0f + expf(-r[j])) * u[j];
    }
    if (a.residual) {
      const float4 x = reinterpret_cast<const float4*>(a.residual)[i4];
      r[0] += x.x; r[1] += x.y; r[2] += x.z; r[3] += x.w;
    }
    if (a.out_f32) reinterpret_cast<float4*>(a.out_f32)[i4] = make_float4(r[0], r[1], r[2], r[3]);
    if (a.out_bf16 && !a.bf16_split) {
      uint2 p;
      p.x = (uint32_t)f32_to_bf16_bits(r[0]) | ((uint32_t)f32_to_bf16_bits(r[1]) << 16);
      p.y = (uint32_t)f32_to_bf16_bits(r[2]) | ((uint32_t)f32_to_bf16_bits(r[3]) << 16);
      reinterpret_cast<uint2*>(a.out_bf16)[i4] = p;
    } else if (a.out_bf16) {
      const int64_t e = 4 * i4, m = e / a.N, n = e - m * a.N;
      uint16_t hi[4], lo[4];
      for (int j = 0; j < 4; ++j) bf16_split(r[j], hi[j], lo[j]);
      uint16_t* ph = a.out_bf16 + (size_t)(2 * m) * a.N + n;
      *reinterpret_cast<uint2*>(ph) =
          make_uint2((uint32_t)hi[0] | ((uint32_t)hi[1] << 16), (uint32_t)hi[2] | ((uint32_t)hi[3] << 16));
      *reinterpret_cast<uint2*>(ph + a.N) =
          make_uint2((uint32_t)lo[0] | ((uint32_t)lo[1] << 16), (uint32_t)lo[2] | ((uint32_t)lo[3] << 16));
    }
  }
}

}  // namespace

int launch_gemm_simt(int dtype, const void* A, int64_t lda, const void* B, int64_t ldb, float* P,
                     int M, int N, int Ks, int nseg, cudaStream_t s) {
  dim3 grid((N + TBN - 1) / TBN, (M + TBM - 1) / TBM, nseg);
  const int64_t seg_stride = (int64_t)M * N;
  if (dtype == TP_F32)
    k_gemm_simt<float><<<grid, 256, 0, s>>>(static_cast<const float*>(A), lda,
                                            static_cast<const float*>(B), ldb, P, M, N, Ks,
                                            seg_stride);
  else
    k_gemm_simt<uint16_t><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(A), lda,
                                               static_cast<const uint16_t*>(B), ldb, P, M, N, Ks,
                                               seg_stride);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

int launch_ffn_merge(const FfnMergeArgs& a, cudaStream_t s) {
  const int64_t n4 = (int64_t)a.M * a.N / 4;
  if (n4 == 0) return TP_OK;
  int64_t blocks = (n4 + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  k_ffn_merge<<<(unsigned)blocks, 256, 0, s>>>(a);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

}  // namespace tp
