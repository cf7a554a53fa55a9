// RMSNorm (+Q8 sync buffer), the cross-slice merge, and the standalone Q8 codec.
//
// distributed-llama issue #29 task list: llamaRmsAttNorm + llamaQuantizeRmsAtt
// (and the FFN twins llamaRmfFfnNorm + llamaQuantizeRmfFfn) become one kernel
// that writes the broadcast buffer every slice reads; llamaDequantizeAtt +
// llamaMergeAtt (and the Ffn2 twins) become one kernel that sums the slices'
// partials in slice order and adds them to the residual, optionally followed
// by the next sublayer's RMSNorm so that the merged row is normalised while it
// is still on chip.
#include "kernels.cuh"

namespace tp {

namespace {

constexpr int kNormThreads = 512;

// Normalise one row held in global memory (already final) and write the
// requested outputs. The loop runs over whole warps so that every 8-lane group
// maps to one 32-value quantisation block.
TP_DEV void norm_row_write(const float* xr, int dim, float rstd, const NormOut& no, int b,
                           float* red) {
  (void)red;
  const int n4 = dim >> 2;
  const int n4r = (n4 + 31) & ~31;
  const float4* g4 = reinterpret_cast<const float4*>(no.gain);
  for (int i4 = threadIdx.x; i4 < n4r; i4 += blockDim.x) {
    const bool in = i4 < n4;
    float4 v = in ? reinterpret_cast<const float4*>(xr)[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 g = in ? g4[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 y;
    y.x = __fmul_rn(__fmul_rn(v.x, rstd), g.x);
    y.y = __fmul_rn(__fmul_rn(v.y, rstd), g.y);
    y.z = __fmul_rn(__fmul_rn(v.z, rstd), g.z);
    y.w = __fmul_rn(__fmul_rn(v.w, rstd), g.w);
    const size_t e = (size_t)b * dim + 4 * (size_t)i4;
    if (no.quant) {
      float* sp = (in && no.xd) ? no.xd + e / kQ8Block : nullptr;
      float a = fmaxf(fmaxf(fabsf(y.x), fabsf(y.y)), fmaxf(fabsf(y.z), fabsf(y.w)));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
      const float d = q8_scale(a);
      if (sp && (threadIdx.x & 7) == 0) *sp = d;
      const int c0 = q8_code(y.x, d), c1 = q8_code(y.y, d), c2 = q8_code(y.z, d), c3 = q8_code(y.w, d);
      if (in) {
        if (no.xq) {
          const uint32_t packed = (uint32_t)(c0 & 0xFF) | ((uint32_t)(c1 & 0xFF) << 8) |
                                  ((uint32_t)(c2 & 0xFF) << 16) | ((uint32_t)(c3 & 0xFF) << 24);
          *reinterpret_cast<uint32_t*>(no.xq + e) = packed;
        }
        // consumers that read float32 / bf16 see the dequantised value
        y = make_float4(q8_value(c0, d), q8_value(c1, d), q8_value(c2, d), q8_value(c3, d));
      }
    }
    if (in) {
      if (no.xn) *reinterpret_cast<float4*>(no.xn + e) = y;
      if (no.xb) {
        uint2 p;
        p.x = (uint32_t)f32_to_bf16_bits(y.x) | ((uint32_t)f32_to_bf16_bits(y.y) << 16);
        p.y = (uint32_t)f32_to_bf16_bits(y.z) | ((uint32_t)f32_to_bf16_bits(y.w) << 16);
        *reinterpret_cast<uint2*>(no.xb + e) = p;
      }
    }
  }
}

__global__ void __launch_bounds__(kNormThreads) k_rmsnorm(const float* __restrict__ x, int dim,
                                                          NormOut no) {
  __shared__ float red[32];
  const int b = blockIdx.x;
  const float* xr = x + (size_t)b * dim;
  float ss = 0.f;
  for (int i4 = threadIdx.x; i4 < (dim >> 2); i4 += blockDim.x) {
    float4 v = reinterpret_cast<const float4*>(xr)[i4];
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = block_sum(ss, red);
  const float rstd = 1.0f / sqrtf(ss / (float)dim + no.eps);
  norm_row_write(xr, dim, rstd, no, b, red);
}

// x[b] += sum_{s=0}^{n-1} sync(part[s][b]) summed in slice order; then the
// optional RMSNorm of the new row.
__global__ void __launch_bounds__(kNormThreads) k_merge(float* __restrict__ x,
                                                        const float* __restrict__ part, int n,
                                                        int B, int dim, int quant, NormOut no) {
  __shared__ float red[32];
  const int b = blockIdx.x;
  float* xr = x + (size_t)b * dim;
  const int n4 = dim >> 2;
  const int n4r = (n4 + 31) & ~31;
  float ss = 0.f;
  for (int i4 = threadIdx.x; i4 < n4r; i4 += blockDim.x) {
    const bool in = i4 < n4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < n; ++s) {
      float4 p = in ? reinterpret_cast<const float4*>(part + ((size_t)s * B + b) * dim)[i4]
                    : make_float4(0.f, 0.f, 0.f, 0.f);
      if (quant) q8_roundtrip4(p);
      acc.x += p.x;
      acc.y += p.y;
      acc.z += p.z;
      acc.w += p.w;
    }
    if (in) {
      float4 v = reinterpret_cast<float4*>(xr)[i4];
      v.x += acc.x;
      v.y += acc.y;
      v.z += acc.z;
      v.w += acc.w;
      reinterpret_cast<float4*>(xr)[i4] = v;
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
  }
  if (no.gain == nullptr) return;
  ss = block_sum(ss, red);  // contains __syncthreads: the row writes above are visible
  const float rstd = 1.0f / sqrtf(ss / (float)dim + no.eps);
  norm_row_write(xr, dim, rstd, no, b, red);
}

__global__ void k_quantize(const float* __restrict__ x, int8_t* __restrict__ q,
                           float* __restrict__ d, int64_t n) {
  const int64_t n4 = n >> 2;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t n4r = (n4 + 31) & ~(int64_t)31;
  for (int64_t i4 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i4 < n4r; i4 += stride) {
    const bool in = i4 < n4;
    float4 v = in ? reinterpret_cast<const float4*>(x)[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
    const uint32_t codes = q8_quantize4(v, in ? d + (i4 >> 3) : nullptr);
    if (in) reinterpret_cast<uint32_t*>(q)[i4] = codes;
  }
}

__global__ void k_dequantize(const int8_t* __restrict__ q, const float* __restrict__ d,
                             float* __restrict__ x, int64_t n) {
  const int64_t n4 = n >> 2;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i4 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i4 < n4; i4 += stride) {
    const uint32_t c = reinterpret_cast<const uint32_t*>(q)[i4];
    reinterpret_cast<float4*>(x)[i4] = q8_unpack4(c, d[i4 >> 3]);
  }
}

}  // namespace

int launch_rmsnorm(const float* x, int B, int dim, const NormOut& no, cudaStream_t s) {
  k_rmsnorm<<<B, kNormThreads, 0, s>>>(x, dim, no);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

int launch_merge(float* x, const float* part, int n, int B, int dim, int quant, const NormOut& no,
                 cudaStream_t s) {
  k_merge<<<B, kNormThreads, 0, s>>>(x, part, n, B, dim, quant, no);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

int launch_quantize(const float* x, int8_t* q, float* d, int64_t n, cudaStream_t s) {
  if (n == 0) return TP_OK;
  const int threads = 256;
  int64_t blocks = ((n >> 2) + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  k_quantize<<<(unsigned)blocks, threads, 0, s>>>(x, q, d, n);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

int launch_dequantize(const int8_t* q, const float* d, float* x, int64_t n, cudaStream_t s) {
  if (n == 0) return TP_OK;
  const int threads = 256;
  int64_t blocks = ((n >> 2) + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  k_dequantize<<<(unsigned)blocks, threads, 0, s>>>(q, d, x, n);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

}  // namespace tp
