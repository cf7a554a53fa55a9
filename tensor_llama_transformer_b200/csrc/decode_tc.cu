// Helper kernel of the batched decode path (batch >= kTcMinBatch), where the
// slice products run on the tcgen05 GEMM with the weights as the M operand and
// the batch as N, each writing float32 partial planes [part, batch, rows]:
//   k_norm_rows     RMSNorm(+Q8) of the residual rows -> the shared input (the
//                   SyncRmsAtt / SyncRmfFfn buffer) and its hi/lo bf16 pair, the
//                   tensor-core operand.
//   k_qkv_finalize  sums the contraction parts of the q/k/v plane, applies RoPE
//                   to q and k pairs, stores q and writes k/v into the cache at pos
//                   (distributed-llama llamaQkv + llamaMultiheadAtt's cache merge);
//   k_swiglu_finalize  silu(W1 row) * W3 row from the W1/W3 plane (llamaFfn).
// The same steps (and the merges) can run instead in the GEMM's epilogue
// (gemm_tc.cu, TcFinish).
#include "kernels.cuh"

namespace tp {
namespace {

constexpr int kRowThreads = 256;

__global__ void __launch_bounds__(kRowThreads) k_norm_rows(NormRowsArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float red[32];
  __shared__ float s_rstd;
  const int b = blockIdx.x;
  const float* xr = a.x + (size_t)b * a.dim;
  if (threadIdx.x == 0 && a.ssq) {
    float t = 0.f;
    for (int c = 0; c < a.ssq_parts; ++c) t += a.ssq[(size_t)b * a.ssq_parts + c];
    s_rstd = 1.0f / sqrtf(t / (float)a.dim + a.eps);
  }
  if (!a.ssq) {
    float ss = 0.f;
    for (int i = threadIdx.x; i < (a.dim >> 2); i += kRowThreads) {
      const float4 v = reinterpret_cast<const float4*>(xr)[i];
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = block_sum(ss, red);
    if (threadIdx.x == 0) s_rstd = 1.0f / sqrtf(ss / (float)a.dim + a.eps);
  }
  __syncthreads();
  const float rstd = s_rstd;
  const int n4 = a.dim >> 2, n4r = (n4 + 31) & ~31;  // whole warps: 8 lanes = one Q8 block
  for (int i4 = threadIdx.x; i4 < n4r; i4 += kRowThreads) {
    const bool in = i4 < n4;
    float4 v = in ? reinterpret_cast<const float4*>(xr)[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 g = in ? reinterpret_cast<const float4*>(a.gain)[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 y = make_float4(__fmul_rn(__fmul_rn(v.x, rstd), g.x), __fmul_rn(__fmul_rn(v.y, rstd), g.y),
                           __fmul_rn(__fmul_rn(v.z, rstd), g.z), __fmul_rn(__fmul_rn(v.w, rstd), g.w));
    const size_t e = (size_t)b * a.dim + 4 * (size_t)i4;
    if (in && a.xn) *reinterpret_cast<float4*>(a.xn + e) = y;  // before any Q8 round trip
    if (a.quant) {
      float am = fmaxf(fmaxf(fabsf(y.x), fabsf(y.y)), fmaxf(fabsf(y.z), fabsf(y.w)));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
      const float d = q8_scale(am);
      const float yv[4] = {y.x, y.y, y.z, y.w};
      float cf[4];
      q8_codes<4>(yv, cf, d, q8_recip(d));
      const int c0 = (int)cf[0], c1 = (int)cf[1], c2 = (int)cf[2], c3 = (int)cf[3];
      if (in) {
        if (a.xq)
          *reinterpret_cast<uint32_t*>(a.xq + e) = (uint32_t)(c0 & 0xFF) | ((uint32_t)(c1 & 0xFF) << 8) |
                                                   ((uint32_t)(c2 & 0xFF) << 16) | ((uint32_t)(c3 & 0xFF) << 24);
        if (a.xd && (threadIdx.x & 7) == 0) a.xd[e / kQ8Block] = d;
      }
      y = make_float4(q8_value(c0, d), q8_value(c1, d), q8_value(c2, d), q8_value(c3, d));
    }
    if (in) {
      uint16_t h[4], l[4];
      bf16_split(y.x, h[0], l[0]);
      bf16_split(y.y, h[1], l[1]);
      bf16_split(y.z, h[2], l[2]);
      bf16_split(y.w, h[3], l[3]);
      const size_t eh = (size_t)(2 * b) * a.dim + 4 * (size_t)i4;  // row 2b: hi, row 2b+1: lo
      *reinterpret_cast<uint2*>(a.xb + eh) =
          make_uint2((uint32_t)h[0] | ((uint32_t)h[1] << 16), (uint32_t)h[2] | ((uint32_t)h[3] << 16));
      *reinterpret_cast<uint2*>(a.xb + eh + a.dim) =
          make_uint2((uint32_t)l[0] | ((uint32_t)l[1] << 16), (uint32_t)l[2] | ((uint32_t)l[3] << 16));
    }
  }
}

// One thread per row pair of the concatenated [q | k | v] rows of one batch row.
__global__ void k_qkv_finalize(QkvFinalizeArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.y;
  const int pr = blockIdx.x * blockDim.x + threadIdx.x;
  const int R = a.qd + 2 * a.kd;
  if (2 * pr >= R) return;
  const int row = 2 * pr;
  float y0 = 0.f, y1 = 0.f;
  for (int p = 0; p < a.parts; ++p) {  // contraction parts in order
    const float2 v = *reinterpret_cast<const float2*>(a.plane + ((size_t)p * a.batch + b) * R + row);
    y0 += v.x;
    y1 += v.y;
  }
  int mat = 0, lrow = row;
  if (lrow >= a.qd) {
    lrow -= a.qd;
    mat = 1;
    if (lrow >= a.kd) {
      lrow -= a.kd;
      mat = 2;
    }
  }
  const int pos = a.pos[b];
  const int d = lrow % kHeadDim;  // even: first element of the RoPE pair
  const int head = lrow / kHeadDim;
  if (mat < 2) {
    const float freq = powf(a.theta, -(float)d / (float)kHeadDim);
    float sn, cs;
    sincosf((float)pos * freq, &sn, &cs);
    const float r0 = y0 * cs - y1 * sn;
    const float r1 = y0 * sn + y1 * cs;
    y0 = r0;
    y1 = r1;
  }
  if (mat == 0) {
    *reinterpret_cast<float2*>(a.q + (size_t)b * a.qd + lrow) = make_float2(y0, y1);
  } else {
    uint16_t* cache = mat == 1 ? a.kc : a.vc;
    const size_t sq = a.seq ? (size_t)a.seq[b] : (size_t)b;
    const size_t o = ((sq * a.n_kv_heads + head) * a.max_seq + pos) * kHeadDim + d;
    *reinterpret_cast<uint32_t*>(cache + o) =
        (uint32_t)f32_to_bf16_bits(y0) | ((uint32_t)f32_to_bf16_bits(y1) << 16);
  }
}

// planes [parts][batch][2F]: columns [0, F) are x W1^T, [F, 2F) are x W3^T, each
// summed over the contraction parts in order.
__global__ void k_swiglu_finalize(const float* __restrict__ plane, int parts, int F, int batch,
                                  float* __restrict__ h, uint16_t* __restrict__ hb) {
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.y;
  const int f = blockIdx.x * blockDim.x + threadIdx.x;
  if (f >= F) return;
  float a = 0.f, g = 0.f;
  for (int p = 0; p < parts; ++p) {
    const float* pl = plane + ((size_t)p * batch + b) * 2 * F;
    a += pl[f];
    g += pl[F + f];
  }
  const float v = a / (1.0f + expf(-a)) * g;
  h[(size_t)b * F + f] = v;
  bf16_split(v, hb[(size_t)(2 * b) * F + f], hb[(size_t)(2 * b + 1) * F + f]);
}

}  // namespace

int launch_norm_rows(const NormRowsArgs& a, int batch, cudaStream_t s) {
  if (a.dim % 128 != 0) return TP_EINVAL;
  return launch_pdl(k_norm_rows, dim3(batch), dim3(kRowThreads), 0, s, a);
}

int launch_qkv_finalize(const QkvFinalizeArgs& a, cudaStream_t s) {
  const int pairs = (a.qd + 2 * a.kd) / 2;
  return launch_pdl(k_qkv_finalize, dim3((pairs + 255) / 256, a.batch), dim3(256), 0, s, a);
}

int launch_swiglu_finalize(const float* plane, int parts, int F, int batch, float* h,
                           uint16_t* hb, cudaStream_t s) {
  return launch_pdl(k_swiglu_finalize, dim3((F + 255) / 256, batch), dim3(256), 0, s, plane, parts,
                    F, batch, h, hb);
}

}  // namespace tp
