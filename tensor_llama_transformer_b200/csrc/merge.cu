// The cross-slice merge and the standalone Q8 codec.
//
// distributed-llama issue #29: llamaDequantizeAtt + llamaMergeAtt (and the Ffn2
// twins) sum the slices' partial outputs into the residual. Here one launch
// does both for every element: each partial (the sum of its contraction parts
// when a GEMM split it further) passes through the sync buffer's format (the Q8
// round trip when quantisation is on), the partials are summed
// in slice order 0..n-1 in float32, and the sum is added to x. One value per
// thread, one 128-value chunk of a row per CTA: the merge of a single token is
// spread over dim/128 SMs, and each thread's chain of dependent steps (loads,
// Q8 round trips, sum) is as short as it can be; a Q8 block is one warp.
#include "kernels.cuh"
#include "pipeline.cuh"

namespace tp {

namespace {

constexpr int kMergeThreads = 128;  // one value per thread: a CTA is one 128-value chunk

// The chunk's sum of squares from every thread's v*v: each warp's butterfly sum,
// then the four warps' sums in order, written by thread 0 (the same bits in both
// merge kernels, so the next RMSNorm sees the same scale either way).
TP_DEV void chunk_ssq(float v, float* ssq_out) {
  __shared__ float w[kMergeThreads / 32];
  const float sq = warp_sum(v * v);
  if ((threadIdx.x & 31) == 0) w[threadIdx.x >> 5] = sq;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = w[0];
#pragma unroll
    for (int i = 1; i < kMergeThreads / 32; ++i) t += w[i];
    *ssq_out = t;
  }
}

// CAP: at most 32 registers a thread (16 CTAs per SM), for grids too large to be resident
// in one wave at the uncapped count (40 registers, 12 CTAs per SM): the 2048 CTAs of a
// 70B-shaped batch-32 merge (dim 8192) took two waves and the step 12 us more; the capped
// form costs the 32-CTA single-token merge about 0.6 us (spilled state of the Q8 path).
template <bool CAP>
__global__ void __launch_bounds__(kMergeThreads, CAP ? 16 : 1) k_merge(float* __restrict__ x,
                                                      const float* __restrict__ part, int n,
                                                      int parts, int B, int dim, int quant,
                                                      float* __restrict__ ssq, MergeTrace tr,
                                                      int late) {
  if (!late) pdl_launch_dependents();
  unsigned long long* st =
      tr.stamps && threadIdx.x == 0 && (int)blockIdx.x < tr.rows ? tr.stamps + (size_t)blockIdx.x * tr.stride
                                                                 : nullptr;
  if (st) st[0] = gtimer();
  pdl_wait();
  if (st) st[1] = gtimer();
  // CTA = (batch row, 128-value chunk), grid (dim / 128) x B
  const int nch = dim >> 7;
  const int b = blockIdx.x / nch, ch = blockIdx.x - b * nch;
  const size_t i = (size_t)b * dim + (size_t)ch * kMergeThreads + threadIdx.x;
  const size_t stride = (size_t)B * dim;
  const float x0 = x[i];
  // slice s's partial: the sum of its contraction parts (planes s*parts .. s*parts+parts-1);
  // the loads of 4 slices at a time are issued together (L2 reads of partials other
  // CTAs just stored: one latency per 4 slices)
  float acc = 0.f;
  for (int s0 = 0; s0 < n; s0 += 4) {
    float p[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      p[j] = 0.f;
      for (int k = 0; k < parts && s0 + j < n; ++k)
        p[j] += __ldcg(part + (size_t)((s0 + j) * parts + k) * stride + i);
    }
    if (late && s0 == 0) {  // the next kernel launches once this CTA's partials are in
      const float dep = x0 + p[0] + p[1] + p[2] + p[3];
      asm volatile("" ::"f"(dep));
      pdl_launch_dependents();
    }
    if (quant) {  // each slice's value through the Q8 round trip of its block (a warp)
      if constexpr (CAP) {
#pragma unroll
        for (int h = 0; h < 4; h += 2) {  // two slices per branch (32 registers)
          float d[2];
#pragma unroll
          for (int j = 0; j < 2; ++j) d[j] = s0 + h + j < n ? q8_scale(warp_max(fabsf(p[h + j]))) : 1.f;
          q8_roundtrip_each<2>(p + h, d);
        }
      } else {  // the four slices' chains side by side
        float d[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) d[j] = s0 + j < n ? q8_scale(warp_max(fabsf(p[j]))) : 1.f;
        q8_roundtrip_each<4>(p, d);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (s0 + j < n) acc += p[j];
    }
  }
  const float v = x0 + acc;
  x[i] = v;
  if (ssq) chunk_ssq(v, ssq + (size_t)b * nch + ch);
  if (st) st[2] = gtimer();
}

__global__ void __launch_bounds__(kMergeThreads) k_sync_pack(const float* __restrict__ part,
                                                             int parts, int B, int dim, int quant,
                                                             uint8_t* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.y, s = blockIdx.z;
  const int i4 = blockIdx.x * kMergeThreads + threadIdx.x;
  const int n4 = dim >> 2;
  if (blockIdx.x * kMergeThreads + (threadIdx.x & ~31) >= n4) return;  // dim % 128: whole warps
  float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k = 0; k < parts; ++k) {
    const float4 v = reinterpret_cast<const float4*>(part + ((size_t)(s * parts + k) * B + b) * dim)[i4];
    p.x += v.x;
    p.y += v.y;
    p.z += v.z;
    p.w += v.w;
  }
  uint8_t* base = out + (size_t)s * sync_slice_bytes(B, dim, quant);
  if (quant) {
    float* scales = reinterpret_cast<float*>(base + (size_t)B * dim);
    const uint32_t codes = q8_quantize4(p, scales + ((size_t)b * dim + 4 * (size_t)i4) / kQ8Block);
    reinterpret_cast<uint32_t*>(base)[(size_t)b * n4 + i4] = codes;
  } else {
    reinterpret_cast<float4*>(base)[(size_t)b * n4 + i4] = p;
  }
}

// The receive side: x[b] += sum_{s<n} deq(slice s of the gathered buffer), in
// slice order, with the same chunk sums of squares as k_merge. Dequantising a
// packed slice gives the same bits as k_merge's in-place round trip, so a block
// whose slices are spread over ranks merges exactly as the whole block does.
__global__ void __launch_bounds__(kMergeThreads) k_merge_sync(float* __restrict__ x,
                                                              const uint8_t* __restrict__ sync,
                                                              int n, int B, int dim, int quant,
                                                              float* __restrict__ ssq) {
  pdl_launch_dependents();
  pdl_wait();
  const int nch = dim >> 7;
  const int b = blockIdx.x / nch, ch = blockIdx.x - b * nch;
  const size_t e = (size_t)b * dim + (size_t)ch * kMergeThreads + threadIdx.x;  // [B, dim] index
  const size_t bytes = (size_t)sync_slice_bytes(B, dim, quant);
  float acc = 0.f;
  for (int s = 0; s < n; ++s) {
    const uint8_t* base = sync + (size_t)s * bytes;
    float p;
    if (quant) {
      const float d = reinterpret_cast<const float*>(base + (size_t)B * dim)[e / kQ8Block];
      p = q8_value((int)reinterpret_cast<const int8_t*>(base)[e], d);
    } else {
      p = reinterpret_cast<const float*>(base)[e];
    }
    acc += p;
  }
  const float v = x[e] + acc;
  x[e] = v;
  if (ssq) chunk_ssq(v, ssq + (size_t)b * nch + ch);
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

// 512 values (4 warps of float4 lanes) per CTA of the sync pack
int merge_grid(int dim) { return (dim / 4 + kMergeThreads - 1) / kMergeThreads; }

int launch_merge(float* x, const float* part, int n, int B, int dim, int quant, float* ssq,
                 cudaStream_t s, int parts, MergeTrace trace, int late) {
  if (parts < 1 || parts > 2 || dim % 128 != 0) return TP_EINVAL;
  const int grid = (dim >> 7) * B;
  if (grid > 12 * num_sms())
    return launch_pdl(k_merge<true>, dim3(grid), dim3(kMergeThreads), 0, s, x, part, n, parts, B, dim,
                      quant, ssq, trace, late);
  return launch_pdl(k_merge<false>, dim3(grid), dim3(kMergeThreads), 0, s, x, part, n, parts, B, dim,
                    quant, ssq, trace, late);
}

int launch_sync_pack(const float* part, int n_local, int parts, int B, int dim, int quant,
                     uint8_t* out, cudaStream_t s) {
  const dim3 grid(merge_grid(dim), B, n_local);
  return launch_pdl(k_sync_pack, grid, dim3(kMergeThreads), 0, s, part, parts, B, dim, quant, out);
}

int launch_merge_sync(float* x, const uint8_t* sync, int n, int B, int dim, int quant, float* ssq,
                      cudaStream_t s) {
  if (dim % 128 != 0) return TP_EINVAL;
  return launch_pdl(k_merge_sync, dim3((dim >> 7) * B), dim3(kMergeThreads), 0, s, x, sync, n, B, dim,
                    quant, ssq);
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
