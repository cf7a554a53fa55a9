// The cross-slice merge and the standalone Q8 codec.
//
// distributed-llama issue #29: llamaDequantizeAtt + llamaMergeAtt (and the Ffn2
// twins) sum the slices' partial outputs into the residual. Here one launch
// does both for every element: each partial (the sum of its contraction parts
// when a GEMM split it further) passes through the sync buffer's format (the Q8
// round trip when quantisation is on), the partials are summed
// in slice order 0..n-1 in float32, and the sum is added to x. The grid covers
// the batch rows in 512-element pieces so that the merge of a single token is
// spread over many SMs instead of waiting on one.
#include "kernels.cuh"

namespace tp {

namespace {

constexpr int kMergeThreads = 128;  // 4 values per thread: 512 values per CTA

__global__ void __launch_bounds__(kMergeThreads) k_merge(float* __restrict__ x,
                                                      const float* __restrict__ part, int n,
                                                      int parts, int B, int dim, int quant,
                                                      float* __restrict__ ssq) {
  pdl_launch_dependents();
  pdl_wait();
  // CTA = (batch row, 512-value piece)
  const int pieces = (dim / 4 + kMergeThreads - 1) / kMergeThreads;
  const int b = blockIdx.x / pieces, piece = blockIdx.x - b * pieces;
  const int i4 = piece * kMergeThreads + threadIdx.x;  // float4 index within the row
  const int n4 = dim >> 2;
  if (piece * kMergeThreads + (threadIdx.x & ~31) >= n4) return;  // dim % 128: whole warps
  // slice s's partial: the sum of its contraction parts (planes s*parts .. s*parts+parts-1)
  float4* xr = reinterpret_cast<float4*>(x + (size_t)b * dim) + i4;
  const float4 v = merge_lane4(part, (size_t)B * dim, (size_t)b * dim + 4 * (size_t)i4, n, parts,
                               quant, *xr);
  *xr = v;
  float sq = v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  if (ssq) {  // each warp's 128 values: their sum of squares, for the next RMSNorm
    sq = warp_sum(sq);
    const int chunk = (piece * kMergeThreads + (threadIdx.x & ~31)) >> 5;
    if ((threadIdx.x & 31) == 0 && chunk < (dim >> 7)) ssq[(size_t)b * (dim >> 7) + chunk] = sq;
  }
}

// Sync-buffer pack for a rank that holds slices of the block (the send side of
// distributed-llama's SyncAtt / SyncFfn2): slice s's partial, the sum of its
// contraction parts, written in the slice's sync format -- float32 [B, dim], or
// with Q8 the codes int8 [B, dim] followed by the scales float32 [B, dim/32].
// Grid (pieces of 512 values, B, local slices).
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
// slice order, with the same per-piece sums of squares as k_merge. Dequantising a
// packed slice gives the same bits as k_merge's in-place round trip, so a block
// whose slices are spread over ranks merges exactly as the whole block does.
__global__ void __launch_bounds__(kMergeThreads) k_merge_sync(float* __restrict__ x,
                                                              const uint8_t* __restrict__ sync,
                                                              int n, int B, int dim, int quant,
                                                              float* __restrict__ ssq) {
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.y;
  const int i4 = blockIdx.x * kMergeThreads + threadIdx.x;
  const int n4 = dim >> 2;
  const bool in = i4 < n4;
  const size_t chunk = (size_t)sync_slice_bytes(B, dim, quant);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < n && in; ++s) {
    const uint8_t* base = sync + (size_t)s * chunk;
    float4 p;
    if (quant) {
      const float d = reinterpret_cast<const float*>(base + (size_t)B * dim)[((size_t)b * dim + 4 * (size_t)i4) / kQ8Block];
      p = q8_unpack4(reinterpret_cast<const uint32_t*>(base)[(size_t)b * n4 + i4], d);
    } else {
      p = reinterpret_cast<const float4*>(base)[(size_t)b * n4 + i4];
    }
    acc.x += p.x;
    acc.y += p.y;
    acc.z += p.z;
    acc.w += p.w;
  }
  float sq = 0.f;
  if (in) {
    float4* xr = reinterpret_cast<float4*>(x + (size_t)b * dim);
    float4 v = xr[i4];
    v.x += acc.x;
    v.y += acc.y;
    v.z += acc.z;
    v.w += acc.w;
    xr[i4] = v;
    sq = v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  if (ssq) {  // as k_merge: one sum of squares per warp's 128 values
    sq = warp_sum(sq);
    const int chunk = (blockIdx.x * kMergeThreads + (threadIdx.x & ~31)) >> 5;
    if ((threadIdx.x & 31) == 0 && chunk < (dim >> 7)) ssq[(size_t)b * (dim >> 7) + chunk] = sq;
  }
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

// 512 values (4 warps of float4 lanes) per CTA
int merge_grid(int dim) { return (dim / 4 + kMergeThreads - 1) / kMergeThreads; }

int launch_merge(float* x, const float* part, int n, int B, int dim, int quant, float* ssq,
                 cudaStream_t s, int parts) {
  if (parts < 1 || parts > 2 || dim % 128 != 0) return TP_EINVAL;
  return launch_pdl(k_merge, dim3(merge_grid(dim) * B), dim3(kMergeThreads), 0, s, x, part, n, parts,
                    B, dim, quant, ssq);
}

int launch_sync_pack(const float* part, int n_local, int parts, int B, int dim, int quant,
                     uint8_t* out, cudaStream_t s) {
  const dim3 grid(merge_grid(dim), B, n_local);
  return launch_pdl(k_sync_pack, grid, dim3(kMergeThreads), 0, s, part, parts, B, dim, quant, out);
}

int launch_merge_sync(float* x, const uint8_t* sync, int n, int B, int dim, int quant, float* ssq,
                      cudaStream_t s) {
  const dim3 grid(merge_grid(dim), B);
  return launch_pdl(k_merge_sync, grid, dim3(kMergeThreads), 0, s, x, sync, n, B, dim, quant, ssq);
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
