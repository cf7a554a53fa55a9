// Weight-streaming slice GEMV for decode (small batch).
//
//   out[seg, b, r] = sum_{k < Ks} W[r, seg*Ks + k] * x[b, seg*Ks + k]
//
// One kernel covers every slice product of the distributed-llama task list:
//   - column split (llamaQkv, llamaFfn, llamaLogits): nseg = 1, the slices are
//     contiguous row ranges and the launch covers all of them at once;
//   - row split (llamaAttOutput, llamaFfn2): nseg = n, slice s reads its column
//     range of every row and writes its own partial [B, dim] of the
//     all-reduce (aiterms.tw "Tensor Parallelism": Linear2 split by rows needs a
//     reduction).
// The kernel is bound by the weight stream: each bf16 weight is read once with
// a 16-byte non-allocating load, multiplied with float32 activations staged
// in shared memory, and reduced across the warp with shuffles. CTAs own
// contiguous, equal shares of the rows of one segment so that every SM streams
// the same number of bytes.
//
// Epilogues: EPI_PLAIN stores (partials, logits); EPI_SWIGLU reads row f of W1
// and W3 together and stores silu(a)*b (llamaFfn); EPI_QKV applies RoPE to the
// q and k row pairs, stores rotated q, and writes k and v into the bf16 cache at
// pos (llamaMultiheadAtt's "merge kv-cache, add RoPE encoding").
#include "kernels.cuh"

namespace tp {

namespace {

constexpr int kGemvThreads = 256;
constexpr int kUnroll = 4;  // 16-byte vectors in flight per lane per row

TP_DEV float dot8(const uint4 w, const float4 lo, const float4 hi) {
  float a = bf16lo(w.x) * lo.x;
  a = fmaf(bf16hi(w.x), lo.y, a);
  a = fmaf(bf16lo(w.y), lo.z, a);
  a = fmaf(bf16hi(w.y), lo.w, a);
  a = fmaf(bf16lo(w.z), hi.x, a);
  a = fmaf(bf16hi(w.z), hi.y, a);
  a = fmaf(bf16lo(w.w), hi.z, a);
  a = fmaf(bf16hi(w.w), hi.w, a);
  return a;
}

// Shared-memory activation layout: for batch row b and 16-byte weight vector v
// (elements 8v..8v+7), lo[b][v] holds elements 8v..8v+3 and hi[b][v] 8v+4..8v+7,
// so a warp reading consecutive v touches consecutive float4s (no bank conflict).
template <int NB>
TP_DEV void stage_x(const GemvArgs& a, int seg, float4* lo, float4* hi, int nv) {
  for (int i = threadIdx.x; i < NB * nv; i += blockDim.x) {
    const int b = i / nv, v = i - b * nv;
    float4 l = make_float4(0.f, 0.f, 0.f, 0.f), h = l;
    if (b < a.nb) {
      const int gb = a.b0 + b;
      const size_t e = (size_t)gb * a.ldx + (size_t)seg * a.Ks + 8 * (size_t)v;
      if (a.xq) {
        const uint2 c = *reinterpret_cast<const uint2*>(a.xq + e);
        const float d = a.xd[e / kQ8Block];
        l = q8_unpack4(c.x, d);
        h = q8_unpack4(c.y, d);
      } else {
        l = *reinterpret_cast<const float4*>(a.x + e);
        h = *reinterpret_cast<const float4*>(a.x + e + 4);
      }
    }
    lo[b * nv + v] = l;
    hi[b * nv + v] = h;
  }
}

// Rows (row pointers r0, r1) dotted with the staged activations; returns the
// warp-reduced sums in acc (valid in every lane).
template <int NB>
TP_DEV void dot_rows2(const uint16_t* __restrict__ r0, const uint16_t* __restrict__ r1,
                      const float4* lo, const float4* hi, int nv, float (&acc)[2][NB]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int b = 0; b < NB; ++b) acc[0][b] = acc[1][b] = 0.f;
  for (int v0 = lane; v0 < nv; v0 += 32 * kUnroll) {
    uint4 w0[kUnroll], w1[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
        w0[u] = ld_stream16(r0 + 8 * (size_t)v);
        w1[u] = ld_stream16(r1 + 8 * (size_t)v);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float4 l = lo[b * nv + v], h = hi[b * nv + v];
          acc[0][b] += dot8(w0[u], l, h);
          acc[1][b] += dot8(w1[u], l, h);
        }
      }
    }
  }
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    acc[0][b] = warp_sum(acc[0][b]);
    acc[1][b] = warp_sum(acc[1][b]);
  }
}

template <int NB, int EPI>
__global__ void __launch_bounds__(kGemvThreads) k_gemv(GemvArgs a) {
  extern __shared__ float4 smem_x[];
  const int seg = blockIdx.x / a.ctas_per_seg;
  const int cta = blockIdx.x - seg * a.ctas_per_seg;
  const int nv = a.Ks >> 3;
  float4* lo = smem_x;
  float4* hi = smem_x + NB * nv;
  stage_x<NB>(a, seg, lo, hi, nv);
  __syncthreads();

  // virtual rows of this segment, processed as pairs
  int vrows = a.rows[0];
  if (EPI == EPI_QKV) vrows += a.rows[1] + a.rows[2];
  const int npairs = EPI == EPI_SWIGLU ? vrows : vrows >> 1;
  const int p_begin = (int)(((int64_t)npairs * cta) / a.ctas_per_seg);
  const int p_end = (int)(((int64_t)npairs * (cta + 1)) / a.ctas_per_seg);
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5, lane = threadIdx.x & 31;
  const size_t col0 = (size_t)seg * a.Ks;

  for (int p = p_begin + warp; p < p_end; p += nwarps) {
    const uint16_t *r0, *r1;
    int mat = 0, lrow = 0;
    if (EPI == EPI_SWIGLU) {
      r0 = a.w[0] + (size_t)p * a.ldw + col0;
      r1 = a.w[1] + (size_t)p * a.ldw + col0;
      lrow = p;
    } else {
      int row = 2 * p;
      if (EPI == EPI_QKV) {
        if (row >= a.rows[0]) {
          row -= a.rows[0];
          mat = 1;
          if (row >= a.rows[1]) {
            row -= a.rows[1];
            mat = 2;
          }
        }
      }
      lrow = row;
      r0 = a.w[mat] + (size_t)row * a.ldw + col0;
      r1 = r0 + a.ldw;
    }
    float acc[2][NB];
    dot_rows2<NB>(r0, r1, lo, hi, nv, acc);

    if (EPI == EPI_PLAIN) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (lane == b && b < a.nb) {
          const size_t o = (size_t)seg * a.out_seg + (size_t)(a.b0 + b) * a.ldo + lrow;
          a.out[o] = acc[0][b];
          a.out[o + 1] = acc[1][b];
          if (a.out_bf16) {
            a.out_bf16[o] = f32_to_bf16_bits(acc[0][b]);
            a.out_bf16[o + 1] = f32_to_bf16_bits(acc[1][b]);
          }
        }
      }
    } else if (EPI == EPI_SWIGLU) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (lane == b && b < a.nb) {
          const float g = acc[0][b], u = acc[1][b];
          const float h = g / (1.0f + expf(-g)) * u;
          const size_t o = (size_t)(a.b0 + b) * a.ldo + lrow;
          a.out[o] = h;
          if (a.out_bf16) a.out_bf16[o] = f32_to_bf16_bits(h);
        }
      }
    } else {  // EPI_QKV
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (lane == b && b < a.nb) {
          const int gb = a.b0 + b;
          const int pos = a.pos[gb];
          const int d = lrow % kHeadDim;  // even: first element of the RoPE pair
          const int head = lrow / kHeadDim;
          float y0 = acc[0][b], y1 = acc[1][b];
          if (mat < 2) {
            const float freq = powf(a.theta, -(float)d / (float)kHeadDim);
            float sn, cs;
            sincosf((float)pos * freq, &sn, &cs);
            const float r0v = y0 * cs - y1 * sn;
            const float r1v = y0 * sn + y1 * cs;
            y0 = r0v;
            y1 = r1v;
          }
          if (mat == 0) {
            float* qo = a.qout + (size_t)gb * a.n_heads * kHeadDim + lrow;
            qo[0] = y0;
            qo[1] = y1;
          } else {
            uint16_t* cache = mat == 1 ? a.kc : a.vc;
            const size_t o =
                (((size_t)gb * a.n_kv_heads + head) * a.max_seq + pos) * kHeadDim + d;
            const uint32_t pair = (uint32_t)f32_to_bf16_bits(y0) | ((uint32_t)f32_to_bf16_bits(y1) << 16);
            *reinterpret_cast<uint32_t*>(cache + o) = pair;
          }
        }
      }
    }
  }
}

template <int NB>
int launch_nb(const GemvArgs& a, int epi, cudaStream_t s) {
  const int nv = a.Ks >> 3;
  const size_t smem = (size_t)2 * NB * nv * sizeof(float4);
  const dim3 grid(a.ctas_per_seg * a.nseg);
  switch (epi) {
    case EPI_PLAIN:
      if (smem > 48 * 1024 && set_smem_once((const void*)k_gemv<NB, EPI_PLAIN>, (int)smem)) return TP_ECUDA;
      k_gemv<NB, EPI_PLAIN><<<grid, kGemvThreads, smem, s>>>(a);
      break;
    case EPI_SWIGLU:
      if (smem > 48 * 1024 && set_smem_once((const void*)k_gemv<NB, EPI_SWIGLU>, (int)smem)) return TP_ECUDA;
      k_gemv<NB, EPI_SWIGLU><<<grid, kGemvThreads, smem, s>>>(a);
      break;
    default:
      if (smem > 48 * 1024 && set_smem_once((const void*)k_gemv<NB, EPI_QKV>, (int)smem)) return TP_ECUDA;
      k_gemv<NB, EPI_QKV><<<grid, kGemvThreads, smem, s>>>(a);
      break;
  }
  TP_LAUNCH_CHECK();
  return TP_OK;
}

}  // namespace

// Batch rows are processed in groups of at most 4 per launch (the activations of
// a group are staged in shared memory: 4 x Ks x 4 bytes).
int launch_gemv(const GemvArgs& a0, int epi, cudaStream_t s) {
  int total = a0.nb;
  for (int b = 0; b < total;) {
    GemvArgs a = a0;
    a.b0 = a0.b0 + b;
    int nb = total - b;
    int maxnb = (a.Ks <= 4096) ? 4 : 2;
    if (nb > maxnb) nb = maxnb;
    a.nb = nb;
    int rc;
    if (nb == 1)
      rc = launch_nb<1>(a, epi, s);
    else if (nb == 2)
      rc = launch_nb<2>(a, epi, s);
    else
      rc = launch_nb<4>(a, epi, s);
    if (rc != TP_OK) return rc;
    b += nb;
  }
  return TP_OK;
}

}  // namespace tp
