// Weight-streaming slice GEMV for decode (small batch).
//
//   out[seg, b, r] = sum_{k < Ks} W[r, seg*Ks + k] * x[b, seg*Ks + k]
//
// One kernel covers every slice product of the distributed-llama task list:
//   - column split (llamaQkv, llamaFfn, llamaLogits): nseg = 1, the slices are
//     contiguous row ranges and one launch covers all of them;
//   - row split (llamaAttOutput, llamaFfn2): nseg = n, slice s reads its column
//     range of every row and writes its own partial [B, rows] of the all-reduce
//     (aiterms.tw "Tensor Parallelism": Linear2 split by rows needs a reduction).
//
// Work split. The kernel is bound by the weight stream, so every SM must stream
// the same bytes until the end. Rows are handled in pairs (a RoPE pair of q/k,
// row f of W1 with row f of W3, or two consecutive rows) and each CTA owns a
// contiguous, equal share of the pairs of one segment. Inside a CTA the 8
// warps split the contraction of every pair: warp w streams the same column
// range of each row, 16 bytes per lane per load, with the activations of that
// range held in registers. Each warp reduces its partial dot products with
// shuffles and leaves them in shared memory; after the last pair the CTA adds
// the 8 warps' partials in a fixed order and runs the epilogue.
//
// Input modes: float32 activations; Q8 codes + scales (dequantised on load);
// or the RMSNorm of a float32 residual computed in the prologue (each CTA
// reduces the whole row for the scale, then normalises, and with Q8 quantises,
// only its warps' column ranges; the first CTA of each segment also writes the
// normalised / quantised buffer that the slices share).
//
// Epilogues: EPI_PLAIN stores (partials, logits); EPI_SWIGLU stores silu(a)*b
// (llamaFfn); EPI_QKV applies RoPE to q and k row pairs, stores rotated q, and
// writes k and v into the bf16 cache at pos (llamaMultiheadAtt's "merge kv-cache,
// add RoPE encoding").
#include "kernels.cuh"

namespace tp {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

TP_DEV float dot8(const uint4 w, const float* x) {
  float a = bf16lo(w.x) * x[0];
  a = fmaf(bf16hi(w.x), x[1], a);
  a = fmaf(bf16lo(w.y), x[2], a);
  a = fmaf(bf16hi(w.y), x[3], a);
  a = fmaf(bf16lo(w.z), x[4], a);
  a = fmaf(bf16hi(w.z), x[5], a);
  a = fmaf(bf16lo(w.w), x[6], a);
  a = fmaf(bf16hi(w.w), x[7], a);
  return a;
}

// The warp's column range, in 16-byte vectors, aligned to 4-vector groups so
// that a 32-value quantisation block never straddles two warps.
TP_DEV void warp_range(int nv, int w, int& vb, int& ve) {
  const int ng = nv >> 2;
  vb = ((ng * w) / kWarps) * 4;
  ve = ((ng * (w + 1)) / kWarps) * 4;
}

// Row pointers of pair p of the segment (see GemvArgs): r0 and r1.
template <int EPI>
TP_DEV void pair_rows(const GemvArgs& a, int p, size_t col0, const uint16_t*& r0,
                      const uint16_t*& r1, int& mat, int& lrow) {
  mat = 0;
  if (EPI == EPI_SWIGLU) {
    r0 = a.w[0] + (size_t)p * a.ldw + col0;
    r1 = a.w[1] + (size_t)p * a.ldw + col0;
    lrow = p;
  } else {
    int row = 2 * p;
    if (EPI == EPI_QKV && row >= a.rows[0]) {
      row -= a.rows[0];
      mat = 1;
      if (row >= a.rows[1]) {
        row -= a.rows[1];
        mat = 2;
      }
    }
    lrow = row;
    r0 = a.w[mat] + (size_t)row * a.ldw + col0;
    r1 = r0 + a.ldw;
  }
}

template <int NB, int EPI, int VPL>
__global__ void __launch_bounds__(kThreads) k_gemv(GemvArgs a) {
  constexpr int U = VPL == 1 ? 4 : (VPL == 2 ? 2 : 1);  // pairs in flight per warp
  extern __shared__ float red[];                        // [pairs][kWarps][2][NB]
  __shared__ float s_rstd[NB];
  const int seg = blockIdx.x / a.ctas_per_seg;
  const int cta = blockIdx.x - seg * a.ctas_per_seg;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = a.Ks >> 3;
  int vb, ve;
  warp_range(nv, warp, vb, ve);
  const size_t col0 = (size_t)seg * a.Ks;

  // ---------------------------------------------------------------- activations
  float xr[NB][VPL][8];
  if (a.gain) {  // RMSNorm of the residual rows (+Q8)
    const int D = a.ldx;
    float ss[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      ss[b] = 0.f;
      if (b < a.nb) {
        const float4* xrow = reinterpret_cast<const float4*>(a.x + (size_t)(a.b0 + b) * D);
        for (int i = threadIdx.x; i < (D >> 2); i += kThreads) {
          const float4 v = xrow[i];
          ss[b] += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
        }
      }
      ss[b] = warp_sum(ss[b]);
    }
    if (lane == 0)
#pragma unroll
      for (int b = 0; b < NB; ++b) red[warp * NB + b] = ss[b];
    __syncthreads();
    if (threadIdx.x < NB) {
      float t = 0.f;
      for (int w = 0; w < kWarps; ++w) t += red[w * NB + threadIdx.x];
      s_rstd[threadIdx.x] = 1.0f / sqrtf(t / (float)D + a.eps);
    }
    __syncthreads();
  }
  const bool writer = cta == 0;  // first CTA of the segment publishes the shared buffer
#pragma unroll
  for (int b = 0; b < NB; ++b) {
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int v = vb + lane + 32 * j;
      float* xv = xr[b][j];
#pragma unroll
      for (int e = 0; e < 8; ++e) xv[e] = 0.f;
      const bool in = b < a.nb && v < ve;
      const size_t e0 = (size_t)(a.b0 + b) * a.ldx + col0 + 8 * (size_t)v;
      if (a.gain) {
        if (in) {
          const float rstd = s_rstd[b];
          const float4 x0 = *reinterpret_cast<const float4*>(a.x + e0);
          const float4 x1 = *reinterpret_cast<const float4*>(a.x + e0 + 4);
          const float4 g0 = *reinterpret_cast<const float4*>(a.gain + col0 + 8 * (size_t)v);
          const float4 g1 = *reinterpret_cast<const float4*>(a.gain + col0 + 8 * (size_t)v + 4);
          xv[0] = __fmul_rn(__fmul_rn(x0.x, rstd), g0.x);
          xv[1] = __fmul_rn(__fmul_rn(x0.y, rstd), g0.y);
          xv[2] = __fmul_rn(__fmul_rn(x0.z, rstd), g0.z);
          xv[3] = __fmul_rn(__fmul_rn(x0.w, rstd), g0.w);
          xv[4] = __fmul_rn(__fmul_rn(x1.x, rstd), g1.x);
          xv[5] = __fmul_rn(__fmul_rn(x1.y, rstd), g1.y);
          xv[6] = __fmul_rn(__fmul_rn(x1.z, rstd), g1.z);
          xv[7] = __fmul_rn(__fmul_rn(x1.w, rstd), g1.w);
        }
        if (a.quant) {  // Q8 of 32-value blocks = 4 consecutive lanes (warp-uniform branch)
          float am = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(xv[e]));
          am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
          am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
          const float d = q8_scale(am);
          uint32_t lo = 0, hi = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int c = q8_code(xv[e], d);
            xv[e] = q8_value(c, d);
            if (e < 4) lo |= (uint32_t)(c & 0xFF) << (8 * e);
            else hi |= (uint32_t)(c & 0xFF) << (8 * (e - 4));
          }
          if (writer && in && a.xq_out) {
            *reinterpret_cast<uint2*>(a.xq_out + e0) = make_uint2(lo, hi);
            if ((lane & 3) == 0) a.xd_out[e0 / kQ8Block] = d;
          }
        }
        if (writer && in && a.xn_out) {
          *reinterpret_cast<float4*>(a.xn_out + e0) = make_float4(xv[0], xv[1], xv[2], xv[3]);
          *reinterpret_cast<float4*>(a.xn_out + e0 + 4) = make_float4(xv[4], xv[5], xv[6], xv[7]);
        }
      } else if (in) {
        if (a.xq) {
          const uint2 c = *reinterpret_cast<const uint2*>(a.xq + e0);
          const float d = a.xd[e0 / kQ8Block];
          const float4 l = q8_unpack4(c.x, d), h = q8_unpack4(c.y, d);
          xv[0] = l.x; xv[1] = l.y; xv[2] = l.z; xv[3] = l.w;
          xv[4] = h.x; xv[5] = h.y; xv[6] = h.z; xv[7] = h.w;
        } else {
          const float4 l = *reinterpret_cast<const float4*>(a.x + e0);
          const float4 h = *reinterpret_cast<const float4*>(a.x + e0 + 4);
          xv[0] = l.x; xv[1] = l.y; xv[2] = l.z; xv[3] = l.w;
          xv[4] = h.x; xv[5] = h.y; xv[6] = h.z; xv[7] = h.w;
        }
      }
    }
  }

  // ---------------------------------------------------------------- weight stream
  int vrows = a.rows[0];
  if (EPI == EPI_QKV) vrows += a.rows[1] + a.rows[2];
  const int npairs = EPI == EPI_SWIGLU ? vrows : vrows >> 1;
  const int p0 = (int)(((int64_t)npairs * cta) / a.ctas_per_seg);
  const int p1 = (int)(((int64_t)npairs * (cta + 1)) / a.ctas_per_seg);

  for (int pb = p0; pb < p1; pb += U) {
    uint4 wv[U][2][VPL];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int p = pb + u;
      if (p < p1) {
        const uint16_t *r0, *r1;
        int mat, lrow;
        pair_rows<EPI>(a, p, col0, r0, r1, mat, lrow);
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
          const int v = vb + lane + 32 * j;
          if (v < ve) {
            wv[u][0][j] = ld_stream16(r0 + 8 * (size_t)v);
            wv[u][1][j] = ld_stream16(r1 + 8 * (size_t)v);
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int p = pb + u;
      if (p >= p1) break;
      float acc[2][NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[0][b] = acc[1][b] = 0.f;
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        const int v = vb + lane + 32 * j;
        if (v < ve) {
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            acc[0][b] += dot8(wv[u][0][j], xr[b][j]);
            acc[1][b] += dot8(wv[u][1][j], xr[b][j]);
          }
        }
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        acc[0][b] = warp_sum(acc[0][b]);
        acc[1][b] = warp_sum(acc[1][b]);
      }
      if (lane == 0) {
        float* r = red + ((size_t)(p - p0) * kWarps + warp) * 2 * NB;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          r[b] = acc[0][b];
          r[NB + b] = acc[1][b];
        }
      }
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- epilogue
  for (int t = threadIdx.x; t < (p1 - p0) * NB; t += kThreads) {
    const int pl = t / NB, b = t - pl * NB;
    if (b >= a.nb) continue;
    const int p = p0 + pl;
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float* r = red + ((size_t)pl * kWarps + w) * 2 * NB;
      y0 += r[b];
      y1 += r[NB + b];
    }
    const uint16_t *r0, *r1;
    int mat, lrow;
    pair_rows<EPI>(a, p, col0, r0, r1, mat, lrow);
    const int gb = a.b0 + b;
    if (EPI == EPI_PLAIN) {
      const size_t o = (size_t)seg * a.out_seg + (size_t)gb * a.ldo + lrow;
      *reinterpret_cast<float2*>(a.out + o) = make_float2(y0, y1);
      if (a.out_bf16)
        *reinterpret_cast<uint32_t*>(a.out_bf16 + o) =
            (uint32_t)f32_to_bf16_bits(y0) | ((uint32_t)f32_to_bf16_bits(y1) << 16);
    } else if (EPI == EPI_SWIGLU) {
      const float h = y0 / (1.0f + expf(-y0)) * y1;
      const size_t o = (size_t)gb * a.ldo + lrow;
      a.out[o] = h;
      if (a.out_bf16) a.out_bf16[o] = f32_to_bf16_bits(h);
    } else {  // EPI_QKV
      const int pos = a.pos[gb];
      const int d = lrow % kHeadDim;  // even: first element of the RoPE pair
      const int head = lrow / kHeadDim;
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
        *reinterpret_cast<float2*>(a.qout + (size_t)gb * a.n_heads * kHeadDim + lrow) =
            make_float2(y0, y1);
      } else {
        uint16_t* cache = mat == 1 ? a.kc : a.vc;
        const size_t o = (((size_t)gb * a.n_kv_heads + head) * a.max_seq + pos) * kHeadDim + d;
        *reinterpret_cast<uint32_t*>(cache + o) =
            (uint32_t)f32_to_bf16_bits(y0) | ((uint32_t)f32_to_bf16_bits(y1) << 16);
      }
    }
  }
}

template <int NB, int EPI, int VPL>
int launch_one(const GemvArgs& a, int max_pairs, cudaStream_t s) {
  const size_t smem = (size_t)max_pairs * kWarps * 2 * NB * sizeof(float);
  if (smem > 48 * 1024 && set_smem_once((const void*)k_gemv<NB, EPI, VPL>, (int)smem))
    return TP_ECUDA;
  k_gemv<NB, EPI, VPL><<<a.ctas_per_seg * a.nseg, kThreads, smem, s>>>(a);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

template <int NB, int EPI>
int launch_vpl(const GemvArgs& a, int max_pairs, cudaStream_t s) {
  const int nv = a.Ks >> 3;
  const int per_warp = ((nv >> 2) + kWarps - 1) / kWarps * 4;  // vectors, rounded up
  if (per_warp <= 32) return launch_one<NB, EPI, 1>(a, max_pairs, s);
  if (per_warp <= 64) return launch_one<NB, EPI, 2>(a, max_pairs, s);
  if constexpr (NB <= 2) {
    if (per_warp <= 128) return launch_one<NB, EPI, 4>(a, max_pairs, s);
  }
  if constexpr (NB == 1) {
    if (per_warp <= 256) return launch_one<NB, EPI, 8>(a, max_pairs, s);
  }
  return TP_ENOTSUP;
}

template <int NB>
int launch_nb(const GemvArgs& a, int epi, cudaStream_t s) {
  int vrows = a.rows[0];
  if (epi == EPI_QKV) vrows += a.rows[1] + a.rows[2];
  const int npairs = epi == EPI_SWIGLU ? vrows : vrows >> 1;
  const int max_pairs = (npairs + a.ctas_per_seg - 1) / a.ctas_per_seg;
  switch (epi) {
    case EPI_PLAIN: return launch_vpl<NB, EPI_PLAIN>(a, max_pairs, s);
    case EPI_SWIGLU: return launch_vpl<NB, EPI_SWIGLU>(a, max_pairs, s);
    default: return launch_vpl<NB, EPI_QKV>(a, max_pairs, s);
  }
}

}  // namespace

// Batch rows are processed in groups of at most 4 per launch (2 when a warp's
// column range needs more than 64 vectors, 1 above 128); the activations of a
// group live in registers. Column ranges above 256 vectors per warp (rows longer
// than 16384 elements per segment) are not supported.
int launch_gemv(const GemvArgs& a0, int epi, cudaStream_t s) {
  if (a0.Ks % 32 != 0 || a0.ctas_per_seg < 1) return TP_EINVAL;
  const int nv = a0.Ks >> 3;
  const int per_warp = ((nv >> 2) + kWarps - 1) / kWarps * 4;
  if (per_warp > 256) return TP_ENOTSUP;
  const int maxnb = per_warp <= 64 ? 4 : (per_warp <= 128 ? 2 : 1);
  for (int b = 0; b < a0.nb;) {
    GemvArgs a = a0;
    a.b0 = a0.b0 + b;
    int nb = a0.nb - b;
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
