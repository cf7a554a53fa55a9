// Decode attention over the bf16 KV cache, split over the context.
//
// distributed-llama issue #29, llamaMultiheadAtt: each slice computes the
// attention of its own heads locally; tt-metal's Llama-2 thread separates GQA
// from MHA. One CTA owns (batch row b, kv head, context chunk of 128
// positions) and all the query heads that share that kv head (1 for MHA, 8 for
// the 70B shape), so a K/V tile read from HBM serves every head of its group.
// The chunk's K and V rows are contiguous in the cache and arrive in shared
// memory by two bulk asynchronous copies (cp.async.bulk, completion counted on
// an mbarrier). Each CTA writes an unnormalised partial (o, running max m,
// sum l); a second kernel combines the chunks with the usual rescaling
//   M = max_c m_c,  o = sum_c e^{m_c - M} o_c / sum_c e^{m_c - M} l_c.
#include "kernels.cuh"

namespace tp {

namespace {

constexpr int kAttnThreads = 128;
constexpr uint32_t kSpinLimit = 1u << 26;  // bounded wait on the copy barrier

TP_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

TP_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

TP_DEV void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

TP_DEV bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(phase)
      : "memory");
  return ok != 0;
}

TP_DEV void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <int G>
__global__ void __launch_bounds__(kAttnThreads) k_attn_chunk(AttnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* Ks = reinterpret_cast<uint16_t*>(smem);                  // [128][128]
  uint16_t* Vs = Ks + kAttnChunk * kHeadDim;                         // [128][128]
  float* qs = reinterpret_cast<float*>(Vs + kAttnChunk * kHeadDim);  // [G][128]
  float* ps = qs + G * kHeadDim;                                     // [G][128]
  float* red = ps + G * kAttnChunk;                                  // [2][G][4]
  __shared__ uint64_t bar;

  const int c = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();  // q and the cache row at pos come from the q/k/v kernel
  const int P = a.pos[b] + 1;
  const int t0 = c * kAttnChunk;
  const size_t pbase = ((size_t)b * a.H + (size_t)kvh * G) * a.nchunk + c;
  if (t0 >= P) {
    if (tid < G) {
      a.part_ml[(pbase + (size_t)tid * a.nchunk) * 2 + 0] = -INFINITY;
      a.part_ml[(pbase + (size_t)tid * a.nchunk) * 2 + 1] = 0.f;
    }
    return;
  }
  const int nt = min(kAttnChunk, P - t0);
  const uint32_t bytes = (uint32_t)nt * kHeadDim * 2;
  const size_t row0 = (((size_t)b * a.Hkv + kvh) * a.max_seq + t0) * kHeadDim;

  if (tid == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_expect_tx(&bar, 2 * bytes);
    bulk_g2s(Ks, a.kc + row0, bytes, &bar);
    bulk_g2s(Vs, a.vc + row0, bytes, &bar);
  }
  // q of the group's heads, pre-scaled by 1/sqrt(hd)
  const float scale = 1.0f / sqrtf((float)kHeadDim);
  for (int i = tid; i < G * kHeadDim; i += kAttnThreads) {
    const int g = i / kHeadDim, d = i - g * kHeadDim;
    qs[i] = a.q[((size_t)b * a.H + (size_t)kvh * G + g) * kHeadDim + d] * scale;
  }
  __syncthreads();
  {
    uint32_t spins = 0;
    while (!mbar_try_wait(&bar, 0)) {
      if (++spins > kSpinLimit) {
        if (tid == 0) atomicExch(a.err, 1);
        break;
      }
    }
  }

  // scores: thread t owns position t0+t; reads its K row in 16-byte chunks with a
  // per-thread rotation so that the 8 threads of a quarter-warp hit 8 different
  // bank groups.
  float s[G];
#pragma unroll
  for (int g = 0; g < G; ++g) s[g] = -INFINITY;
  if (tid < nt) {
#pragma unroll
    for (int g = 0; g < G; ++g) s[g] = 0.f;
    const uint4* krow = reinterpret_cast<const uint4*>(Ks + tid * kHeadDim);
#pragma unroll 4
    for (int j = 0; j < 16; ++j) {
      const int cch = (j + tid) & 15;
      const uint4 kv = krow[cch];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float4 q0 = reinterpret_cast<const float4*>(qs + g * kHeadDim)[2 * cch];
        const float4 q1 = reinterpret_cast<const float4*>(qs + g * kHeadDim)[2 * cch + 1];
        float acc = s[g];
        acc = fmaf(bf16lo(kv.x), q0.x, acc);
        acc = fmaf(bf16hi(kv.x), q0.y, acc);
        acc = fmaf(bf16lo(kv.y), q0.z, acc);
        acc = fmaf(bf16hi(kv.y), q0.w, acc);
        acc = fmaf(bf16lo(kv.z), q1.x, acc);
        acc = fmaf(bf16hi(kv.z), q1.y, acc);
        acc = fmaf(bf16lo(kv.w), q1.z, acc);
        acc = fmaf(bf16hi(kv.w), q1.w, acc);
        s[g] = acc;
      }
    }
  }
  // softmax over the chunk (per head of the group)
  const int lane = tid & 31, wid = tid >> 5;
  float* rmax = red;
  float* rsum = red + G * 4;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float m = warp_max(s[g]);
    if (lane == 0) rmax[g * 4 + wid] = m;
  }
  __syncthreads();
  float mg[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    mg[g] = fmaxf(fmaxf(rmax[g * 4 + 0], rmax[g * 4 + 1]), fmaxf(rmax[g * 4 + 2], rmax[g * 4 + 3]));
    const float p = tid < nt ? expf(s[g] - mg[g]) : 0.f;
    ps[g * kAttnChunk + tid] = p;
    const float l = warp_sum(p);
    if (lane == 0) rsum[g * 4 + wid] = l;
  }
  __syncthreads();

  // o[g][d] = sum_t p[g][t] v[t][d]; thread tid owns dimension d = tid
  float o[G];
#pragma unroll
  for (int g = 0; g < G; ++g) o[g] = 0.f;
  const int d = tid;
#pragma unroll 4
  for (int t = 0; t < nt; ++t) {
    const float v = __uint_as_float(((uint32_t)Vs[t * kHeadDim + d]) << 16);
#pragma unroll
    for (int g = 0; g < G; ++g) o[g] = fmaf(ps[g * kAttnChunk + t], v, o[g]);
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const size_t pi = pbase + (size_t)g * a.nchunk;
    a.part_o[pi * kHeadDim + d] = o[g];
    if (tid == 0) {
      a.part_ml[pi * 2 + 0] = mg[g];
      a.part_ml[pi * 2 + 1] = rsum[g * 4 + 0] + rsum[g * 4 + 1] + rsum[g * 4 + 2] + rsum[g * 4 + 3];
    }
  }
}

// One CTA per (head, batch row); thread d owns output dimension d.
__global__ void __launch_bounds__(kHeadDim) k_attn_combine(AttnArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int P = a.pos[b] + 1;
  const int nc = (P + kAttnChunk - 1) / kAttnChunk;
  const size_t base = ((size_t)b * a.H + h) * a.nchunk;
  float M = -INFINITY;
  for (int c = 0; c < nc; ++c) M = fmaxf(M, a.part_ml[(base + c) * 2]);
  float l = 0.f, o = 0.f;
  for (int c = 0; c < nc; ++c) {
    const float w = expf(a.part_ml[(base + c) * 2] - M);
    l = fmaf(w, a.part_ml[(base + c) * 2 + 1], l);
    o = fmaf(w, a.part_o[(base + c) * kHeadDim + d], o);
  }
  const float r = o / l;
  const size_t oi = ((size_t)b * a.H + h) * kHeadDim + d;
  a.att[oi] = r;
  if (a.att_bf16) {  // hi/lo bf16 pair: rows 2b and 2b+1 of [2B, H*hd]
    const size_t row = (size_t)a.H * kHeadDim;
    const size_t hi = (size_t)(2 * b) * row + (size_t)h * kHeadDim + d;
    bf16_split(r, a.att_bf16[hi], a.att_bf16[hi + row]);
  }
}

template <int G>
int launch_g(const AttnArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)2 * kAttnChunk * kHeadDim * 2 + (size_t)G * kHeadDim * 4 +
                      (size_t)G * kAttnChunk * 4 + (size_t)2 * G * 4 * 4;
  if (set_smem_once((const void*)k_attn_chunk<G>, (int)smem)) return TP_ECUDA;
  return launch_pdl(k_attn_chunk<G>, dim3(a.nchunk, a.Hkv, a.B), dim3(kAttnThreads), smem, s, a);
}

}  // namespace

int launch_attention(const AttnArgs& a, cudaStream_t s) {
  const int G = a.H / a.Hkv;
  int rc;
  switch (G) {
    case 1: rc = launch_g<1>(a, s); break;
    case 2: rc = launch_g<2>(a, s); break;
    case 4: rc = launch_g<4>(a, s); break;
    case 8: rc = launch_g<8>(a, s); break;
    default: return TP_ENOTSUP;
  }
  if (rc != TP_OK) return rc;
  return launch_pdl(k_attn_combine, dim3(a.H, a.B), dim3(kHeadDim), 0, s, a);
}

}  // namespace tp
