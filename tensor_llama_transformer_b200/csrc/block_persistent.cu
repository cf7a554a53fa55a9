// Persistent decode block for batch 1-2: the whole block forward as ONE
// cooperative kernel, one CTA per SM.
//
// The block's steps (distributed-llama issue #29 task list: RMSNorm(+Q8) ->
// q/k/v slice products with RoPE and the cache write -> per-slice attention ->
// W_O row-split partials -> merge -> RMSNorm(+Q8) -> W1/W3 slice products with
// SwiGLU -> W2 row-split partials -> merge) become phases of one launch,
// separated by grid-wide barriers:
//   A  q/k/v rows      (activation: RMSNorm(x)*g, +Q8 when the sync is quantised)
//   -- barrier 1
//   B  attention tiles (64-position K/V tiles of every (batch row, kv head))
//   -- barrier 2
//   C  W_O rows        (activation: the context splits of each head combined)
//   -- barrier 3
//   M  x_mid = x + sum_s sync(W_O partial_s), each 128-value chunk by one warp
//   -- barrier 4
//   D  W1/W3 rows      (activation: RMSNorm(x_mid)*g, +Q8)
//   -- barrier 5
//   E  W2 rows         (activation: the SwiGLU output h)
//   -- barrier 6
//   F  x = x_mid + sum_s sync(W2 partial_s)
// Within a CTA, one producer warp streams everything the CTA will read from HBM
// (the RMSNorm inputs, its share of every weight matrix, its attention tiles)
// through one shared-memory ring of variable-size stages, and never waits for a
// grid barrier: weights are read-only, x changes only in phase F, and cache rows
// below pos are not written in this step. Only the attention tiles that hold
// position pos (written in phase A by another CTA) wait for barrier 1. So while
// the consumer warps sit at a barrier, the next phase's first ~200 KB per SM is
// already arriving, and HBM stays busy across the step instead of draining at
// every kernel boundary. Weights and cache tiles are read with an L2 evict-first
// policy, which keeps the small activations and partials that the phases pass
// to one another resident in L2.
//
// The eight consumer warps do the arithmetic of each phase:
//   GEMV phases: as the ring-buffer slice GEMV (rows in pairs, each pair split
//   over 8 / pairs warps, packed f32x2 FMA against float32 activations staged
//   in shared memory, per-row partial sums combined in a fixed order);
//   attention: as the split flash-decoding kernel (mma.m16n8k16 with hi/lo bf16
//   Q and P rows, online softmax in registers), four warps per tile, the two
//   halves of the consumers taking alternate tiles of a head; each CTA writes
//   one partial (o, m, l) per head group it touched.
// Activations that several CTAs need (normalised x_mid, the attention output
// combined from its splits) are recomputed by every CTA that needs them, from
// the previous phase's outputs in L2, instead of by a separate kernel.
//
// Every wait is bounded (2 s): mbarrier waits and grid-barrier spins raise the
// error word and the kernel walks on without the data, so it always exits.
#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "pipeline.cuh"

namespace tp {

namespace {

constexpr int kNC = 8;                      // consumer warps
constexpr int kNCons = 32 * kNC;
constexpr int kThreads = kNCons + 32;       // + the producer warp
constexpr int kMaxQ = 16;                   // stages in flight (mbarrier pairs)
constexpr int kTileP = 64;                  // positions per attention tile
constexpr uint32_t kTileBytes = 4 * 8192;   // K and V, two 64-dim boxes each
constexpr int kQStride = 136;               // staged Q rows (bf16), padded
constexpr uint32_t kQsBytes = 16 * kQStride * 2;
constexpr int kMaxSlices = 8;               // slices whose partials a merge holds at once
constexpr int kMaxSegHeads = 64;            // query heads per W_O segment

enum { PH_QKV = 0, PH_WO = 1, PH_W13 = 2, PH_W2 = 3 };

TP_DEV uint32_t round1k(uint32_t v) { return (v + 1023u) & ~1023u; }

TP_DEV void stamp(const BpArgs& a, int slot) {
  if (a.trace) a.trace[(size_t)blockIdx.x * TP_BLOCK_TRACE_SLOTS + slot] = gtimer();
}

TP_DEV unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

TP_DEV bool wait_count(const unsigned* p, unsigned target, int* err) {
  if (ld_acquire(p) >= target) return true;
  const uint64_t t0 = gtimer();
  while (ld_acquire(p) < target) {
    if (gtimer() - t0 > kWaitTimeoutNs) {
      atomicExch(err, 1);
      return false;
    }
  }
  return true;
}

// Grid barrier k (1-based) among the consumer warps of every CTA: a release
// add on the arrival counter, then acquire loads until every CTA has arrived.
// The counter starts at zero and the last CTA to leave the kernel puts it back.
TP_DEV void grid_barrier(unsigned* bar, int k, int* err) {
  consumers_sync(kNCons);
  if (threadIdx.x == 0) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(bar) : "memory");
    wait_count(bar, (unsigned)k * gridDim.x, err);
  }
  consumers_sync(kNCons);
}

// Stages take contiguous ring bytes; a stage that would straddle the end starts
// over at offset 0. The producer also keeps a virtual (monotone) byte position
// to tell which stages in flight a new stage would overwrite.
TP_DEV uint32_t ring_take(uint32_t& phys, uint64_t& virt, uint32_t sz, uint32_t ring) {
  if (phys + sz > ring) {
    virt += ring - phys;
    phys = 0;
  }
  const uint32_t off = phys;
  phys += sz;
  virt += sz;
  return off;
}

// ------------------------------------------------------------------ GEMV phases
TP_DEV void gemv_range(const BpGemv& g, int& R0, int& nrows) {
  const int npairs = g.nseg * (g.rps >> 1);
  const int P0 = (int)(((int64_t)npairs * blockIdx.x) / gridDim.x);
  const int P1 = (int)(((int64_t)npairs * (blockIdx.x + 1)) / gridDim.x);
  R0 = 2 * P0;
  nrows = 2 * (P1 - P0);
}

// Matrix and row of virtual row r of a segment (SwiGLU interleaves W1[f], W3[f];
// q/k/v stack the three matrices).
template <int EPI>
TP_DEV void row_of(const BpGemv& g, int r, int& mat, int& lrow) {
  mat = 0;
  lrow = r;
  if (EPI == EPI_SWIGLU) {
    mat = r & 1;
    lrow = r >> 1;
  } else if (EPI == EPI_QKV && lrow >= g.rows[0]) {
    lrow -= g.rows[0];
    mat = 1;
    if (lrow >= g.rows[1]) {
      lrow -= g.rows[1];
      mat = 2;
    }
  }
}

struct Producer {
  uint8_t* ring;
  uint32_t ring_bytes;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* st_start;  // virtual start of each stage in flight
  uint64_t virt;
  uint32_t phys;
  int t, tail;
  int* err;
  uint64_t pol;  // L2 evict-first: weights and cache tiles are read once per step

  // Reserves sz ring bytes for stage t once the stages occupying them (and the
  // stage that last used descriptor t % kMaxQ) have been handed back.
  TP_DEV bool acquire(uint32_t sz, uint32_t& off) {
    off = ring_take(phys, virt, sz, ring_bytes);
    const uint64_t vs = virt - sz;
    while (tail < t && (t - tail >= kMaxQ || virt - st_start[tail % kMaxQ] > ring_bytes)) {
      if (!mbar_wait(&empty[tail % kMaxQ], (uint32_t)(tail / kMaxQ) & 1u, err)) return false;
      ++tail;
    }
    st_start[t % kMaxQ] = vs;
    return true;
  }

  // The inputs of an RMSNorm staging, ahead of the phase's weights: the residual
  // rows x [nb, D] (nb = 0: none) and the gain [D]; x changes only in the final
  // merge.
  TP_DEV bool norm_inputs(const float* x, int nb, int D, const float* gain) {
    const uint32_t xb = (uint32_t)nb * D * 4, gb = (uint32_t)D * 4;
    uint32_t off;
    if (!acquire(round1k(xb + gb), off)) return false;
    uint64_t* bar = &full[t % kMaxQ];
    mbar_expect_tx(bar, xb + gb);
    if (xb) bulk_g2s(ring + off, x, xb, bar);
    bulk_g2s(ring + off + xb, gain, gb, bar);
    ++t;
    return true;
  }

  template <int EPI>
  TP_DEV bool gemv(const BpGemv& g) {
    int R0, nrows;
    gemv_range(g, R0, nrows);
    const uint32_t rb = (uint32_t)g.Ks * 2;
    int seg = R0 / g.rps, seg_end = (seg + 1) * g.rps - R0;  // CTA-local end of the segment
    for (int cur = 0; cur < nrows;) {
      if (cur == seg_end) {
        ++seg;
        seg_end += g.rps;
      }
      const int end = min(min(nrows, seg_end), cur + 2 * g.pairs);
      const int n = end - cur;
      uint32_t off;
      if (!acquire(round1k((uint32_t)n * rb), off)) return false;
      uint64_t* bar = &full[t % kMaxQ];
      mbar_expect_tx(bar, (uint32_t)n * rb);
      uint8_t* dst = ring + off;
      const int lr0 = R0 + cur - seg * g.rps;
      const size_t col0 = (size_t)seg * g.Ks;
      if (EPI == EPI_SWIGLU) {  // rows alternate W1[f], W3[f]
        const uint16_t* p1 = g.w[0] + (size_t)(lr0 >> 1) * g.ldw + col0;
        const uint16_t* p3 = g.w[1] + (size_t)(lr0 >> 1) * g.ldw + col0;
        for (int i = 0; i < n; i += 2) {
          bulk_g2s_hint(dst + (size_t)i * rb, p1, rb, bar, pol);
          bulk_g2s_hint(dst + (size_t)(i + 1) * rb, p3, rb, bar, pol);
          p1 += g.ldw;
          p3 += g.ldw;
        }
      } else {  // runs of rows inside one matrix; one copy per run of contiguous rows
        int done = 0, r = lr0;
        while (done < n) {
          int mat, lrow;
          row_of<EPI>(g, r, mat, lrow);
          const uint16_t* src = g.w[mat] + (size_t)lrow * g.ldw + col0;
          int mat_end = g.rows[0];
          if (EPI == EPI_QKV) mat_end = mat == 0 ? g.rows[0] : (mat == 1 ? g.rows[0] + g.rows[1] : g.rps);
          const int run = min(n - done, mat_end - r);
          if (g.ldw == g.Ks) {
            bulk_g2s_hint(dst + (size_t)done * rb, src, (uint32_t)run * rb, bar, pol);
          } else {
            for (int i = 0; i < run; ++i, src += g.ldw)
              bulk_g2s_hint(dst + (size_t)(done + i) * rb, src, rb, bar, pol);
          }
          done += run;
          r += run;
        }
      }
      ++t;
      cur = end;
    }
    return true;
  }
};

// ------------------------------------------------------------------ attention work
// The attention work of the step is the list of (batch row, kv head, tile)
// in that order; CTA c takes the contiguous range [c T / G, (c+1) T / G).
struct AttnWork {
  int total;
  int nt[2];   // tiles per head of each batch row
  int off[2];  // first list index of each batch row
  int u0, u1;  // this CTA's range
};

TP_DEV void attn_work(const BpArgs& a, AttnWork& w) {
  w.total = 0;
  for (int b = 0; b < 2; ++b) {
    w.off[b] = w.total;
    w.nt[b] = b < a.nb ? (a.pos[b] + kTileP) / kTileP : 0;  // ceil((pos + 1) / 64)
    w.total += a.Hkv * w.nt[b];
  }
  // total * grid stays far below 2^32 (at most 2 x 128 heads x 2048 tiles x 148)
  w.u0 = (int)(((unsigned)w.total * blockIdx.x) / gridDim.x);
  w.u1 = (int)(((unsigned)w.total * (blockIdx.x + 1)) / gridDim.x);
}

TP_DEV void attn_decode(const AttnWork& w, int u, int& b, int& kvh, int& i) {
  b = (w.nt[1] > 0 && u >= w.off[1]) ? 1 : 0;
  const int r = u - w.off[b];
  kvh = r / w.nt[b];
  i = r - kvh * w.nt[b];
}

// The CTA whose range holds list index u.
TP_DEV int attn_cta_of(const AttnWork& w, int u) {
  return (int)(((unsigned)(u + 1) * gridDim.x - 1u) / (unsigned)w.total);
}

// Context split of CTA c for the head group whose first list index is uf: the
// split is stored at slot = the group's first tile in that CTA's range; -1 when
// the CTA has no tiles at all (fewer tiles than CTAs).
TP_DEV int split_slot(const AttnWork& w, int uf, int c) {
  const int start = (int)(((unsigned)w.total * (unsigned)c) / gridDim.x);
  const int end = (int)(((unsigned)w.total * (unsigned)(c + 1)) / gridDim.x);
  if (end <= start) return -1;
  return (start > uf ? start : uf) - uf;
}

TP_DEV bool produce_attn(Producer& pr, const BpArgs& a, const CUtensorMap* mK,
                         const CUtensorMap* mV) {
  AttnWork w;
  attn_work(a, w);
  bool after_b1 = false;
  for (int u = w.u0; u < w.u1; ++u) {
    int b, kvh, i;
    attn_decode(w, u, b, kvh, i);
    if (i == w.nt[b] - 1 && !after_b1) {  // the tile holds row pos, written in phase A
      wait_count(a.bar, gridDim.x, a.err);
      asm volatile("fence.proxy.async.global;" ::: "memory");
      after_b1 = true;
    }
    uint32_t off;
    if (!pr.acquire(kTileBytes, off)) return false;
    uint64_t* bar = &pr.full[pr.t % kMaxQ];
    mbar_expect_tx(bar, kTileBytes);
    uint8_t* st = pr.ring + off;
    const int y = (b * a.Hkv + kvh) * a.max_seq + i * kTileP;
    tma_load_2d_hint(st, mK, 0, y, bar, pr.pol);
    tma_load_2d_hint(st + 8192, mK, 64, y, bar, pr.pol);
    tma_load_2d_hint(st + 16384, mV, 0, y, bar, pr.pol);
    tma_load_2d_hint(st + 24576, mV, 64, y, bar, pr.pol);
    ++pr.t;
  }
  return true;
}

// ------------------------------------------------------------------ consumers
struct Consumer {
  uint8_t* ring;
  uint32_t ring_bytes;
  uint64_t* full;
  uint64_t* empty;
  uint64_t virt;
  uint32_t phys;
  int t;
  bool ok;
  int* err;

  uint64_t waited;  // ns spent waiting for stages (thread 0, when tracing)
  bool timed;

  // Waits for the next stage (sz bytes); returns its shared-memory offset.
  TP_DEV uint32_t next(uint32_t sz) {
    const uint32_t off = ring_take(phys, virt, sz, ring_bytes);
    const uint64_t t0 = timed ? gtimer() : 0;
    const bool got = ok ? mbar_wait(&full[t % kMaxQ], (uint32_t)(t / kMaxQ) & 1u, err) : false;
    if (timed) waited += gtimer() - t0;
    ok = __all_sync(0xffffffffu, got);
    return off;
  }
  TP_DEV void release() {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&empty[t % kMaxQ]);
    ++t;
  }
};

// One GEMV phase for the consumer warps. stage(seg, publish) fills xs with the
// segment's activations (lo halves [NB][nv], then hi halves); res receives the
// per-row partial sums [row][NB][split].
template <int NB, int EPI, class Stage>
TP_DEV void consume_gemv(Consumer& c, const BpGemv& g, float4* xs, float* res, int& R0, int& nrows,
                         Stage&& stage, bool release_input = false) {
  gemv_range(g, R0, nrows);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = g.Ks >> 3;
  const uint32_t rb = (uint32_t)g.Ks * 2;
  const int Q = g.split;
  const int pw = warp / Q, part = warp - pw * Q;
  const int vb = (nv * part) / Q, ve = (nv * (part + 1)) / Q;
  int seg = R0 / g.rps, seg_end = (seg + 1) * g.rps - R0;  // CTA-local end of the segment
  for (int cur = 0; cur < nrows;) {
    if (cur == 0 || cur == seg_end) {
      if (cur == seg_end) {
        ++seg;
        seg_end += g.rps;
      }
      consumers_sync(kNCons);
      stage(seg, (R0 + cur) == seg * g.rps);
      consumers_sync(kNCons);
      if (release_input && cur == 0) c.release();  // the staged inputs' ring stage
    }
    const int end = min(min(nrows, seg_end), cur + 2 * g.pairs);
    const uint32_t off = c.next(round1k((uint32_t)(end - cur) * rb));
    if (c.ok) {
      if (g.pw == 2) ring_pairs_dot<NB, 2>(c.ring + off, cur, end, xs, res, nv, rb, pw, part, Q, vb, ve, lane);
      else ring_pairs_dot<NB, 1>(c.ring + off, cur, end, xs, res, nv, rb, pw, part, Q, vb, ve, lane);
    }
    c.release();
    cur = end;
  }
  if (release_input && nrows == 0) c.release();
  consumers_sync(kNCons);
}

// Sum of the split parts of the CTA's row pair pr for batch row b.
template <int NB>
TP_DEV void pair_sums(const float* res, int Q, int pr, int b, float& y0, float& y1) {
  y0 = 0.f;
  y1 = 0.f;
  for (int q = 0; q < Q; ++q) {
    y0 += res[((size_t)(2 * pr) * NB + b) * Q + q];
    y1 += res[((size_t)(2 * pr + 1) * NB + b) * Q + q];
  }
}

TP_DEV void load8(const float* p, float (&v)[8]) {
  const float4 l = *reinterpret_cast<const float4*>(p);
  const float4 h = *reinterpret_cast<const float4*>(p + 4);
  v[0] = l.x; v[1] = l.y; v[2] = l.z; v[3] = l.w;
  v[4] = h.x; v[5] = h.y; v[6] = h.z; v[7] = h.w;
}

// The same through L2 only: data written by other CTAs during this launch.
TP_DEV void load8cg(const float* p, float (&v)[8]) {
  const float4 l = __ldcg(reinterpret_cast<const float4*>(p));
  const float4 h = __ldcg(reinterpret_cast<const float4*>(p + 4));
  v[0] = l.x; v[1] = l.y; v[2] = l.z; v[3] = l.w;
  v[4] = h.x; v[5] = h.y; v[6] = h.z; v[7] = h.w;
}

TP_DEV void store8(float* p, const float (&v)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// Activations of phases A and D: RMSNorm(src) * gain (+Q8). Phase A: src = x
// from the ring (shared memory), the scale from its own sum of squares. Phase D:
// src = x_mid from L2, the scale from the per-chunk sums of squares the merge
// wrote (ssq, [nb][D/128], summed in order). The CTA that owns the first row
// publishes the shared buffers (xq/xd, xn).
template <int NB>
TP_DEV void stage_norm(const BpArgs& a, float4* xs, const float* xsrc, bool src_global,
                       const float* gain, const float* ssq, bool publish, float (*s_red)[2],
                       float* s_rstd) {
  const int D = a.D, nv = D >> 3, nvr = (nv + 31) & ~31;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int b = 0; b < NB; ++b) {
    float ss = 0.f;
#pragma unroll 4
    for (int v = threadIdx.x; v < nv; v += kNCons) {
      const size_t e0 = (size_t)b * D + 8 * (size_t)v;
      float xm[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (b < a.nb) {
        if (src_global) load8cg(xsrc + e0, xm);
        else load8(xsrc + e0, xm);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += xm[e] * xm[e];
      xs[b * nv + v] = make_float4(xm[0], xm[1], xm[2], xm[3]);
      xs[(NB + b) * nv + v] = make_float4(xm[4], xm[5], xm[6], xm[7]);
    }
    if (!ssq) {
      ss = warp_sum(ss);
      if (lane == 0) s_red[warp][b] = ss;
    }
  }
  if (ssq && warp < NB) {  // warp b sums row b's per-chunk sums of squares
    const int chunks = D >> 7;
    float t = 0.f;
    if (warp < a.nb)
      for (int k = lane; k < chunks; k += 32) t += __ldcg(ssq + (size_t)warp * chunks + k);
    t = warp_sum(t);
    if (lane == 0) s_red[0][warp] = t;
  }
  consumers_sync(kNCons);
  if (threadIdx.x < NB) {
    float tsum = 0.f;
    if (ssq) {
      tsum = s_red[0][threadIdx.x];
    } else {
      for (int w = 0; w < kNC; ++w) tsum += s_red[w][threadIdx.x];
    }
    s_rstd[threadIdx.x] = 1.0f / sqrtf(tsum / (float)D + a.eps);
  }
  consumers_sync(kNCons);
  for (int b = 0; b < NB; ++b) {
    const float rstd = s_rstd[b];
    for (int v = threadIdx.x; v < nvr; v += kNCons) {
      const bool in = b < a.nb && v < nv;
      const size_t e0 = (size_t)b * D + 8 * (size_t)v;
      float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (in) {
        const float4 l = xs[b * nv + v], h = xs[(NB + b) * nv + v];
        const float xm[8] = {l.x, l.y, l.z, l.w, h.x, h.y, h.z, h.w};
        float gg[8];
        load8(gain + 8 * (size_t)v, gg);
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = __fmul_rn(__fmul_rn(xm[e], rstd), gg[e]);
        if (publish) store8(a.xn + e0, y);  // before any Q8 round trip
      }
      if (a.quant) {
        float am = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(y[e]));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
        const float d = q8_scale(am);
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int code = q8_code(y[e], d);
          y[e] = q8_value(code, d);
          if (e < 4) lo |= (uint32_t)(code & 0xFF) << (8 * e);
          else hi |= (uint32_t)(code & 0xFF) << (8 * (e - 4));
        }
        if (publish && in) {
          *reinterpret_cast<uint2*>(a.xq + e0) = make_uint2(lo, hi);
          if ((lane & 3) == 0) a.xd[e0 / kQ8Block] = d;
        }
      }
      if (in) {
        xs[b * nv + v] = make_float4(y[0], y[1], y[2], y[3]);
        xs[(NB + b) * nv + v] = make_float4(y[4], y[5], y[6], y[7]);
      }
    }
  }
}

// out = base + sum_s sync(part_s), slices in order (the merge kernel's
// arithmetic): one warp per 128 values of a row (a float4 per lane, 8-lane Q8
// groups), spread over the whole grid. With ssq_out, each warp also writes the
// sum of squares of its 128 values, [nb][D/128].
TP_DEV void merge_rows(const BpArgs& a, const float* base, float* out, float* ssq_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int D = a.D, chunks = D >> 7;
  // item i goes to CTA i % grid, warp i / grid: one warp per SM while there are
  // fewer items than SMs
  for (int item = warp * gridDim.x + blockIdx.x; item < a.nb * chunks; item += gridDim.x * kNC) {
    const int b = item / chunks, i4 = (item - b * chunks) * 32 + lane;
    float4 p[kMaxSlices];
#pragma unroll
    for (int s = 0; s < kMaxSlices; ++s)
      p[s] = s < a.n ? __ldcg(reinterpret_cast<const float4*>(a.part + ((size_t)s * a.nb + b) * D) + i4)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 v = __ldcg(reinterpret_cast<const float4*>(base + (size_t)b * D) + i4);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < kMaxSlices; ++s) {
      if (s >= a.n) break;
      if (a.quant) q8_roundtrip4(p[s]);
      acc.x += p[s].x;
      acc.y += p[s].y;
      acc.z += p[s].z;
      acc.w += p[s].w;
    }
    v.x += acc.x;
    v.y += acc.y;
    v.z += acc.z;
    v.w += acc.w;
    reinterpret_cast<float4*>(out + (size_t)b * D)[i4] = v;
    if (ssq_out) {
      const float sq = warp_sum(v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w);
      if (lane == 0) ssq_out[item] = sq;
    }
  }
}

// Activations of phase C for W_O segment seg: the attention output of the
// segment's heads, each combined from its context splits (the CTAs whose tile
// ranges cover the head group):
//   M = max_j m_j,  o = sum_j e^{m_j - M} o_j / sum_j e^{m_j - M} l_j.
// Each thread combines 8 output values in two rounds of loads: the splits'
// maxima, then their sums and partial outputs (splits in CTA order). The owner
// of the segment's first row publishes att.
template <int NB>
TP_DEV void stage_att(const BpArgs& a, const AttnWork& w, int seg, int Ks, bool publish,
                      float4* xs) {
  const int hs = Ks / kHeadDim, G = a.H / a.Hkv, nv = Ks >> 3;
  for (int idx = threadIdx.x; idx < NB * nv; idx += kNCons) {
    const int b = idx / nv, v = idx - b * nv;
    float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (b < a.nb) {
      const int hl = v >> 4, d0 = (v & 15) * 8;  // 16 vectors of 8 per head
      const int h = seg * hs + hl, uf = w.off[b] + (h / G) * w.nt[b];
      const int clo = attn_cta_of(w, uf), chi = attn_cta_of(w, uf + w.nt[b] - 1);
      const float* ml = a.part_ml + ((size_t)b * a.H + h) * a.nchunk * 2;
      const float* po = a.part_o + ((size_t)b * a.H + h) * a.nchunk * kHeadDim + d0;
      float M = -INFINITY;
      for (int c0 = clo; c0 <= chi; c0 += 8) {  // eight splits' loads in flight
        float mq[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int slot = c0 + q <= chi ? split_slot(w, uf, c0 + q) : -1;
          mq[q] = slot >= 0 ? __ldcg(ml + 2 * slot) : -INFINITY;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) M = fmaxf(M, mq[q]);
      }
      float L = 0.f;
      for (int c0 = clo; c0 <= chi; c0 += 4) {  // four splits' loads in flight
        float mj[4], lj[4], pj[4][8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int slot = c0 + q <= chi ? split_slot(w, uf, c0 + q) : -1;
          mj[q] = -INFINITY;
          lj[q] = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) pj[q][e] = 0.f;
          if (slot >= 0) {
            mj[q] = __ldcg(ml + 2 * slot);
            lj[q] = __ldcg(ml + 2 * slot + 1);
            load8cg(po + (size_t)slot * kHeadDim, pj[q]);
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float wj = mj[q] == -INFINITY ? 0.f : expf(mj[q] - M);
          L = fmaf(wj, lj[q], L);
#pragma unroll
          for (int e = 0; e < 8; ++e) o[e] = fmaf(wj, pj[q][e], o[e]);
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = o[e] / L;
      if (publish) store8(a.att + (size_t)b * a.QD + (size_t)seg * Ks + 8 * v, o);
    }
    xs[b * nv + v] = make_float4(o[0], o[1], o[2], o[3]);
    xs[(NB + b) * nv + v] = make_float4(o[4], o[5], o[6], o[7]);
  }
}

// Activations of phases C and E for segment seg: a float32 row segment that
// other CTAs wrote earlier in this launch (the attention output, the SwiGLU
// output h), read through L2.
template <int NB>
TP_DEV void stage_plain(const float* src, int ld, int nb, int seg, int Ks, float4* xs) {
  const int nv = Ks >> 3;
  for (int idx = threadIdx.x; idx < NB * nv; idx += kNCons) {
    const int b = idx / nv, v = idx - b * nv;
    float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (b < nb) load8cg(src + (size_t)b * ld + (size_t)seg * Ks + 8 * v, y);
    xs[b * nv + v] = make_float4(y[0], y[1], y[2], y[3]);
    xs[(NB + b) * nv + v] = make_float4(y[4], y[5], y[6], y[7]);
  }
}

// Attention of the CTA's tiles (phase B). Warps 0-3 take the even tiles of a
// head, warps 4-7 the odd ones; each warp covers 16 positions of a tile. At the
// end of each head the 8 warps' partials are merged and written as the CTA's
// split of that head.
template <int NB>
TP_DEV void consume_attn(Consumer& c, const BpArgs& a, const AttnWork& w, uint8_t* xsb,
                         float (*s_m)[8], float (*s_l)[8]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.H / a.Hkv;
  float* ro = reinterpret_cast<float*>(xsb);  // the warps' partials [8][G][128]
  uint16_t* qs = reinterpret_cast<uint16_t*>(xsb + (size_t)kNC * (a.H / a.Hkv) * kHeadDim * 4);
  const int grp = warp >> 2, w0 = 16 * (warp & 3);
  const int g = lane >> 2;
  const float scale = 1.0f / sqrtf((float)kHeadDim);
  for (int u = w.u0; u < w.u1;) {
    int b, kvh, i0;
    attn_decode(w, u, b, kvh, i0);
    const int uf = w.off[b] + kvh * w.nt[b];
    const int useg = min(w.u1, uf + w.nt[b]);  // this head's tiles in the range: [u, useg)
    const int P = a.pos[b] + 1;
    consumers_sync(kNCons);  // ro / qs free
    for (int idx = threadIdx.x; idx < 8 * kHeadDim; idx += kNCons) {
      const int gg = idx / kHeadDim, d = idx - gg * kHeadDim;
      uint16_t hi = 0, lo = 0;
      if (gg < G)
        bf16_split(a.q[((size_t)b * a.H + (size_t)kvh * G + gg) * kHeadDim + d] * scale, hi, lo);
      qs[gg * kQStride + d] = hi;
      qs[(gg + 8) * kQStride + d] = lo;
    }
    consumers_sync(kNCons);
    uint32_t qa[8][4];
    {
      const uint32_t qb = s2u(qs);
      const int r = (lane & 7) + 8 * ((lane >> 3) & 1), ch = lane >> 4;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        ldsm_x4(qb + (uint32_t)((r * kQStride + 16 * ks + 8 * ch) * 2), qa[ks]);
    }
    float m_run = -INFINITY, l_run = 0.f;
    float o[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    for (int k = 0; u + k < useg; ++k) {
      const uint32_t off = c.next(kTileBytes);
      if (c.ok && (k & 1) == grp) {
        const uint32_t kb = s2u(c.ring + off), vb = kb + 16384;
        const int t0 = (i0 + k) * kTileP;
        if (t0 + w0 + 16 > P) {  // V rows past pos -> 0 (only the head's last tile)
          for (int idx = lane; idx < 16 * 16; idx += 32) {
            const int r = idx >> 4, cc = idx & 15;
            if (t0 + w0 + r >= P)
              *reinterpret_cast<uint4*>(c.ring + (kv_tile_addr(vb, w0 + r, cc) - s2u(c.ring))) =
                  make_uint4(0u, 0u, 0u, 0u);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
        }
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
          const int tt = w0 + (lane & 7) + 8 * (lane >> 4), ch = (lane >> 3) & 1;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            uint32_t bf[4];
            ldsm_x4(kv_tile_addr(kb, tt, 2 * ks + ch), bf);
            mma_bf16(sc[0], qa[ks], bf[0], bf[1]);
            mma_bf16(sc[1], qa[ks], bf[2], bf[3]);
          }
        }
        float sv[2][2], tmax = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int tp = t0 + w0 + 8 * nt + 2 * (lane & 3) + j;
            const float v = sc[nt][j] + sc[nt][2 + j];
            sv[nt][j] = tp < P ? v : -INFINITY;
            tmax = fmaxf(tmax, sv[nt][j]);
          }
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
        const float m_new = fmaxf(m_run, tmax);
        const float resc = m_new == -INFINITY ? 1.f : expf(m_run - m_new);
        uint16_t ph[2][2], pl[2][2];
        float psum = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const float p = sv[nt][j] == -INFINITY ? 0.f : expf(sv[nt][j] - m_new);
            psum += p;
            bf16_split(p, ph[nt][j], pl[nt][j]);
          }
        const uint32_t pa[4] = {pack_bf16x2(ph[0][0], ph[0][1]), pack_bf16x2(pl[0][0], pl[0][1]),
                                pack_bf16x2(ph[1][0], ph[1][1]), pack_bf16x2(pl[1][0], pl[1][1])};
        l_run = l_run * resc + psum;
        m_run = m_new;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          o[nt][0] *= resc;
          o[nt][1] *= resc;
          o[nt][2] *= resc;
          o[nt][3] *= resc;
        }
        {
          const int tt = w0 + (lane & 7) + 8 * ((lane >> 3) & 1), ch = lane >> 4;
#pragma unroll
          for (int np = 0; np < 8; ++np) {
            uint32_t bf[4];
            ldsm_x4_t(kv_tile_addr(vb, tt, 2 * np + ch), bf);
            mma_bf16(o[2 * np], pa, bf[0], bf[1]);
            mma_bf16(o[2 * np + 1], pa, bf[2], bf[3]);
          }
        }
      }
      c.release();
    }
    // merge the 8 warps' partials of this head group and write the CTA's split
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    if ((lane & 3) == 0) {
      s_m[warp][g] = m_run;
      s_l[warp][g] = l_run;
    }
    if (g < G) {
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const int d = 8 * nt + 2 * (lane & 3);
        ro[(warp * G + g) * kHeadDim + d] = o[nt][0] + o[nt][2];
        ro[(warp * G + g) * kHeadDim + d + 1] = o[nt][1] + o[nt][3];
      }
    }
    consumers_sync(kNCons);
    const int slot = i0;  // the head's first tile in this CTA
    for (int idx = threadIdx.x; idx < G * kHeadDim; idx += kNCons) {
      const int gg = idx / kHeadDim, d = idx - gg * kHeadDim;
      float M = -INFINITY;
#pragma unroll
      for (int ww = 0; ww < kNC; ++ww) M = fmaxf(M, s_m[ww][gg]);
      float os = 0.f, ls = 0.f;
#pragma unroll
      for (int ww = 0; ww < kNC; ++ww) {
        const float f = s_m[ww][gg] == -INFINITY ? 0.f : expf(s_m[ww][gg] - M);
        os = fmaf(f, ro[(ww * G + gg) * kHeadDim + d], os);
        ls = fmaf(f, s_l[ww][gg], ls);
      }
      const size_t pi = ((size_t)b * a.H + (size_t)kvh * G + gg) * a.nchunk + slot;
      a.part_o[pi * kHeadDim + d] = os;
      if (d == 0) {
        a.part_ml[pi * 2 + 0] = M;
        a.part_ml[pi * 2 + 1] = ls;
      }
    }
    u = useg;
  }
}

template <int NB>
__global__ void __launch_bounds__(kThreads, 1)
    k_block_persistent(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                       const BpArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* xsb = smem + a.xs_off;
  float4* xs = reinterpret_cast<float4*>(xsb);
  float* res = reinterpret_cast<float*>(smem + a.res_off);
  __shared__ uint64_t full[kMaxQ], empty[kMaxQ], st_start[kMaxQ];
  __shared__ float s_red[kNC][2], s_rstd[2];
  __shared__ float s_m[kNC][8], s_l[kNC][8];

  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxQ; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kNC);
    }
    mbar_init_fence();
  }
  __syncthreads();

  if (warp == kNC) {
    // ------------------------------------------------------------ producer warp
    if ((threadIdx.x & 31) == 0) {
      Producer pr{smem, a.ring_bytes, full, empty, st_start, 0ull, 0u, 0, 0, a.err, l2_evict_first()};
      bool ok = pr.norm_inputs(a.x, a.nb, a.D, a.attn_norm);
      if (ok) ok = pr.gemv<EPI_QKV>(a.g[PH_QKV]);
      if (ok) ok = produce_attn(pr, a, &mK, &mV);
      if (ok) ok = pr.gemv<EPI_PLAIN>(a.g[PH_WO]);
      if (ok) ok = pr.norm_inputs(nullptr, 0, a.D, a.ffn_norm);
      if (ok) ok = pr.gemv<EPI_SWIGLU>(a.g[PH_W13]);
      if (ok) pr.gemv<EPI_PLAIN>(a.g[PH_W2]);
      stamp(a, 12);
    }
    return;  // the consumers synchronise among themselves from here on
  }

  Consumer c{smem, a.ring_bytes, full, empty, 0ull, 0u, 0, true, a.err, 0ull, false};
  int R0, nrows;
  const bool tr = a.trace && threadIdx.x == 0;
  c.timed = tr;
  if (tr) stamp(a, 0);

  // ---------------------------------------------------------------- A: q/k/v
  {
    const BpGemv& g = a.g[PH_QKV];
    const uint32_t in_off = c.next(round1k((uint32_t)(a.nb + 1) * a.D * 4));
    const float* xin = reinterpret_cast<const float*>(c.ring + in_off);
    consume_gemv<NB, EPI_QKV>(c, g, xs, res, R0, nrows, [&](int, bool publish) {
      stage_norm<NB>(a, xs, xin, false, xin + (size_t)a.nb * a.D, nullptr, publish, s_red, s_rstd);
    }, true);
    for (int tt = threadIdx.x; tt < (nrows >> 1) * NB; tt += kNCons) {
      const int pr = tt / NB, b = tt - pr * NB;
      if (b >= a.nb) continue;
      float y0, y1;
      pair_sums<NB>(res, g.split, pr, b, y0, y1);
      int mat, lrow;
      row_of<EPI_QKV>(g, R0 + 2 * pr, mat, lrow);
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
        *reinterpret_cast<float2*>(a.q + (size_t)b * a.QD + lrow) = make_float2(y0, y1);
      } else {
        uint16_t* cache = mat == 1 ? a.kc : a.vc;
        const size_t o = (((size_t)b * a.Hkv + head) * a.max_seq + pos) * kHeadDim + d;
        *reinterpret_cast<uint32_t*>(cache + o) =
            (uint32_t)f32_to_bf16_bits(y0) | ((uint32_t)f32_to_bf16_bits(y1) << 16);
      }
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");  // the cache rows are read by TMA
  }
  if (tr) stamp(a, 1);
  grid_barrier(a.bar, 1, a.err);
  if (tr) stamp(a, 2);

  // ---------------------------------------------------------------- B: attention
  AttnWork w;
  attn_work(a, w);
  consume_attn<NB>(c, a, w, xsb, s_m, s_l);
  if (tr) stamp(a, 3);
  grid_barrier(a.bar, 2, a.err);
  if (tr) stamp(a, 4);

  // ---------------------------------------------------------------- C: W_O partials
  {
    const BpGemv& g = a.g[PH_WO];
    consume_gemv<NB, EPI_PLAIN>(c, g, xs, res, R0, nrows, [&](int seg, bool publish) {
      stage_att<NB>(a, w, seg, g.Ks, publish, xs);
    });
    for (int tt = threadIdx.x; tt < (nrows >> 1) * NB; tt += kNCons) {
      const int pr = tt / NB, b = tt - pr * NB;
      if (b >= a.nb) continue;
      float y0, y1;
      pair_sums<NB>(res, g.split, pr, b, y0, y1);
      const int gr = R0 + 2 * pr, seg = gr / g.rps, lrow = gr - seg * g.rps;
      *reinterpret_cast<float2*>(a.part + ((size_t)seg * a.nb + b) * a.D + lrow) = make_float2(y0, y1);
    }
  }
  if (tr) stamp(a, 5);
  grid_barrier(a.bar, 3, a.err);
  if (tr) stamp(a, 6);

  // ------------------------------------------------ merge of the W_O partials
  // x_mid = x + sum_s sync(W_O partial_s), each 128-value chunk once, with its
  // sum of squares for the RMSNorm
  merge_rows(a, a.x, a.xmid, a.ssq);
  grid_barrier(a.bar, 4, a.err);
  if (tr) stamp(a, 13);

  // ---------------------------------------------------------------- D: W1/W3 + SwiGLU
  {
    const BpGemv& g = a.g[PH_W13];
    c.waited = 0;
    const uint32_t in_off = c.next(round1k((uint32_t)a.D * 4));  // the gain
    const float* gin = reinterpret_cast<const float*>(c.ring + in_off);
    consume_gemv<NB, EPI_SWIGLU>(c, g, xs, res, R0, nrows, [&](int, bool publish) {
      stage_norm<NB>(a, xs, a.xmid, true, gin, a.ssq, publish, s_red, s_rstd);
      if (tr) stamp(a, 14);
    }, true);
    if (tr) a.trace[(size_t)blockIdx.x * TP_BLOCK_TRACE_SLOTS + 15] = c.waited;
    for (int tt = threadIdx.x; tt < (nrows >> 1) * NB; tt += kNCons) {
      const int pr = tt / NB, b = tt - pr * NB;
      if (b >= a.nb) continue;
      float y0, y1;
      pair_sums<NB>(res, g.split, pr, b, y0, y1);
      const int f = (R0 + 2 * pr) >> 1;
      a.h[(size_t)b * a.F + f] = y0 / (1.0f + expf(-y0)) * y1;
    }
  }
  if (tr) stamp(a, 7);
  grid_barrier(a.bar, 5, a.err);
  if (tr) stamp(a, 8);

  // ---------------------------------------------------------------- E: W2 partials
  {
    const BpGemv& g = a.g[PH_W2];
    consume_gemv<NB, EPI_PLAIN>(c, g, xs, res, R0, nrows, [&](int seg, bool) {
      stage_plain<NB>(a.h, a.F, a.nb, seg, g.Ks, xs);
    });
    for (int tt = threadIdx.x; tt < (nrows >> 1) * NB; tt += kNCons) {
      const int pr = tt / NB, b = tt - pr * NB;
      if (b >= a.nb) continue;
      float y0, y1;
      pair_sums<NB>(res, g.split, pr, b, y0, y1);
      const int gr = R0 + 2 * pr, seg = gr / g.rps, lrow = gr - seg * g.rps;
      *reinterpret_cast<float2*>(a.part + ((size_t)seg * a.nb + b) * a.D + lrow) = make_float2(y0, y1);
    }
  }
  if (tr) stamp(a, 9);
  grid_barrier(a.bar, 6, a.err);
  if (tr) stamp(a, 10);

  // ---------------------------------------------------------------- F: final merge
  merge_rows(a, a.xmid, a.x, nullptr);  // x = x_mid + sum_s sync(W2 partial_s)

  // the last CTA out puts the barrier counters back to zero for the next launch
  consumers_sync(kNCons);
  if (tr) stamp(a, 11);
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(a.bar + 1, 1u) == gridDim.x - 1) {
      atomicExch(a.bar, 0u);
      atomicExch(a.bar + 1, 0u);
    }
  }
}


// Rows per stage for a phase: the most row pairs (16, 8, 4, 2, 1) whose stage
// stays within a third of the ring, so that at least three stages are in
// flight; 16 pairs give each warp two pairs, fewer are split over 8 / pairs
// warps each.
bool plan_phase(BpGemv& g, uint32_t max_stage) {
  const uint32_t rb = (uint32_t)g.Ks * 2;
  for (int P = 16; P >= 1; P >>= 1) {
    if ((uint32_t)(2 * P) * rb <= max_stage) {
      g.pairs = P;
      g.split = P >= 8 ? 1 : 8 / P;
      g.pw = P == 16 ? 2 : 1;
      return true;
    }
  }
  return false;
}

}  // namespace

// Shared-memory plan: ring | activations (also the attention merge area) |
// per-row partial sums. Returns false when the shapes do not fit, in which case
// the caller runs the multi-kernel path.
// The persistent kernel is opt-in (TP_PERSISTENT=1, or per handle) until it is
// faster than the kernel-per-step path on every shape it takes.
bool persistent_default() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("TP_PERSISTENT");
    v = (e && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

bool plan_block_persistent(BpArgs& a, int nb_max) {
  if (nb_max < 1 || nb_max > 2 || a.n < 1) return false;
  if (a.n > kMaxSlices || a.H / a.Hkv > 8 || a.QD / a.n / kHeadDim > kMaxSegHeads) return false;
  // every CTA gets at least one row pair of every phase (so that the owner of
  // each segment's first row, which publishes its activations, exists)
  int grid = num_sms();
  int kmax = 0;
  for (int p = 0; p < 4; ++p) {
    const int npairs = a.g[p].nseg * (a.g[p].rps >> 1);
    grid = npairs < grid ? npairs : grid;
    kmax = a.g[p].Ks > kmax ? a.g[p].Ks : kmax;
  }
  if (grid < 1) return false;
  const uint32_t xs_bytes = (uint32_t)nb_max * (uint32_t)kmax * 4u;  // NB rows of Ks floats
  // attention: the warps' partials [8][G][128] floats, then Q; the split combine
  // reuses the partials' area
  const uint32_t G = (uint32_t)(a.H / a.Hkv);
  const uint32_t merge_bytes = kNC * G * kHeadDim * 4u;
  uint32_t xs_region = xs_bytes > merge_bytes + kQsBytes ? xs_bytes : merge_bytes + kQsBytes;
  xs_region = (xs_region + 1023u) & ~1023u;
  uint32_t res_bytes = 0;  // per-row partial sums, bounded by the widest split (8)
  for (int p = 0; p < 4; ++p) {
    const int npairs = a.g[p].nseg * (a.g[p].rps >> 1);
    const uint32_t rows = 2u * (uint32_t)((npairs + grid - 1) / grid);
    const uint32_t r = rows * (uint32_t)nb_max * 8u * 4u;
    res_bytes = r > res_bytes ? r : res_bytes;
  }
  res_bytes = (res_bytes + 1023u) & ~1023u;
  // 227 KB per CTA, less the 1 KB alignment pad and the static shared arrays
  const uint32_t limit = 227u * 1024u - 1024u - 4096u;
  if (xs_region + res_bytes + 128u * 1024u > limit) return false;
  const uint32_t ring = (limit - xs_region - res_bytes) & ~1023u;
  for (int p = 0; p < 4; ++p)
    if (!plan_phase(a.g[p], ring / 3)) return false;
  if (kTileBytes > ring / 3 || (uint32_t)(nb_max + 1) * a.D * 4u > ring / 3) return false;
  a.grid = grid;
  a.ring_bytes = ring;
  a.xs_off = ring;
  a.res_off = ring + xs_region;
  a.smem_total = 1024 + ring + xs_region + res_bytes;
  return true;
}

int launch_block_persistent(const BpArgs& a, int nb_max, cudaStream_t s) {
  CUtensorMap mK, mV;
  const uint64_t rows = (uint64_t)a.nb * a.Hkv * a.max_seq;
  if (!make_tensor_map_2d(&mK, a.kc, rows, kHeadDim, kHeadDim, 64, kTileP) ||
      !make_tensor_map_2d(&mV, a.vc, rows, kHeadDim, kHeadDim, 64, kTileP))
    return TP_ECUDA;
  const void* fn = nb_max == 2 ? (const void*)k_block_persistent<2> : (const void*)k_block_persistent<1>;
  if (set_smem_once(fn, (int)a.smem_total)) return TP_ECUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = a.smem_total;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = nb_max == 2 ? cudaLaunchKernelEx(&cfg, k_block_persistent<2>, mK, mV, a)
                              : cudaLaunchKernelEx(&cfg, k_block_persistent<1>, mK, mV, a);
  return e == cudaSuccess ? TP_OK : TP_ECUDA;
}

}  // namespace tp
