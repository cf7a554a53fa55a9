// Weight-streaming slice GEMV for decode (batch 1 or 2 per launch).
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
// Structure (one persistent CTA per SM). The rows of all segments form one list
// of row pairs (a RoPE pair of q/k, row f of W1 with row f of W3, or two
// consecutive rows); every CTA owns a contiguous, equal share of the pairs, so
// every SM streams the same bytes. A producer warp copies the CTA's rows into a
// ring of shared-memory stages with bulk asynchronous copies (cp.async.bulk, L2
// evict-first: the weights are read once per step, the activations often),
// completion counted on one mbarrier per stage; a stage holds one row pair for
// each of the NC consumer warps and never crosses a segment boundary, and the
// ring keeps 100-200 KB per SM in flight. A consumer warp dots its pair with the
// activations (staged once per segment in shared memory, float32), reduces the
// two sums across the warp with shuffles, and hands the stage back with an
// mbarrier arrive. The producer only reads weights, which no kernel writes, so
// under programmatic dependent launch it starts streaming while the previous
// kernel finishes; the consumers wait for that kernel before reading the
// activations. Every mbarrier wait is bounded (2 s) and sets the error flag
// instead of hanging.
//
// Input modes: float32 activations; Q8 codes + scales (dequantised while
// staging); or the RMSNorm of a float32 residual computed while staging (each
// CTA reduces the whole row for the scale; with Q8 the normalised values pass
// through the int8 block format, and the CTA that owns the first row of a
// segment also writes the shared int8 (or float32) buffer of that segment).
//
// Epilogues (after the last stage): EPI_PLAIN stores partials or logits;
// EPI_SWIGLU stores silu(a)*b (llamaFfn); EPI_QKV applies RoPE to q and k
// pairs, stores rotated q, and writes k and v into the bf16 cache at pos
// (llamaMultiheadAtt's "merge kv-cache, add RoPE encoding").
#include <cstdlib>

#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "pipeline.cuh"

namespace tp {

namespace {

constexpr int kMaxStages = 16;
// Dynamic shared memory of a GEMV CTA. bf16: 222 KB, which leaves room on the SM for a
// merge CTA beside the row-split GEMVs (152 registers). int8 weights: 223 KB, which fits
// 3 stages of 8 row pairs for the 7B W1/W3 rows (4 KB of codes + their scales; 5,504
// bytes of activations, partial sums and barriers): 8 pairs per stage instead of 4,
// one consumer warp per pair. Its kernels take 158 registers or more, so a merge CTA
// never fits beside them anyway.
constexpr int kSmemBudget = 222 * 1024;
constexpr int kSmemBudgetQ8 = 223 * 1024;

template <int EPI>
TP_DEV int rows_per_seg(const GemvArgs& a) {
  if (EPI == EPI_SWIGLU) return 2 * a.rows[0];
  if (EPI == EPI_QKV) return a.rows[0] + a.rows[1] + a.rows[2];
  return a.rows[0];
}

// Global address of virtual row `r` of segment `seg`; mat/lrow name the matrix
// and its row (SwiGLU interleaves row f of W1 and row f of W3).
template <int EPI>
TP_DEV const uint16_t* row_ptr(const GemvArgs& a, int seg, int r, int& mat, int& lrow) {
  mat = 0;
  if (EPI == EPI_SWIGLU) {
    mat = r & 1;
    lrow = r >> 1;
  } else {
    lrow = r;
    if (EPI == EPI_QKV && lrow >= a.rows[0]) {
      lrow -= a.rows[0];
      mat = 1;
      if (lrow >= a.rows[1]) {
        lrow -= a.rows[1];
        mat = 2;
      }
    }
  }
  return a.w[mat] + (size_t)lrow * a.ldw + (size_t)seg * a.Ks;
}

// Next stage of a CTA's row range: rows [cur, end) with end - cur <= 2*P (P row
// pairs per stage) and no segment boundary inside. Producer and consumers walk
// the same sequence.
TP_DEV int stage_end(int cur, int nrows, int R0, int rps, int P) {
  const int g = R0 + cur;
  const int seg_end = (g / rps + 1) * rps - R0;
  return min(min(nrows, seg_end), cur + 2 * P);
}

// Stage bytes of one row of int8 weights beyond its codes: the 16-byte-aligned
// run of global memory that covers the row's scales (a segment's scales need
// not start on a 16-byte boundary), with room for the misalignment.
inline __host__ __device__ uint32_t q8w_scale_slot(int Ks) {
  return (((uint32_t)Ks / 32u * 4u + 15u) & ~15u) + 16u;
}

template <int NB, int PW>
TP_DEV void ring_pairs_dot_q8(const uint8_t* stage, uint32_t cstride, uint32_t soff, uint32_t sstride,
                              const int* pad, int cur, int end, const int8_t* xsq, const float* xsd,
                              float* res, int Ks, int pw, int part, int Q, int cb, int ce, int lane);

// The weight tensor map of the row-split kernels that read through one (MAP); the
// other kernels take an empty parameter, so their launches carry no descriptor.
template <bool MAP>
struct WeightMap {
  CUtensorMap m;
};
template <>
struct WeightMap<false> {};

// PW: row pairs per consumer warp and stage (GemvPlan::pw), a template parameter so
// that each kernel's streaming loop holds only the dot-product variant it runs
template <int NB, int EPI, bool WQ8, int PW, bool MAP = false>
__global__ void __launch_bounds__(288, 1) k_gemv(GemvArgs a, GemvPlan pl,
                                                  const __grid_constant__ WeightMap<MAP> wmap) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_rstd[NB];
  __shared__ float s_red[8][NB];
  const int nc = pl.nc, nstage = pl.nstage, P = pl.pairs, Q = pl.split;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = a.Ks >> 3;  // 8-element vectors per row
  const uint32_t row_bytes = WQ8 ? (uint32_t)a.Ks : (uint32_t)a.Ks * 2;  // weight bytes of a row
  const uint32_t slot = WQ8 ? row_bytes + q8w_scale_slot(a.Ks) : row_bytes;  // stage bytes of a row
  uint8_t* ring = smem + pl.ring_off;
  float4* xs = reinterpret_cast<float4*>(smem + pl.x_off);  // lo[NB][nv] then hi[NB][nv]
  // int8 weights: the activations as Q8 codes [NB][Ks] and scales [NB][Ks / 32]
  int8_t* xsq = reinterpret_cast<int8_t*>(smem + pl.x_off);
  float* xsd = reinterpret_cast<float*>(smem + pl.x_off + (size_t)NB * a.Ks);
  float* res = reinterpret_cast<float*>(smem + pl.res_off);  // [rows of this CTA][NB]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + pl.bar_off);
  uint64_t* empty = full + kMaxStages;

  const int rps = rows_per_seg<EPI>(a);
  const int npairs = a.nseg * (rps >> 1);
  const int P0 = (int)(((int64_t)npairs * blockIdx.x) / gridDim.x);
  const int P1 = (int)(((int64_t)npairs * (blockIdx.x + 1)) / gridDim.x);
  const int R0 = 2 * P0, nrows = 2 * (P1 - P0);  // flattened rows [R0, R0 + nrows)

  if (threadIdx.x == 0) {
    for (int s = 0; s < nstage; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], nc);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  pdl_launch_dependents();
  unsigned long long* tr = a.trace ? a.trace + (size_t)blockIdx.x * a.trace_stride : nullptr;
  if (tr && threadIdx.x == 0) tr[0] = gtimer();

  if (warp == nc) {
    // ---------------------------------------------------------------- producer
    // (bf16 weights: lane 0 issues the copies; int8 weights, whose rows take two
    // small copies each, spread them over the warp's lanes)
    // the RMSNorm gain (a constant input: no wait) into L2 before the weights, for the
    // consumers' prologue
    if (a.gain && lane == 0) bulk_prefetch_l2(a.gain, (uint32_t)a.ldx * 4);
    if constexpr (MAP) {  // the weight map's descriptor, early
      if (lane == 0)
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&wmap.m)) : "memory");
    }
    if (WQ8 || lane == 0) {
      const uint64_t pol = l2_evict_first();  // weights are read once per step
      int t = 0;
      for (int cur = 0; cur < nrows; ++t) {
        const int end = stage_end(cur, nrows, R0, rps, P);
        const int s = t % nstage;
        const uint32_t ph = (uint32_t)(t / nstage) & 1u;
        bool waited = mbar_wait(&empty[s], ph ^ 1u, a.err);
        if (WQ8) waited = __all_sync(0xffffffffu, waited);
        if (!waited) break;
        uint8_t* dst = ring + (size_t)s * 2 * P * slot;
        // one division per stage; rows are then walked with pointer increments
        const int seg = (R0 + cur) / rps;
        const int lr0 = R0 + cur - seg * rps;
        const int n = end - cur;
        const size_t col0 = (size_t)seg * a.Ks;
        if constexpr (WQ8) {
          // per row: its codes, then the aligned run covering its scales; with the weight
          // map, the stage's codes in boxes of map_box rows (first, dense) and the rows'
          // scale runs after them
          const size_t sstride = (size_t)(a.ldw / 32) * 4, sseg = (size_t)seg * (a.Ks / 32) * 4;
          const uint32_t sbytes = (uint32_t)(a.Ks / 32) * 4;
          uint32_t tx = 0;
          for (int i = lane; i < n; i += 32) {
            int mat, lrow;
            row_ptr<EPI>(a, seg, lr0 + i, mat, lrow);
            const size_t s0 = (size_t)lrow * sstride + sseg;
            tx += (MAP ? 0u : row_bytes) +
                  (uint32_t)(((s0 + sbytes + 15) & ~(size_t)15) - (s0 & ~(size_t)15));
          }
          tx = __reduce_add_sync(0xffffffffu, tx);
          const int nbox = MAP ? (n + pl.map_box - 1) / pl.map_box : 0;
          if (lane == 0) mbar_expect_tx(&full[s], tx + (uint32_t)(nbox * pl.map_box) * row_bytes);
          __syncwarp();
          if constexpr (MAP) {
            if (lane == 0)
              for (int k = 0; k < nbox; ++k)
                tma_load_3d_hint(dst + (size_t)k * pl.map_box * row_bytes, &wmap.m, 0,
                                 seg * pl.map_nchunk, lr0 + k * pl.map_box, &full[s], pol);
          }
          uint8_t* sdst = MAP ? dst + (size_t)2 * P * row_bytes : dst + row_bytes;
          const uint32_t sstep = MAP ? slot - row_bytes : slot;
          for (int i = lane; i < n; i += 32) {
            int mat, lrow;
            row_ptr<EPI>(a, seg, lr0 + i, mat, lrow);
            if (!MAP) {
              const int8_t* src = reinterpret_cast<const int8_t*>(a.w[mat]) + (size_t)lrow * a.ldw + col0;
              bulk_g2s_hint(dst + (size_t)i * slot, src, row_bytes, &full[s], pol);
            }
            const size_t s0 = (size_t)lrow * sstride + sseg, slo = s0 & ~(size_t)15;
            const uint32_t sl = (uint32_t)(((s0 + sbytes + 15) & ~(size_t)15) - slo);
            bulk_g2s_hint(sdst + (size_t)i * sstep, reinterpret_cast<const uint8_t*>(a.wd[mat]) + slo, sl,
                          &full[s], pol);
          }
          cur = end;
          continue;
        }
        if constexpr (MAP) {
          // whole boxes of map_box rows (a short last box reads a few rows past the
          // CTA's range, or zeros past the matrix; the stage holds them)
          const int nbox = (n + pl.map_box - 1) / pl.map_box;
          mbar_expect_tx(&full[s], (uint32_t)(nbox * pl.map_box) * row_bytes);
          for (int i = 0; i < nbox; ++i)
            tma_load_3d_hint(dst + (size_t)i * pl.map_box * row_bytes, &wmap.m, 0,
                             seg * pl.map_nchunk, lr0 + i * pl.map_box, &full[s], pol);
          cur = end;
          continue;
        }
        mbar_expect_tx(&full[s], (uint32_t)(end - cur) * row_bytes);
        if (EPI == EPI_SWIGLU) {  // rows alternate W1[f], W3[f]
          const uint16_t* p1 = a.w[0] + (size_t)(lr0 >> 1) * a.ldw + col0;
          const uint16_t* p3 = a.w[1] + (size_t)(lr0 >> 1) * a.ldw + col0;
          for (int i = 0; i < n; i += 2) {
            bulk_g2s_hint(dst + (size_t)i * row_bytes, p1, row_bytes, &full[s], pol);
            bulk_g2s_hint(dst + (size_t)(i + 1) * row_bytes, p3, row_bytes, &full[s], pol);
            p1 += a.ldw;
            p3 += a.ldw;
          }
        } else {  // runs of rows inside one matrix; one copy per run when rows are contiguous
          int done = 0, r = lr0;
          while (done < n) {
            int mat, lrow;
            const uint16_t* src = row_ptr<EPI>(a, seg, r, mat, lrow);
            int mat_end = a.rows[0];
            if (EPI == EPI_QKV) mat_end = mat == 0 ? a.rows[0] : (mat == 1 ? a.rows[0] + a.rows[1] : rps);
            const int run = min(n - done, mat_end - r);
            if (a.ldw == a.Ks) {
              bulk_g2s_hint(dst + (size_t)done * row_bytes, src, (uint32_t)run * row_bytes, &full[s], pol);
            } else {
              for (int i = 0; i < run; ++i, src += a.ldw)
                bulk_g2s_hint(dst + (size_t)(done + i) * row_bytes, src, row_bytes, &full[s], pol);
            }
            done += run;
            r += run;
          }
        }
        cur = end;
      }
    }
    pdl_wait();  // the epilogue below writes buffers earlier kernels may read
  } else {
    // ---------------------------------------------------------------- consumers
    const int ncons = nc * 32;
    // RMSNorm input with one segment (q/k/v, W1/W3 in 1D), one batch row per launch:
    // each consumer thread loads the x and gain values of its vectors (8 values,
    // v = thread + 256 k) once, up front, for the scale and the staging both: one
    // round of loads, not two (two rows would spill registers)
    constexpr int kPreV = 2;
    const bool pre = NB == 1 && a.gain && a.nseg == 1 && nc == 8 && nv <= kPreV * 256;
    float4 px[NB][kPreV][2], pg[kPreV][2];
    // The staging of the preloaded row (one segment, one batch row): RMSNorm, and the Q8
    // round trip, of the thread's two vectors v = thread and v = thread + 256 side by side
    // (zeros past the row); the same values, codes and shared-buffer writes as `stage`.
    auto stage_pre = [&](bool publish) {
      float xv[2][8], am[2], d[2], r[2], cf[2][8];
      const float rstd = s_rstd[0];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float4 x0 = px[0][k][0], x1 = px[0][k][1], g0 = pg[k][0], g1 = pg[k][1];
        xv[k][0] = __fmul_rn(__fmul_rn(x0.x, rstd), g0.x);
        xv[k][1] = __fmul_rn(__fmul_rn(x0.y, rstd), g0.y);
        xv[k][2] = __fmul_rn(__fmul_rn(x0.z, rstd), g0.z);
        xv[k][3] = __fmul_rn(__fmul_rn(x0.w, rstd), g0.w);
        xv[k][4] = __fmul_rn(__fmul_rn(x1.x, rstd), g1.x);
        xv[k][5] = __fmul_rn(__fmul_rn(x1.y, rstd), g1.y);
        xv[k][6] = __fmul_rn(__fmul_rn(x1.z, rstd), g1.z);
        xv[k][7] = __fmul_rn(__fmul_rn(x1.w, rstd), g1.w);
        const int v = threadIdx.x + 256 * k;
        if (publish && v < nv && a.xn_out) {
          float* dst = a.xn_out + (size_t)a.b0 * a.ldx + 8 * (size_t)v;
          *reinterpret_cast<float4*>(dst) = make_float4(xv[k][0], xv[k][1], xv[k][2], xv[k][3]);
          *reinterpret_cast<float4*>(dst + 4) = make_float4(xv[k][4], xv[k][5], xv[k][6], xv[k][7]);
        }
      }
      if (WQ8 || a.quant) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          am[k] = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) am[k] = fmaxf(am[k], fabsf(xv[k][e]));
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) am[k] = fmaxf(am[k], __shfl_xor_sync(0xffffffffu, am[k], 1));
#pragma unroll
        for (int k = 0; k < 2; ++k) am[k] = fmaxf(am[k], __shfl_xor_sync(0xffffffffu, am[k], 2));
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          d[k] = q8_scale(am[k]);
          r[k] = q8_recip(d[k]);
        }
        q8_codes_g<8, 2>(&xv[0][0], &cf[0][0], d, r);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int v = threadIdx.x + 256 * k;
          uint32_t lo = 0, hi = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            xv[k][e] = __fmul_rn(cf[k][e], d[k]);
            const uint32_t c = (uint32_t)((int)cf[k][e] & 0xFF);
            if (e < 4) lo |= c << (8 * e);
            else hi |= c << (8 * (e - 4));
          }
          const size_t e0 = (size_t)a.b0 * a.ldx + 8 * (size_t)v;
          if (publish && v < nv && a.xq_out) {
            *reinterpret_cast<uint2*>(a.xq_out + e0) = make_uint2(lo, hi);
            if ((lane & 3) == 0) a.xd_out[e0 / kQ8Block] = d[k];
          }
          if (WQ8 && v < nv) {
            *reinterpret_cast<uint2*>(xsq + 8 * (size_t)v) = make_uint2(lo, hi);
            if ((v & 3) == 0) xsd[v >> 2] = d[k];
          }
        }
      }
      if (!WQ8) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int v = threadIdx.x + 256 * k;
          if (v < nv) {
            xs[v] = make_float4(xv[k][0], xv[k][1], xv[k][2], xv[k][3]);
            xs[NB * nv + v] = make_float4(xv[k][4], xv[k][5], xv[k][6], xv[k][7]);
          }
        }
      }
    };
    // (re)stage the activations of segment `seg`; whole warps per iteration so that 4
    // consecutive lanes always hold one 32-value Q8 block. publish: this CTA owns the
    // segment's first row and writes the shared buffers.
    auto stage_segment = [&](int seg, bool publish) {
      const size_t col0 = (size_t)seg * a.Ks;
      const int nvr = (nv + 31) & ~31;
      consumers_sync(ncons);
      // one 8-value vector v of batch row b (x, g: the preloaded values when have_pre)
      auto stage = [&](int b, int v, bool have_pre, float4 px0, float4 px1, float4 pg0,
                       float4 pg1) {
          const bool in = b < a.nb && v < nv;
          const size_t e0 = (size_t)(a.b0 + b) * a.ldx + col0 + 8 * (size_t)v;
          float xv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          uint2 qin = make_uint2(0u, 0u);  // codes as read (Q8 input)
          float din = 0.f;
          if (in) {
            if (a.gain) {
              const float rstd = s_rstd[b];
              const float4 x0 = have_pre ? px0 : *reinterpret_cast<const float4*>(a.x + e0);
              const float4 x1 = have_pre ? px1 : *reinterpret_cast<const float4*>(a.x + e0 + 4);
              const float4 g0 =
                  have_pre ? pg0 : *reinterpret_cast<const float4*>(a.gain + col0 + 8 * (size_t)v);
              const float4 g1 = have_pre ? pg1
                                         : *reinterpret_cast<const float4*>(a.gain + col0 +
                                                                            8 * (size_t)v + 4);
              xv[0] = __fmul_rn(__fmul_rn(x0.x, rstd), g0.x);
              xv[1] = __fmul_rn(__fmul_rn(x0.y, rstd), g0.y);
              xv[2] = __fmul_rn(__fmul_rn(x0.z, rstd), g0.z);
              xv[3] = __fmul_rn(__fmul_rn(x0.w, rstd), g0.w);
              xv[4] = __fmul_rn(__fmul_rn(x1.x, rstd), g1.x);
              xv[5] = __fmul_rn(__fmul_rn(x1.y, rstd), g1.y);
              xv[6] = __fmul_rn(__fmul_rn(x1.z, rstd), g1.z);
              xv[7] = __fmul_rn(__fmul_rn(x1.w, rstd), g1.w);
            } else if (a.att_po) {
              // the attention output of these 8 dims, combined from the context splits:
              // M = max_c m_c, o = sum_c e^{m_c - M} o_c / sum_c e^{m_c - M} l_c
              const int gb = a.b0 + b;
              const int P = a.pos[gb] + 1, ntiles = (P + 63) / 64;
              const int tpc = (ntiles + a.att_nsplit - 1) / a.att_nsplit;
              const int ncs = (ntiles + tpc - 1) / tpc;
              const int col = (int)col0 + 8 * v, h = col / kHeadDim, d0 = col - h * kHeadDim;
              const size_t base = ((size_t)gb * a.n_heads + h) * a.att_nsplit;
              // the splits' (m, l) in one round of loads, then their outputs 4 splits
              // at a time (the same sums, in split order)
              constexpr int kCm = 8;
              float mcs[kCm], lcs[kCm];
#pragma unroll
              for (int c = 0; c < kCm; ++c) {
                mcs[c] = c < ncs ? a.att_pml[(base + c) * 2] : -INFINITY;
                lcs[c] = c < ncs ? a.att_pml[(base + c) * 2 + 1] : 0.f;
              }
              float M = -INFINITY;
              for (int c = kCm; c < ncs; ++c) M = fmaxf(M, a.att_pml[(base + c) * 2]);
#pragma unroll
              for (int c = 0; c < kCm; ++c) M = fmaxf(M, mcs[c]);
              float L = 0.f;
              auto add_split = [&](float mc, float lc, float4 o0, float4 o1) {
                const float w = mc == -INFINITY ? 0.f : expf(mc - M);
                L = fmaf(w, lc, L);
                xv[0] = fmaf(w, o0.x, xv[0]); xv[1] = fmaf(w, o0.y, xv[1]);
                xv[2] = fmaf(w, o0.z, xv[2]); xv[3] = fmaf(w, o0.w, xv[3]);
                xv[4] = fmaf(w, o1.x, xv[4]); xv[5] = fmaf(w, o1.y, xv[5]);
                xv[6] = fmaf(w, o1.z, xv[6]); xv[7] = fmaf(w, o1.w, xv[7]);
              };
#pragma unroll
              for (int c0 = 0; c0 < kCm; c0 += 4) {
                if (c0 >= ncs) break;
                float4 o[4][2];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const float* op = a.att_po + (base + c0 + j) * kHeadDim + d0;
                  const bool cin = c0 + j < ncs;
                  o[j][0] = cin ? *reinterpret_cast<const float4*>(op) : make_float4(0.f, 0.f, 0.f, 0.f);
                  o[j][1] = cin ? *reinterpret_cast<const float4*>(op + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  if (c0 + j < ncs) add_split(mcs[c0 + j], lcs[c0 + j], o[j][0], o[j][1]);
              }
              for (int c = kCm; c < ncs; ++c) {  // beyond 8 splits: one at a time
                const float* op = a.att_po + (base + c) * kHeadDim + d0;
                add_split(a.att_pml[(base + c) * 2], a.att_pml[(base + c) * 2 + 1],
                          *reinterpret_cast<const float4*>(op), *reinterpret_cast<const float4*>(op + 4));
              }
#pragma unroll
              for (int e = 0; e < 8; ++e) xv[e] = xv[e] / L;
              if (publish && a.att_out) {
                float* dst = a.att_out + (size_t)gb * a.ldx + col;
                *reinterpret_cast<float4*>(dst) = make_float4(xv[0], xv[1], xv[2], xv[3]);
                *reinterpret_cast<float4*>(dst + 4) = make_float4(xv[4], xv[5], xv[6], xv[7]);
              }
            } else if (a.xq) {
              const uint2 c = *reinterpret_cast<const uint2*>(a.xq + e0);
              const float d = a.xd[e0 / kQ8Block];
              qin = c;
              din = d;
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
          // the normalised value before any Q8 round trip (float32 RMSNorm output)
          if (a.gain && publish && in && a.xn_out) {
            *reinterpret_cast<float4*>(a.xn_out + e0) = make_float4(xv[0], xv[1], xv[2], xv[3]);
            *reinterpret_cast<float4*>(a.xn_out + e0 + 4) =
                make_float4(xv[4], xv[5], xv[6], xv[7]);
          }
          if (WQ8) {
            // the integer products need Q8 activations: the codes read, or those of xv
            uint2 qc = qin;
            float qd = din;
            if (!a.xq || a.gain) {
              float am = 0.f;
#pragma unroll
              for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(xv[e]));
              am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
              am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
              qd = q8_scale(am);
              float cf[8];
              q8_codes<8>(xv, cf, qd, q8_recip(qd));
              qc = make_uint2(0u, 0u);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                xv[e] = __fmul_rn(cf[e], qd);
                const uint32_t c = (uint32_t)((int)cf[e] & 0xFF);
                if (e < 4) qc.x |= c << (8 * e);
                else qc.y |= c << (8 * (e - 4));
              }
              if (a.gain && publish && in && a.xq_out) {
                *reinterpret_cast<uint2*>(a.xq_out + e0) = qc;
                if ((lane & 3) == 0) a.xd_out[e0 / kQ8Block] = qd;
              }
            }
            if (v < nv) {
              *reinterpret_cast<uint2*>(xsq + (size_t)b * a.Ks + 8 * (size_t)v) = qc;
              if ((v & 3) == 0) xsd[(size_t)b * (a.Ks / 32) + (v >> 2)] = qd;
            }
          } else if (a.gain && a.quant) {
            float am = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(xv[e]));
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
            const float d = q8_scale(am);
            float cf[8];  // the codes as integral floats; integers only where they are stored
            q8_codes<8>(xv, cf, d, q8_recip(d));
#pragma unroll
            for (int e = 0; e < 8; ++e) xv[e] = __fmul_rn(cf[e], d);
            if (publish && in && a.xq_out) {
              uint32_t lo = 0, hi = 0;
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const uint32_t c = (uint32_t)((int)cf[e] & 0xFF);
                if (e < 4) lo |= c << (8 * e);
                else hi |= c << (8 * (e - 4));
              }
              *reinterpret_cast<uint2*>(a.xq_out + e0) = make_uint2(lo, hi);
              if ((lane & 3) == 0) a.xd_out[e0 / kQ8Block] = d;
            }
          }
          if (!WQ8 && v < nv) {
            xs[b * nv + v] = make_float4(xv[0], xv[1], xv[2], xv[3]);
            xs[(NB + b) * nv + v] = make_float4(xv[4], xv[5], xv[6], xv[7]);
          }
      };
      // q/k/v and W1/W3 over bf16 weights: the two-wide form when preloaded. Measured on
      // the 7B block: RMSNorm scale -> staged 1.3-1.5 us instead of 1.8-2.6 us, the 32-layer
      // step 3.293 against 3.307 ms; the int8-weight block was 0.3 us slower with it
      if constexpr (EPI != EPI_PLAIN && !WQ8) {
        if (pre) {
          stage_pre(publish);
          consumers_sync(ncons);
          return;
        }
      }
      // one call site of `stage` (its code is large): the preloaded registers of vector
      // k = 0, 1 are picked by selects, not by a second, unrolled copy of the loop
      for (int b = 0; b < NB; ++b) {
        int k = 0;
#pragma unroll 1
        for (int v = threadIdx.x; v < nvr; v += ncons, ++k) {
          const bool hp = pre && k < kPreV;
          const int b1 = NB == 1 ? 0 : b;
          stage(b, v, hp, k == 0 ? px[b1][0][0] : px[b1][1][0], k == 0 ? px[b1][0][1] : px[b1][1][1],
                k == 0 ? pg[0][0] : pg[1][0], k == 0 ? pg[0][1] : pg[1][1]);
        }
      }
      consumers_sync(ncons);
    };

    pdl_wait();  // activations / residual come from the previous kernel
    if (tr && threadIdx.x == 0) tr[1] = gtimer();
    if (pre) {
#pragma unroll
      for (int k = 0; k < kPreV; ++k) {
        const int v = threadIdx.x + 256 * k;
        const bool vin = v < nv;  // past the row: zero
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        pg[k][0] = vin ? *reinterpret_cast<const float4*>(a.gain + 8 * (size_t)v) : z;
        pg[k][1] = vin ? *reinterpret_cast<const float4*>(a.gain + 8 * (size_t)v + 4) : z;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const bool in = vin && b < a.nb;
          const float* xr = a.x + (size_t)(a.b0 + b) * a.ldx + 8 * (size_t)v;
          px[b][k][0] = in ? *reinterpret_cast<const float4*>(xr) : z;
          px[b][k][1] = in ? *reinterpret_cast<const float4*>(xr + 4) : z;
        }
      }
    }
    if (a.gain && a.ssq) {  // sums of squares left by the merge that produced x
      if (warp < NB) {  // warp b: row b's parts, lanes in stride, then the butterfly
        float t = 0.f;
        if (warp < a.nb)
          for (int c = lane; c < a.ssq_parts; c += 32) t += a.ssq[(size_t)(a.b0 + warp) * a.ssq_parts + c];
        t = warp_sum(t);
        if (lane == 0) s_rstd[warp] = 1.0f / sqrtf(t / (float)a.ldx + a.eps);
      }
      consumers_sync(ncons);
    } else if (a.gain) {  // RMSNorm scale of each batch row, over the whole row
      const int D = a.ldx;
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        float ss = 0.f;
        if (pre) {
#pragma unroll
          for (int k = 0; k < kPreV; ++k)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float4 v = px[b][k][h];
              ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
            }
        } else if (b < a.nb) {
          const float4* xrow = reinterpret_cast<const float4*>(a.x + (size_t)(a.b0 + b) * D);
          for (int i = threadIdx.x; i < (D >> 2); i += ncons) {
            const float4 v = xrow[i];
            ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
          }
        }
        ss = warp_sum(ss);
        if (lane == 0) s_red[warp][b] = ss;
      }
      consumers_sync(ncons);
      if (threadIdx.x < NB) {
        float t = 0.f;
        for (int w = 0; w < nc; ++w) t += s_red[w][threadIdx.x];
        s_rstd[threadIdx.x] = 1.0f / sqrtf(t / (float)D + a.eps);
      }
      consumers_sync(ncons);
    }
    if (tr && threadIdx.x == 0) tr[2] = gtimer();  // the RMSNorm scale known
    bool ok = true;
    int t = 0;
    // this warp's share of a stage: row pair `pw` of the stage, vectors [vb, ve)
    const int pw = warp / Q, part = warp - pw * Q;
    const int vb = (nv * part) / Q, ve = (nv * (part + 1)) / Q;
    // one pass per segment of the CTA's rows: stage that segment's activations, then
    // consume its ring stages (a stage never crosses a segment boundary); the staging
    // code has this one call site, outside the streaming loop
    for (int cur = 0; cur < nrows;) {
      const int seg = (R0 + cur) / rps;
      stage_segment(seg, (R0 + cur) == seg * rps);
      if (tr && cur == 0 && threadIdx.x == 0) tr[3] = gtimer();
      const int seg_end = min(nrows, (seg + 1) * rps - R0);
      for (; cur < seg_end; ++t) {
        const int end = stage_end(cur, nrows, R0, rps, P);
        const int s = t % nstage;
        const uint32_t ph = (uint32_t)(t / nstage) & 1u;
        // after a wait gives up, keep walking the stages (so that every consumer warp
        // reaches the same named barriers) but skip the work
        if (ok && !mbar_wait(&full[s], ph, a.err)) ok = false;
        if (tr && t == 0 && threadIdx.x == 0) tr[4] = gtimer();
        if (ok) {
          const uint8_t* st = ring + (size_t)s * 2 * P * slot;
          if constexpr (WQ8) {
            // scale offset (floats) of each of the warp's rows inside its aligned run:
            // (lrow * ldw / 32 + seg * Ks / 32) mod 4. Matrix boundaries inside a
            // segment's rows are multiples of 4 rows (multiples of 128), so lrow mod 4
            // follows from the row's place in its segment (halved for W1/W3 pairs).
            int pad[2 * 2];
            const int s32 = (int)((a.ldw / 32) & 3), segpad = (int)(((size_t)seg * (a.Ks / 32)) & 3);
            const int seg_first = seg * rps - R0;  // CTA-local row where this segment starts
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int r = cur + 2 * (pw + 8 * (i >> 1)) + (i & 1);
              int lr = r - seg_first;
              if (EPI == EPI_SWIGLU) lr >>= 1;
              pad[i] = ((lr & 3) * s32 + segpad) & 3;
            }
            const int nc16 = a.Ks >> 4, cb = (nc16 * part) / Q, ce = (nc16 * (part + 1)) / Q;
            // rows as [codes | scale run] slots, or with the weight map all codes of the
            // stage first (dense rows of Ks), then the scale runs
            if constexpr (MAP)
              ring_pairs_dot_q8<NB, PW>(st, (uint32_t)a.Ks, (uint32_t)(2 * P * a.Ks), slot - (uint32_t)a.Ks,
                                        pad, cur, end, xsq, xsd, res, a.Ks, pw, part, Q, cb, ce, lane);
            else
              ring_pairs_dot_q8<NB, PW>(st, slot, row_bytes, slot, pad, cur, end, xsq, xsd, res, a.Ks, pw,
                                        part, Q, cb, ce, lane);
          } else {
            ring_pairs_dot<NB, PW>(st, cur, end, xs, res, nv, row_bytes, pw, part, Q, vb, ve, lane);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        cur = end;
      }
    }
    if (tr && threadIdx.x == 0) tr[5] = gtimer();
  }
  __syncthreads();

  // ---------------------------------------------------------------- epilogue
  for (int t = threadIdx.x; t < (nrows >> 1) * NB; t += blockDim.x) {
    const int pr = t / NB, b = t - pr * NB;
    if (b >= a.nb) continue;
    const int g = R0 + 2 * pr, seg = g / rps, lr = g - seg * rps;
    float y0 = 0.f, y1 = 0.f;
    for (int q = 0; q < pl.split; ++q) {  // the row's parts, in a fixed order
      y0 += res[((size_t)(2 * pr) * NB + b) * pl.split + q];
      y1 += res[((size_t)(2 * pr + 1) * NB + b) * pl.split + q];
    }
    int mat, lrow;
    row_ptr<EPI>(a, seg, lr, mat, lrow);
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
        const size_t sq = a.seq ? (size_t)a.seq[gb] : (size_t)gb;
        const size_t o = ((sq * a.n_kv_heads + head) * a.max_seq + pos) * kHeadDim + d;
        *reinterpret_cast<uint32_t*>(cache + o) =
            (uint32_t)f32_to_bf16_bits(y0) | ((uint32_t)f32_to_bf16_bits(y1) << 16);
      }
    }
  }
  if (tr && threadIdx.x == 0) tr[6] = gtimer();
}

// The int8-weight consumer step (see ring_pairs_dot): each row's codes are read
// 16 at a time, 16 consecutive bytes per lane (conflict-free), against the
// activation codes with four dp4a; the integer sum of a half block is scaled by
// d_w d_x of its 32-value block and accumulated in float32. pad[i] is the offset
// (floats) of row i's scales inside its aligned run in the stage.
template <int NB, int PW>
TP_DEV void ring_pairs_dot_q8(const uint8_t* stage, uint32_t cstride, uint32_t soff, uint32_t sstride,
                              const int* pad, int cur, int end, const int8_t* xsq, const float* xsd,
                              float* res, int Ks, int pw, int part, int Q, int cb, int ce, int lane) {
  constexpr int R = 2 * PW * NB;  // values: (pair j, row, batch row)
  int rr[PW];
  bool valid[PW];
#pragma unroll
  for (int j = 0; j < PW; ++j) {
    rr[j] = cur + 2 * (pw + 8 * j);
    valid[j] = rr[j] < end;
  }
  if (!valid[0]) return;
  const int nblk = Ks >> 5;
  float acc[R];
#pragma unroll
  for (int i = 0; i < R; ++i) acc[i] = 0.f;
#pragma unroll 2
  for (int c = cb + lane; c < ce; c += 32) {
    int4 xq[NB];
    float xd[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      xq[b] = *reinterpret_cast<const int4*>(xsq + (size_t)b * Ks + 16 * c);
      xd[b] = xsd[b * nblk + (c >> 1)];
    }
#pragma unroll
    for (int j = 0; j < PW; ++j) {
      if (!valid[j]) continue;
#pragma unroll
      for (int row = 0; row < 2; ++row) {
        const int lr = rr[j] + row - cur;  // row within the stage
        const int4 wq = *reinterpret_cast<const int4*>(stage + (size_t)lr * cstride + 16 * c);
        const float dw = reinterpret_cast<const float*>(stage + soff + (size_t)lr * sstride)
            [pad[2 * j + row] + (c >> 1)];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          int sdot = __dp4a(wq.x, xq[b].x, 0);
          sdot = __dp4a(wq.y, xq[b].y, sdot);
          sdot = __dp4a(wq.z, xq[b].z, sdot);
          sdot = __dp4a(wq.w, xq[b].w, sdot);
          acc[(2 * j + row) * NB + b] = fmaf((float)sdot, dw * xd[b], acc[(2 * j + row) * NB + b]);
        }
      }
    }
  }
  const float tot = warp_sum_multi<R>(acc, lane);
  constexpr int kLanes = 32 / R;
  if ((lane & (kLanes - 1)) == 0) {
    const int i = lane / kLanes, j = i / (2 * NB), row = (i / NB) & 1, b = i % NB;
    if (valid[j]) res[((size_t)(rr[j] + row) * NB + b) * Q + part] = tot;
  }
}

size_t a128(size_t v) { return (v + 127) & ~(size_t)127; }

// Shared-memory plan: 8 consumer warps; the most row pairs per stage (16, 8, 4,
// 2, 1) that still leave a ring of at least 2 stages (bf16) or 3 (int8; else 2):
// 16 pairs give each warp two pairs, fewer are each split over 8 / pairs warps.
bool make_plan(int NB, int Ks, int cta_rows, bool wq8, GemvPlan* p) {
  const size_t row_bytes = wq8 ? (size_t)Ks + q8w_scale_slot(Ks) : (size_t)Ks * 2;
  const size_t x_bytes = wq8 ? a128((size_t)NB * Ks + (size_t)NB * (Ks / 32) * 4)
                             : a128((size_t)NB * Ks * 4);
  const size_t bar_bytes = 2 * kMaxStages * 8;
  // the most row pairs per stage with at least 2 ring stages (bf16) or 3 (int8); measured
  // on the 7B block: the bf16 W2 rows (5.5 KB over 4 slices) in 2 stages of 8 pairs
  // instead of 4 of 4 took 1.3 us off the step, while the int8 W2 in 2 stages of 16 pairs
  // instead of 4 of 8 added 1.7 us to its block
  for (int min_stages : {wq8 ? 3 : 2, 2}) {
    for (int P = 16; P >= 1; P >>= 1) {
      const int Q = P >= 8 ? 1 : 8 / P;
      const size_t res_bytes = a128((size_t)cta_rows * NB * Q * 4);
      const size_t fixed = x_bytes + res_bytes + bar_bytes;
      const size_t budget = wq8 ? kSmemBudgetQ8 : kSmemBudget;
      if (fixed >= budget) continue;
      const size_t stage = 2 * (size_t)P * row_bytes;
      int ns = (int)((budget - fixed) / stage);
      if (ns > kMaxStages) ns = kMaxStages;
      if (ns >= min_stages) {
        p->nc = 8;
        p->pairs = P;
        p->split = Q;
        p->pw = P == 16 ? 2 : 1;
        p->nstage = ns;
        p->cta_rows = cta_rows;
        p->ring_off = 0;
        p->x_off = a128((size_t)ns * stage);
        p->res_off = p->x_off + x_bytes;
        p->bar_off = p->res_off + res_bytes;
        p->total = p->bar_off + bar_bytes;
        return true;
      }
    }
  }
  return false;
}

template <int NB, int EPI, bool WQ8>
int launch_one(const GemvArgs& a, cudaStream_t s) {
  int rps = a.rows[0];
  if (EPI == EPI_SWIGLU) rps = 2 * a.rows[0];
  if (EPI == EPI_QKV) rps = a.rows[0] + a.rows[1] + a.rows[2];
  const int npairs = a.nseg * (rps >> 1);
  int grid = num_sms();
  if (grid > npairs) grid = npairs;
  const int cta_rows = 2 * ((npairs + grid - 1) / grid);
  GemvPlan pl;
  if (!make_plan(NB, a.Ks, cta_rows, WQ8, &pl)) return TP_ENOTSUP;
  // Row-split bf16 weights (W_O, W2) with segments of up to 2 KB a row: one bulk copy per
  // row is bound by the copy unit's request rate (about 22 M copies/s per SM: 1 KB rows
  // streamed at 3.2 TB/s, 2 KB rows at 6.5, and W_O's 2 KB rows of the 7B block over 4
  // slices at 3.7 in the step); a 3D tensor map moves several rows per request (W_O of the
  // 7B block over 8 slices: 10.5 -> 5.9 us). Its boxes are 2 rows high: with 8, a
  // stage's few large requests held back the W_O staging's loads of the attention splits
  // (staging 3.1 -> 5.4 us, the 7B step over 4 slices +0.7 us), while 2-row boxes took
  // 0.3 us off that step and 0.5 % off the 32-layer one against bulk copies and 8-row boxes.
  WeightMap<true> wmap{};
  pl.map_box = 0;
  pl.map_nchunk = 0;
  // int8 rows take two bulk copies each (codes, scale run): the map carries the codes
  // when those are under 4 KB a row (W_O and W2 of the 7B block over 4 slices), in boxes
  // of 8 rows (2 or 4 measured slower for the int8 block: 68.8 and 66.6 against 65.8 us).
  // A box's shared-memory destination is box x row bytes into the stage, which a TMA
  // load needs 128-byte aligned: 8 int8 rows and 2 bf16 rows always are (rows are
  // multiples of 32 elements).
  const int esize = WQ8 ? 1 : 2;
  const int box = WQ8 ? 8 : 2;
  if (EPI == EPI_PLAIN && a.nseg > 1 && a.ldw != a.Ks && a.Ks * esize <= (WQ8 ? 4095 : 2048) &&
      ((size_t)box * a.Ks * esize) % 128 == 0 && 2 * pl.pairs >= 8) {
    int chunk = 0;
    for (int c : {256, 128, 64, 32, 16, 8})
      if (a.Ks % c == 0 && a.ldw % c == 0 && a.Ks / c <= 256 && c * esize >= 16) {
        chunk = c;
        break;
      }
    if (chunk && make_tensor_map_rows(&wmap.m, a.w[0], (uint64_t)a.rows[0], (uint64_t)a.ldw, chunk,
                                      a.Ks / chunk, box, esize)) {
      pl.map_box = box;
      pl.map_nchunk = a.Ks / chunk;
    }
  }
  const dim3 block(32 * (pl.nc + 1));
  if constexpr (EPI == EPI_PLAIN) {
    if (pl.map_box) {
      auto kernel = pl.pw == 2 ? k_gemv<NB, EPI, WQ8, 2, true> : k_gemv<NB, EPI, WQ8, 1, true>;
      if (set_smem_once((const void*)kernel, (int)pl.total)) return TP_ECUDA;
      return launch_pdl(kernel, dim3(grid), block, pl.total, s, a, pl, wmap);
    }
  }
  auto kernel = pl.pw == 2 ? k_gemv<NB, EPI, WQ8, 2> : k_gemv<NB, EPI, WQ8, 1>;
  if (set_smem_once((const void*)kernel, (int)pl.total)) return TP_ECUDA;
  return launch_pdl(kernel, dim3(grid), block, pl.total, s, a, pl, WeightMap<false>{});
}

template <int NB, bool WQ8>
int launch_nbw(const GemvArgs& a, int epi, cudaStream_t s) {
  switch (epi) {
    case EPI_PLAIN: return launch_one<NB, EPI_PLAIN, WQ8>(a, s);
    case EPI_SWIGLU: return launch_one<NB, EPI_SWIGLU, WQ8>(a, s);
    default: return launch_one<NB, EPI_QKV, WQ8>(a, s);
  }
}

template <int NB>
int launch_nb(const GemvArgs& a, int epi, cudaStream_t s) {
  return a.wd[0] ? launch_nbw<NB, true>(a, epi, s) : launch_nbw<NB, false>(a, epi, s);
}

}  // namespace

// Batch rows are handled two at a time (each launch streams the weights once).
int launch_gemv(const GemvArgs& a0, int epi, cudaStream_t s) {
  if (a0.Ks % 32 != 0 || a0.Ks < 32 || a0.nseg < 1) return TP_EINVAL;
  if (a0.wd[0] && a0.ldw % 64 != 0) return TP_EINVAL;  // whole 16-byte scale runs per matrix
  if (((a0.rows[0] | a0.rows[1] | a0.rows[2]) & 1) != 0) return TP_EINVAL;
  for (int b = 0; b < a0.nb;) {
    GemvArgs a = a0;
    a.b0 = a0.b0 + b;
    a.nb = a0.nb - b >= 2 ? 2 : 1;
    const int rc = a.nb == 2 ? launch_nb<2>(a, epi, s) : launch_nb<1>(a, epi, s);
    if (rc != TP_OK) return rc;
    b += a.nb;
  }
  return TP_OK;
}

}  // namespace tp
