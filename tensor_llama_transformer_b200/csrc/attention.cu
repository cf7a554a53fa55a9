// Decode attention over the bf16 KV cache: split-context flash decoding on
// warp-level tensor-core MMAs.
//
// distributed-llama issue #29, llamaMultiheadAtt: each slice computes the
// attention of its own heads locally; tt-metal's Llama-2 thread separates GQA
// from MHA. A CTA owns (context split, kv head, batch row) and every query head
// that reads that kv head (1 for MHA, 8 for the 70B shape), so each K/V byte is
// read from HBM once per step. With more query heads per kv head (multi-query
// attention, Pope et al. demo 3: up to 64 on one kv head) the heads go in groups
// of 8 to CTAs that read the same tiles, concurrently, mostly from L2. The split's 64-position K and V tiles stream
// through a 3-stage shared-memory ring by TMA (128-byte swizzle, so the
// ldmatrix reads below are conflict-free), issued by a producer warp. Four
// consumer warps take 16 positions of each tile:
//   S = Q K^T and O += P V on mma.m16n8k16 (bf16 operands, float32 accumulate),
//   with an online softmax in registers (running max m, sum l, rescaled O).
// Q and P enter the MMAs as hi/lo bf16 pairs in the two 8-row halves of the
// 16-row operand (row g holds bf16(v), row g+8 holds bf16(v - bf16(v)) for head
// g of the group), so the products keep about 16 significant bits; the halves
// of S and of O are added in registers. The warps' partials are merged in
// shared memory and the split writes one unnormalised partial (o, m, l) per
// head; a second kernel combines the splits with the usual rescaling
//   M = max_c m_c,  o = sum_c e^{m_c - M} o_c / sum_c e^{m_c - M} l_c.
// Positions past pos are masked (score -inf, and the V rows zeroed in shared
// memory), so stale cache contents never reach the output. Rows may share a
// cache sequence (a prefill chunk): each reads its own positions 0..pos, which
// the q/k/v kernel before this one has written for every row of the step, so
// the chunk attends causally. The MMAs do at most
// 16 FLOP per KV byte, far below the tensor pipe's rate: the kernel is HBM-bound.
#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "pipeline.cuh"

namespace tp {

namespace {

constexpr int kTile = 64;                // positions per tile
constexpr int kStages = 3;
constexpr int kCWarps = 4;               // consumer warps, 16 positions of each tile
constexpr int kAThreads = 32 * (kCWarps + 1);
constexpr int kBox = kTile * 64 * 2;     // one box: 64 positions x 64 dims of bf16 (8 KB)
constexpr int kStageBytes = 4 * kBox;    // K (two dim halves) + V (two dim halves)
constexpr int kQStride = 136;            // staged Q row stride (bf16), padded against conflicts
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 16 * kQStride * 2;
static_assert(kCWarps * 8 * kHeadDim * 4 <= kStageBytes, "merge staging must fit in stage 0");

// Tiles of one split for a context of P positions: the same for both kernels.
TP_DEV int tiles_per_split(int P, int nsplit) {
  const int ntiles = (P + kTile - 1) / kTile;
  return (ntiles + nsplit - 1) / nsplit;
}

// One K/V tile of a consumer warp (positions t0 + w0 .. t0 + w0 + 15): S = Q K^T,
// the online softmax of the thread's head row (positions >= P_row masked), and
// O += P V. V rows at positions >= p_zero (past every context the CTA serves)
// are zeroed first so that stale cache contents never reach O.
TP_DEV void attn_tile(uint8_t* smem, uint32_t kb, const uint32_t (&qa)[8][4], float (&o)[16][4],
                      float& m_run, float& l_run, int lane, int w0, int t0, int P_row,
                      int p_zero) {
  const uint32_t vb = kb + 2 * kBox;
  if (t0 + w0 + 16 > p_zero) {  // V rows past every context -> 0 (a context's last tile)
    for (int idx = lane; idx < 16 * 16; idx += 32) {
      const int r = idx >> 4, c = idx & 15;
      if (t0 + w0 + r >= p_zero)
        *reinterpret_cast<uint4*>(smem + (kv_tile_addr(vb, w0 + r, c) - s2u(smem))) =
            make_uint4(0u, 0u, 0u, 0u);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
  }
  // S = Q K^T over the warp's two 8-position column tiles
  float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  {
    const int t = w0 + (lane & 7) + 8 * (lane >> 4), ch = (lane >> 3) & 1;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t bf[4];
      ldsm_x4(kv_tile_addr(kb, t, 2 * ks + ch), bf);
      mma_bf16(sc[0], qa[ks], bf[0], bf[1]);
      mma_bf16(sc[1], qa[ks], bf[2], bf[3]);
    }
  }
  // this thread's scores of head g: positions t0 + w0 + 8 nt + 2 (lane & 3) + j
  float sv[2][2], tmax = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int tp = t0 + w0 + 8 * nt + 2 * (lane & 3) + j;
      const float v = sc[nt][j] + sc[nt][2 + j];  // hi row + lo row
      sv[nt][j] = tp < P_row ? v : -INFINITY;
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
  // O += P V over the warp's 16 positions, 16 dim tiles of 8
  {
    const int t = w0 + (lane & 7) + 8 * ((lane >> 3) & 1), ch = lane >> 4;
#pragma unroll
    for (int np = 0; np < 8; ++np) {
      uint32_t bf[4];
      ldsm_x4_t(kv_tile_addr(vb, t, 2 * np + ch), bf);
      mma_bf16(o[2 * np], pa, bf[0], bf[1]);
      mma_bf16(o[2 * np + 1], pa, bf[2], bf[3]);
    }
  }
}

template <int G>
__global__ void __launch_bounds__(kAThreads) k_attn_split(const __grid_constant__ CUtensorMap mK,
                                                          const __grid_constant__ CUtensorMap mV,
                                                          AttnArgs a, int nsplit) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem + kStages * kStageBytes);  // [16][kQStride]
  __shared__ uint64_t full[kStages], empty[kStages];
  __shared__ float s_m[kCWarps][8], s_l[kCWarps][8];

  // blockIdx.y = kv head x groups of G query heads: with more than 8 query heads
  // per kv head (multi-query attention), groups of 8 share the kv head's tiles
  const int hgroups = a.H / a.Hkv / G;
  const int split = blockIdx.x, kvh = blockIdx.y / hgroups, b = blockIdx.z;
  const int h0 = kvh * (a.H / a.Hkv) + (blockIdx.y - kvh * hgroups) * G;  // first query head
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();
  // pos and seq are the caller's inputs (no kernel of the step writes them)
  const int P = a.pos[b] + 1;
  const int ntiles = (P + kTile - 1) / kTile;
  const int tpc = tiles_per_split(P, nsplit);
  const int i0 = split * tpc, i1 = min(ntiles, i0 + tpc);
  const size_t pbase = ((size_t)b * a.H + (size_t)h0) * nsplit + split;
  if (i0 >= i1) {  // nothing left for this split: an empty partial (m = -inf, l = 0)
    pdl_wait();
    if (threadIdx.x < G) {
      a.part_ml[(pbase + (size_t)threadIdx.x * nsplit) * 2 + 0] = -INFINITY;
      a.part_ml[(pbase + (size_t)threadIdx.x * nsplit) * 2 + 1] = 0.f;
    }
    return;
  }
  const int sq = a.seq ? a.seq[b] : b;  // the row's cache sequence
  const int row_base = (sq * a.Hkv + kvh) * a.max_seq;
  // The q/k/v kernel before this one writes q and, in the cache, the row's
  // position pos only (with a sequence map, the positions of every row of the
  // step): the tiles below pos's tile are streamed before waiting for it.
  const int first_dep = a.seq ? i0 : ntiles - 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCWarps);
    }
    mbar_init_fence();
  }
  __syncthreads();

  if (warp == kCWarps) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      const uint64_t pol = l2_evict_first();  // cache tiles are read once per step
      bool waited = false;
      for (int i = i0; i < i1; ++i) {
        const int k = i - i0, s = k % kStages;
        if (i >= first_dep && !waited) {
          pdl_wait();
          waited = true;
        }
        if (!mbar_wait(&empty[s], ((uint32_t)(k / kStages) & 1u) ^ 1u, a.err)) break;
        mbar_expect_tx(&full[s], kStageBytes);
        uint8_t* st = smem + s * kStageBytes;
        const int y = row_base + i * kTile;
        tma_load_2d_hint(st, &mK, 0, y, &full[s], pol);
        tma_load_2d_hint(st + kBox, &mK, 64, y, &full[s], pol);
        tma_load_2d_hint(st + 2 * kBox, &mV, 0, y, &full[s], pol);
        tma_load_2d_hint(st + 3 * kBox, &mV, 64, y, &full[s], pol);
      }
      if (!waited) pdl_wait();
    }
    __syncwarp();
    pdl_wait();  // (every thread: the partials below overwrite a buffer earlier kernels read)
  } else {
    // ------------------------------------------------------------ consumer warps
    pdl_wait();  // q comes from the q/k/v kernel
    // Q of the group's heads scaled by 1/sqrt(hd): hi in row g, lo in row g + 8
    const float scale = 1.0f / sqrtf((float)kHeadDim);
    for (int i = threadIdx.x; i < 8 * kHeadDim; i += kCWarps * 32) {
      const int gq = i / kHeadDim, d = i - gq * kHeadDim;
      uint16_t hi = 0, lo = 0;
      if (gq < G)
        bf16_split(a.q[((size_t)b * a.H + (size_t)h0 + gq) * kHeadDim + d] * scale, hi, lo);
      qs[gq * kQStride + d] = hi;
      qs[(gq + 8) * kQStride + d] = lo;
    }
    consumers_sync(kCWarps * 32);
    const int g = lane >> 2;  // the head row whose scores this thread holds
    uint32_t qa[8][4];        // A fragments of Q, one per 16-dim step
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
    bool ok = true;
    const int w0 = 16 * warp;  // this warp's positions within a tile
    for (int i = i0; i < i1; ++i) {
      const int k = i - i0, s = k % kStages;
      const bool got = ok ? mbar_wait(&full[s], (uint32_t)(k / kStages) & 1u, a.err) : false;
      ok = __all_sync(0xffffffffu, got);
      if (ok)
        attn_tile(smem, s2u(smem + s * kStageBytes), qa, o, m_run, l_run, lane, w0, i * kTile, P, P);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // the warp's partial of head g: l summed over the row's 4 lanes
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    if ((lane & 3) == 0) {
      s_m[warp][g] = m_run;
      s_l[warp][g] = l_run;
    }
    // every tile has been consumed by all consumer warps: stage 0 takes the O partials
    consumers_sync(kCWarps * 32);
    float* ro = reinterpret_cast<float*>(smem);  // [kCWarps][8][kHeadDim]
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int d = 8 * nt + 2 * (lane & 3);
      ro[(warp * 8 + g) * kHeadDim + d] = o[nt][0] + o[nt][2];
      ro[(warp * 8 + g) * kHeadDim + d + 1] = o[nt][1] + o[nt][3];
    }
  }
  __syncthreads();
  // merge the consumer warps: thread per (head, dim)
  const float* ro = reinterpret_cast<const float*>(smem);
  for (int idx = threadIdx.x; idx < G * kHeadDim; idx += kAThreads) {
    const int gg = idx / kHeadDim, d = idx - gg * kHeadDim;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kCWarps; ++w) M = fmaxf(M, s_m[w][gg]);
    float os = 0.f, ls = 0.f;
#pragma unroll
    for (int w = 0; w < kCWarps; ++w) {
      const float f = s_m[w][gg] == -INFINITY ? 0.f : expf(s_m[w][gg] - M);
      os = fmaf(f, ro[(w * 8 + gg) * kHeadDim + d], os);
      ls = fmaf(f, s_l[w][gg], ls);
    }
    const size_t pi = pbase + (size_t)gg * nsplit;
    a.part_o[pi * kHeadDim + d] = os;
    if (d == 0) {
      a.part_ml[pi * 2 + 0] = M;
      a.part_ml[pi * 2 + 1] = ls;
    }
  }
}

// Rows that share a cache sequence (a prefill chunk, given a sequence map on the
// batched path): a CTA takes R = 8 / G consecutive rows and the G query heads of
// one kv head, so its 8 head rows are (row, head) pairs that read the same K/V
// tiles -- each tile crosses into shared memory once for R tokens instead of
// once per token. Rows of different sequences in one CTA (a step mixing decode
// rows of several sequences) are taken in passes, one per sequence. A pass's
// split covers tiles of the longest context among its rows; every row masks the
// positions past its own, so it attends causally. Each (row, head, split) slot
// gets a partial, empty ones (m = -inf, l = 0) included, and k_attn_combine reads
// all splits.
template <int G>
__global__ void __launch_bounds__(kAThreads) k_attn_rows(const __grid_constant__ CUtensorMap mK,
                                                         const __grid_constant__ CUtensorMap mV,
                                                         AttnArgs a, int nsplit) {
  constexpr int R = 8 / G;  // rows per CTA
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem + kStages * kStageBytes);  // [16][kQStride]
  __shared__ uint64_t full[kStages], empty[kStages];
  __shared__ float s_m[kCWarps][8], s_l[kCWarps][8];
  __shared__ int s_seq[R], s_pmax[R], s_i0[R], s_i1[R];  // per pass
  __shared__ unsigned s_act[R];  // per pass: bit g set when head row g's token is in it
  __shared__ int s_npass;

  const int split = blockIdx.x, kvh = blockIdx.y, b0 = blockIdx.z * R;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();
  pdl_wait();  // q and the cache rows of this step come from the q/k/v kernel
  if (threadIdx.x == 0) {
    int np = 0;
    for (int r = 0; r < R && b0 + r < a.B; ++r) {
      const int sq = a.seq[b0 + r], P = a.pos[b0 + r] + 1;
      int p = 0;
      while (p < np && s_seq[p] != sq) ++p;
      if (p == np) {
        s_seq[p] = sq;
        s_pmax[p] = 0;
        s_act[p] = 0u;
        ++np;
      }
      s_pmax[p] = max(s_pmax[p], P);
      s_act[p] |= ((1u << G) - 1u) << (r * G);
    }
    for (int p = 0; p < np; ++p) {
      const int ntiles = (s_pmax[p] + kTile - 1) / kTile;
      const int tpc = tiles_per_split(s_pmax[p], nsplit);
      s_i0[p] = split * tpc;
      s_i1[p] = min(ntiles, split * tpc + tpc);
    }
    s_npass = np;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCWarps);
    }
    mbar_init_fence();
  }
  // head row g = (token b0 + g / G, query head kvh G + g % G), scaled by 1/sqrt(hd):
  // hi in row g, lo in row g + 8
  const float scale = 1.0f / sqrtf((float)kHeadDim);
  for (int i = threadIdx.x; i < 8 * kHeadDim; i += kAThreads) {
    const int g = i / kHeadDim, d = i - g * kHeadDim, b = b0 + g / G;
    uint16_t hi = 0, lo = 0;
    if (b < a.B)
      bf16_split(a.q[((size_t)b * a.H + (size_t)kvh * G + g % G) * kHeadDim + d] * scale, hi, lo);
    qs[g * kQStride + d] = hi;
    qs[(g + 8) * kQStride + d] = lo;
  }
  __syncthreads();
  const int npass = s_npass;

  if (warp == kCWarps) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      const uint64_t pol = l2_evict_first();
      bool ok = true;
      int k = 0;
      for (int p = 0; p < npass && ok; ++p) {
        const int row_base = (s_seq[p] * a.Hkv + kvh) * a.max_seq;
        for (int i = s_i0[p]; i < s_i1[p]; ++i, ++k) {
          const int s = k % kStages;
          if (!mbar_wait(&empty[s], ((uint32_t)(k / kStages) & 1u) ^ 1u, a.err)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&full[s], kStageBytes);
          uint8_t* st = smem + s * kStageBytes;
          const int y = row_base + i * kTile;
          tma_load_2d_hint(st, &mK, 0, y, &full[s], pol);
          tma_load_2d_hint(st + kBox, &mK, 64, y, &full[s], pol);
          tma_load_2d_hint(st + 2 * kBox, &mV, 0, y, &full[s], pol);
          tma_load_2d_hint(st + 3 * kBox, &mV, 64, y, &full[s], pol);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumer warps
    const int g = lane >> 2;  // the head row whose scores this thread holds
    const int bg = b0 + g / G;
    const int Pg = bg < a.B ? a.pos[bg] + 1 : 0;
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
    bool ok = true;
    const int w0 = 16 * warp;
    int k = 0;
    for (int p = 0; p < npass; ++p) {
      const int P_row = ((s_act[p] >> g) & 1u) ? Pg : 0;  // 0: not this pass's sequence
      for (int i = s_i0[p]; i < s_i1[p]; ++i, ++k) {
        const int s = k % kStages;
        const bool got = ok ? mbar_wait(&full[s], (uint32_t)(k / kStages) & 1u, a.err) : false;
        ok = __all_sync(0xffffffffu, got);
        if (ok)
          attn_tile(smem, s2u(smem + s * kStageBytes), qa, o, m_run, l_run, lane, w0, i * kTile,
                    P_row, s_pmax[p]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
    }
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    if ((lane & 3) == 0) {
      s_m[warp][g] = m_run;
      s_l[warp][g] = l_run;
    }
    consumers_sync(kCWarps * 32);
    float* ro = reinterpret_cast<float*>(smem);  // [kCWarps][8][kHeadDim]
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int d = 8 * nt + 2 * (lane & 3);
      ro[(warp * 8 + g) * kHeadDim + d] = o[nt][0] + o[nt][2];
      ro[(warp * 8 + g) * kHeadDim + d + 1] = o[nt][1] + o[nt][3];
    }
  }
  __syncthreads();
  const float* ro = reinterpret_cast<const float*>(smem);
  for (int idx = threadIdx.x; idx < 8 * kHeadDim; idx += kAThreads) {
    const int gg = idx / kHeadDim, d = idx - gg * kHeadDim, b = b0 + gg / G;
    if (b >= a.B) continue;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kCWarps; ++w) M = fmaxf(M, s_m[w][gg]);
    float os = 0.f, ls = 0.f;
#pragma unroll
    for (int w = 0; w < kCWarps; ++w) {
      const float f = s_m[w][gg] == -INFINITY ? 0.f : expf(s_m[w][gg] - M);
      os = fmaf(f, ro[(w * 8 + gg) * kHeadDim + d], os);
      ls = fmaf(f, s_l[w][gg], ls);
    }
    const size_t pi = ((size_t)b * a.H + (size_t)kvh * G + gg % G) * nsplit + split;
    a.part_o[pi * kHeadDim + d] = os;
    if (d == 0) {
      a.part_ml[pi * 2 + 0] = M;
      a.part_ml[pi * 2 + 1] = ls;
    }
  }
}

// One CTA per (head, batch row); thread d owns output dimension d.
__global__ void __launch_bounds__(kHeadDim) k_attn_combine(AttnArgs a, int nsplit) {
  pdl_launch_dependents();
  pdl_wait();
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  // every split of every (row, head) holds a partial, the empty ones m = -inf, l = 0
  const size_t base = ((size_t)b * a.H + h) * nsplit;
  float M = -INFINITY;
  for (int c = 0; c < nsplit; ++c) M = fmaxf(M, a.part_ml[(base + c) * 2]);
  float l = 0.f, o = 0.f;
  for (int c = 0; c < nsplit; ++c) {
    const float mc = a.part_ml[(base + c) * 2];
    if (mc == -INFINITY) continue;  // an empty split: its o may be stale, never read it
    const float w = expf(mc - M);
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
int launch_rows(const AttnArgs& a, const CUtensorMap& mK, const CUtensorMap& mV, int nsplit,
                cudaStream_t s) {
  if (set_smem_once((const void*)k_attn_rows<G>, kSmemBytes)) return TP_ECUDA;
  return launch_pdl(k_attn_rows<G>, dim3(nsplit, a.Hkv, (a.B + 8 / G - 1) / (8 / G)),
                    dim3(kAThreads), kSmemBytes, s, mK, mV, a, nsplit);
}

template <int G>
int launch_g(const AttnArgs& a, const CUtensorMap& mK, const CUtensorMap& mV, int nsplit,
             cudaStream_t s) {
  if (set_smem_once((const void*)k_attn_split<G>, kSmemBytes)) return TP_ECUDA;
  const int hgroups = a.H / a.Hkv / G;
  return launch_pdl(k_attn_split<G>, dim3(nsplit, a.Hkv * hgroups, a.B), dim3(kAThreads), kSmemBytes, s,
                    mK, mV, a, nsplit);
}

}  // namespace

int attention_max_splits(int max_seq) { return (max_seq + kTile - 1) / kTile; }

// Splits per (batch row, kv head): the count that minimises waves x (tiles per
// CTA + 4), two CTAs resident per SM, over a context of max_seq positions. The
// kernels divide the actual context (pos + 1) over that many splits.
int attention_splits(int B, int Hkv, int max_seq) {
  const int T = attention_max_splits(max_seq);
  const long slots = 2L * num_sms();
  // a CTA's fixed work (barrier setup, the dependency wait, staging Q, combining its
  // consumer warps and writing the partials) costs about as much as 4 tiles (measured:
  // the 70B block at batch 32 and context 4096 took 449 us with 8 splits of 8 tiles,
  // 436 us with one split of 64 tiles; its multi-query form 426 and 403 us)
  constexpr int over = 4;
  int best = 1;
  long best_cost = -1;
  for (int sp = 1; sp <= T; ++sp) {
    const int tpc = (T + sp - 1) / sp;
    if ((T + tpc - 1) / tpc != sp) continue;  // an equivalent smaller count exists
    const long ctas = (long)B * Hkv * sp;
    const long cost = ((ctas + slots - 1) / slots) * (tpc + over);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = sp;
    }
  }
  return best;
}

int attention_nsplit(int B, int H, int Hkv, int max_seq) {
  const int G = H / Hkv;
  const int hgroups = G > 8 ? G / 8 : 1;  // CTAs per kv head
  return attention_splits(B, Hkv * hgroups, max_seq);
}

int launch_attention(const AttnArgs& a, cudaStream_t s, bool combine) {
  const int G = a.H / a.Hkv;
  // rows mapped to cache sequences share tiles (k_attn_rows) when the splits are
  // combined here and a CTA holds at least two rows
  const bool shared = a.seq && combine && G <= 4;
  const int nsplit = a.nsplit > 0 ? a.nsplit
                     : shared ? attention_splits((a.B + 8 / G - 1) / (8 / G), a.Hkv, a.max_seq)
                              : attention_nsplit(a.B, a.H, a.Hkv, a.max_seq);
  if (nsplit > a.nchunk) return TP_EINVAL;
  if (!aligned16(a.kc) || !aligned16(a.vc)) return TP_EALIGN;
  CUtensorMap mK, mV;
  const uint64_t rows = (uint64_t)(a.seq ? a.nseq : a.B) * a.Hkv * a.max_seq;
  if (!make_tensor_map_2d(&mK, a.kc, rows, kHeadDim, kHeadDim, 64, kTile) ||
      !make_tensor_map_2d(&mV, a.vc, rows, kHeadDim, kHeadDim, 64, kTile))
    return TP_ECUDA;
  int rc;
  if (shared) {
    rc = G == 1 ? launch_rows<1>(a, mK, mV, nsplit, s)
       : G == 2 ? launch_rows<2>(a, mK, mV, nsplit, s)
                : launch_rows<4>(a, mK, mV, nsplit, s);
    if (rc != TP_OK) return rc;
    return launch_pdl(k_attn_combine, dim3(a.H, a.B), dim3(kHeadDim), 0, s, a, nsplit);
  }
  switch (G) {
    case 1: rc = launch_g<1>(a, mK, mV, nsplit, s); break;
    case 2: rc = launch_g<2>(a, mK, mV, nsplit, s); break;
    case 4: rc = launch_g<4>(a, mK, mV, nsplit, s); break;
    case 8: rc = launch_g<8>(a, mK, mV, nsplit, s); break;
    default:
      if (G % 8 != 0 || G > 64) return TP_ENOTSUP;
      rc = launch_g<8>(a, mK, mV, nsplit, s);  // groups of 8 query heads per CTA
      break;
  }
  if (rc != TP_OK || !combine) return rc;
  return launch_pdl(k_attn_combine, dim3(a.H, a.B), dim3(kHeadDim), 0, s, a, nsplit);
}

}  // namespace tp
