// Persistent tcgen05 GEMM for the batched FFN and the batched decode products (sm_100a).
//
//   D[seg, m, n] = sum_{k < K} A[m, seg*K + k] * B[n, seg*K + k]
//
// Both operands bf16 with the contraction dimension contiguous (a PyTorch
// Linear weight is already in this layout). A segment is the contraction range
// one tensor-parallel slice owns (a row split); with nseg > 1 each slice's
// partial product goes to its own plane of the output, to be summed by the
// merge (aiterms.tw "Tensor Parallelism": Linear2 split by rows, then an
// all-reduce; Pope et al. demo1: 2D weight-stationary adds a partial-sum stage
// before the activation), or, with the segment-sum epilogue, is summed in
// slice order by the CTA that owns the output tile: it computes the tile's
// segments one after another, each into a fresh TMEM accumulator, and adds
// each partial (through the Q8 round trip when quantising) to a running sum
// in registers, so the partials never reach HBM. The FFN puts tokens on M and
// features on N (N tile 256, 128 with the segment sum); batched decode puts
// weight rows on M and the batch on N (N tile 32 or 64, transposed store), so
// the weight stream is the M x K operand.
//
// Structure (one CTA per SM, 192 threads; 320 with the quantised segment sum):
//   warp 0  : TMA producer — 128x64 A tile and BNx64 B tile per stage, 128-byte
//             swizzle, a ring of 4 (BN 256) to 10 (BN 32) stages of shared
//             memory, completion on mbarriers.
//   warp 1  : allocates TMEM for two 128xBN fp32 accumulators and one lane
//             issues tcgen05.mma (M=128, N=BN, K=16, bf16 -> fp32);
//             tcgen05.commit releases each smem stage and publishes each tile.
//   warps 2-5: epilogue — tcgen05.ld of the accumulator (each warp its 32 TMEM
//             lanes = 32 output rows), activation, stores to global memory,
//             overlapped with the next tile's mainloop (double-buffered TMEM);
//             warps 2-9 with the quantised segment sum, two per lane quarter,
//             each owning half of the tile's columns.
// Tiles are visited m-fastest so that the CTAs working at the same time share
// the weight tile through L2. No TMA multicast is used. Every wait on an
// mbarrier is bounded by a 2 s timer; on expiry the kernel sets *err and the
// roles leave their loops, so a fault in the pipeline cannot hang the GPU.
#include <cuda.h>

#include "gemm_tc.cuh"
#include "pipeline.cuh"

namespace tp {
namespace {

constexpr int BM = 128, BK = 64;

// EW epilogue warps: 4 (one per 32-lane quarter of TMEM), or 8 for the segment sum with
// the Q8 round trip (the only 8-warp form, so EW == 8 also selects the round trip at
// compile time), where two warps share a lane quarter and each owns half of the
// tile's columns: each then waits for two column loads per segment instead of four,
// keeps half the running sums and quantises half the values, and every SM
// sub-partition has two epilogue warps to hide the latencies (measured: Q8 faithful
// 1D-64 FFN 5.8 -> 3.6 ms; without Q8 the 4-warp form is 4 % faster).
constexpr int tc_threads(int ew) { return 64 + 32 * ew; }
constexpr int A_BYTES = BM * BK * 2;  // 16 KB

template <int BN>
struct TcCfg {
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (200 * 1024) / STAGE_BYTES > 10 ? 10 : (200 * 1024) / STAGE_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  // two accumulators of BN columns, allocated as a power of two >= 32
  static constexpr uint32_t TMEM_COLS = 2 * BN <= 32 ? 32 : (2 * BN <= 64 ? 64 : (2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512)));
};

TP_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
TP_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

TP_DEV void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                      uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

TP_DEV void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   s2u(bar))
               : "memory");
}

TP_DEV void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
TP_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart (stride
// byte offset), descriptor version 1, layout type 2 = SWIZZLE_128B. The leading
// byte offset is not used by this layout. Advancing K by 16 bf16 elements inside
// the swizzle atom adds 32 bytes (2 in the >>4 encoding) to the start address.
TP_DEV uint64_t desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t idesc_bf16(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

TP_DEV uint32_t pack_bf16x2(float a, float b) {
  return (uint32_t)f32_to_bf16_bits(a) | ((uint32_t)f32_to_bf16_bits(b) << 16);
}

// m-tiles of the concatenated A matrices: matrix j owns m-tiles [mt_off[j], mt_off[j+1]).
struct TcTiles {
  int mt_off[4];
  int num_n;
  int ntiles;
};

template <int BN, int EPI, int EW>
__global__ void __launch_bounds__(tc_threads(EW), 1)
    k_tc_gemm(const __grid_constant__ CUtensorMap mA0, const __grid_constant__ CUtensorMap mA1,
              const __grid_constant__ CUtensorMap mA2, const __grid_constant__ CUtensorMap mB,
              const __grid_constant__ CUtensorMap mB2, TcGemm g, TcTiles tt) {
  using C = TcCfg<BN>;
  constexpr int STAGES = C::STAGES, B_BYTES = C::B_BYTES, STAGE_BYTES = C::STAGE_BYTES;
  constexpr uint32_t TMEM_COLS = C::TMEM_COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&tfull[j], 1);
      mbar_init(&tempty[j], EW);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     s2u(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nk = (g.K + BK - 1) / BK;  // a partial last block reads zeros past the segment
  const int num_m = tt.mt_off[g.nA];
  const int per_seg = num_m * tt.num_n;
  const int ntiles = tt.ntiles;
  constexpr int NOUT = EPI == TC_EPI_SWIGLU_BF16 ? BN / 2 : BN;  // output columns per tile
  constexpr bool SEGSUM = EPI == TC_EPI_SEGSUM_F32 || EPI == TC_EPI_SEGSUM_RELU_BF16;
  // The CTA's i-th tile, or -1 past its last: tiles blockIdx.x, + gridDim.x, ...; with
  // the segment sum, all segments of one output tile in order, then the next output tile.
  auto tile_of = [&](int i) -> int {
    if (!SEGSUM) {
      const int64_t t = blockIdx.x + (int64_t)i * gridDim.x;
      return t < ntiles ? (int)t : -1;
    }
    const int64_t u = blockIdx.x + (int64_t)(i / g.nseg) * gridDim.x;
    return u < per_seg ? (i % g.nseg) * per_seg + (int)u : -1;
  };
  // tile -> (segment, n block, matrix, first row in the matrix, first output row)
  auto decode = [&](int tile, int& seg, int& nb, int& mat, int& m0, int& orow0) {
    seg = tile / per_seg;
    const int r = tile - seg * per_seg;
    nb = r / num_m;
    const int mt = r - nb * num_m;
    mat = (mt >= tt.mt_off[1]) + (mt >= tt.mt_off[2]);
    m0 = (mt - tt.mt_off[mat]) * BM;
    orow0 = m0;
    for (int j = 0; j < mat; ++j) orow0 += g.Am[j];
  };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      bool ok = true;
      // The first ring stages take only the operand no earlier kernel writes (g.indep)
      // before the wait for the previous kernel; the other operand's tiles of those
      // stages follow the wait. Without such an operand the producer waits first.
      const bool pre_a = (g.indep & TC_INDEP_A) != 0, pre_b = !pre_a && (g.indep & TC_INDEP_B);
      bool waited = !(pre_a || pre_b);
      if (waited) pdl_wait();
      int npend = 0;
      int pend_stage[STAGES], pend_kx[STAGES], pend_seg[STAGES], pend_m0[STAGES], pend_n0[STAGES],
          pend_mat[STAGES];
      auto load_a = [&](int st, int mat, int kx, int seg, int m0) {
        const CUtensorMap* mA = mat == 0 ? &mA0 : (mat == 1 ? &mA1 : &mA2);
        tma_load_3d(sA + st * A_BYTES, mA, kx, seg, m0, &full[st]);
      };
      auto load_b = [&](int st, int kx, int seg, int n0) {
        tma_load_3d(sB + st * B_BYTES, &mB, kx, seg, n0, &full[st]);
        if (EPI == TC_EPI_SWIGLU_BF16)
          tma_load_3d(sB + st * B_BYTES + B_BYTES / 2, &mB2, kx, seg, n0, &full[st]);
      };
      auto flush = [&]() {  // wait for the previous kernel, then the deferred tiles
        pdl_wait();
        waited = true;
        for (int i = 0; i < npend; ++i) {
          if (pre_a) load_b(pend_stage[i], pend_kx[i], pend_seg[i], pend_n0[i]);
          else load_a(pend_stage[i], pend_mat[i], pend_kx[i], pend_seg[i], pend_m0[i]);
        }
        npend = 0;
      };
      for (int i = 0; ok; ++i) {
        const int tile = tile_of(i);
        if (tile < 0) break;
        int seg, nb, mat, m0, orow0;
        decode(tile, seg, nb, mat, m0, orow0);
        const int n0 = nb * NOUT;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], ph ^ 1, g.err)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&full[stage], STAGE_BYTES);
          const int kx = kb * BK;
          if (waited) {
            load_a(stage, mat, kx, seg, m0);
            load_b(stage, kx, seg, n0);
          } else {
            if (pre_a) load_a(stage, mat, kx, seg, m0);
            else load_b(stage, kx, seg, n0);
            pend_stage[npend] = stage;
            pend_kx[npend] = kx;
            pend_seg[npend] = seg;
            pend_m0[npend] = m0;
            pend_n0[npend] = n0;
            pend_mat[npend] = mat;
            if (++npend == STAGES) flush();
          }
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
      }
      if (!waited) flush();
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(BM, BN);
      int stage = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int it = 0; ok && tile_of(it) >= 0; ++it) {
        const int acc = it & 1;
        const uint32_t aph = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], aph ^ 1, g.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], ph, g.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = desc_sw128(s2u(sA + stage * A_BYTES));
          const uint64_t b0 = desc_sw128(s2u(sB + stage * B_BYTES));
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16(d_tmem, a0 + 2 * k, b0 + 2 * k, IDESC, (kb | k) != 0 ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (ok) umma_commit(&tfull[acc]);
      }
    }
  } else {
    // epilogue warps 2..5: TMEM lanes 32*(warp%4) .. +31
    const int q = warp & 3;  // TMEM lane quarter (hardware: warp w reads lanes 32 (w % 4) ..)
    // segment sum: the warp's half of the tile's columns, [cw * cpart, cw * (cpart + 1))
    constexpr int CW = BN * 4 / EW;
    const int cpart = (warp - 2) >> 2;
    // TC_EPI_SEGSUM_*: the thread's row of the output tile, summed over the segments so far
    float run[SEGSUM ? CW : 1];
    for (int it = 0;; ++it) {
      const int tile = tile_of(it);
      if (tile < 0) break;
      const int acc = it & 1;
      const uint32_t aph = (uint32_t)(it >> 1) & 1u;
      if (!mbar_wait(&tfull[acc], aph, g.err)) break;
      tc_fence_after();
      int seg, nb, mat, m0, orow0;
      decode(tile, seg, nb, mat, m0, orow0);
      const int row = m0 + 32 * q + lane;  // row within matrix `mat`
      const int n0 = nb * NOUT;
      const bool row_ok = row < g.Am[mat];
      const uint32_t taddr = tmem + (uint32_t)(acc * BN) + ((uint32_t)(32 * q) << 16);
      if constexpr (SEGSUM) {
        // run[j] += sync(partial of this segment), in segment order from 0.f: the same
        // float32 additions as summing materialised partials one slice after another
        if (seg == 0) {
#pragma unroll
          for (int j = 0; j < CW; ++j) run[j] = 0.f;
        }
        const bool last = seg == g.nseg - 1;
        const int cb = cpart * CW;  // the warp's first column within the tile
#pragma unroll
        for (int h = 0; h < CW / 32; ++h) {
          const int c = cb + 32 * h;  // tile column of this 32-column block
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_wait_ld();
          float p[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) p[j] = __uint_as_float(v[j]);
          if constexpr (EW == 8) {  // quantised (the host runs the Q8 segment sum with 8 warps):
            // the 32 columns are one Q8 block of the row (n0 + c is a multiple of 32)
            float am = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) am = fmaxf(am, fabsf(p[j]));
            const float d = q8_scale(am), r = q8_recip(d);
            q8_codes<16>(p, p, d, r);  // the block's codes in place, 16 at a time
            q8_codes<16>(p + 16, p + 16, d, r);
#pragma unroll
            for (int j = 0; j < 32; ++j) p[j] = __fmul_rn(p[j], d);
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) run[32 * h + j] += p[j];
          if (last && row_ok && n0 + c < g.N) {
            if (EPI == TC_EPI_SEGSUM_F32) {
              float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(g.out) +
                                                     (size_t)row * g.ldo + n0 + c);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                o4[j] = make_float4(run[32 * h + 4 * j], run[32 * h + 4 * j + 1],
                                    run[32 * h + 4 * j + 2], run[32 * h + 4 * j + 3]);
            } else {
              uint4* o4 = reinterpret_cast<uint4*>(static_cast<uint16_t*>(g.out) +
                                                   (size_t)row * g.ldo + n0 + c);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = fmaxf(run[32 * h + 8 * j + e], 0.f);
                o4[j] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                   pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
              }
            }
          }
        }
      } else if (EPI == TC_EPI_STORE_T_PAIRS_F32) {
        // columns (2j, 2j+1) hold batch row j's hi and lo terms: fold them
        float* o = static_cast<float*>(g.out) + (size_t)seg * g.out_seg + orow0 + 32 * q + lane;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int col = n0 + c + 2 * j;
              if (col < g.N)
                o[(size_t)(col >> 1) * g.ldo] = __uint_as_float(v[2 * j]) + __uint_as_float(v[2 * j + 1]);
            }
          }
        }
      } else if (EPI == TC_EPI_STORE_T_F32) {
        // thread = one output row, 32 consecutive batch columns per TMEM load;
        // across the warp the stores to one batch column are contiguous
        float* o = static_cast<float*>(g.out) + (size_t)seg * g.out_seg + orow0 + 32 * q + lane;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n0 + c + j < g.N) o[(size_t)(n0 + c + j) * g.ldo] = __uint_as_float(v[j]);
          }
        }
      } else if (EPI == TC_EPI_STORE_F32) {
        float* o = static_cast<float*>(g.out) + (size_t)seg * g.out_seg + (size_t)row * g.ldo + n0;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_wait_ld();
          if (row_ok && n0 + c < g.N) {
            float4* o4 = reinterpret_cast<float4*>(o + c);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              o4[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                  __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          }
        }
      } else if (EPI == TC_EPI_RELU_BF16) {
        uint16_t* o = static_cast<uint16_t*>(g.out) + (size_t)row * g.ldo + n0;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_wait_ld();
          if (row_ok && n0 + c < g.N) {
            uint4* o4 = reinterpret_cast<uint4*>(o + c);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) f[e] = fmaxf(__uint_as_float(v[8 * j + e]), 0.f);
              o4[j] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                 pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
            }
          }
        }
      } else {  // TC_EPI_SWIGLU_BF16: columns [0,128) = X W1^T, [128,256) = X W3^T
        uint16_t* o = static_cast<uint16_t*>(g.out) + (size_t)row * g.ldo + n0;
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t a[32], b[32];
          tmem_ld32(taddr + c, a);
          tmem_ld32(taddr + BN / 2 + c, b);
          tmem_wait_ld();
          if (row_ok && n0 + c < g.N) {
            uint4* o4 = reinterpret_cast<uint4*>(o + c);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float z = __uint_as_float(a[8 * j + e]);
                f[e] = z / (1.0f + expf(-z)) * __uint_as_float(b[8 * j + e]);
              }
              o4[j] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                 pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3D map over a bf16 row-major matrix whose first nseg*K columns are nseg
// segments of K: dims {K, nseg, rows}, strides {K*2, ld*2} bytes (the matrix's
// own memory order), box = 64 elements (128 bytes) x 1 segment x box_rows,
// 128-byte swizzle, zero fill outside (so a partial last K block of a segment
// reads zeros, not the next segment).
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int nseg, int64_t K, int64_t ld,
              int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t gdim[3] = {(cuuint64_t)K, (cuuint64_t)nseg, (cuuint64_t)rows};
  cuuint64_t gstride[2] = {(cuuint64_t)K * 2, (cuuint64_t)ld * 2};
  cuuint32_t box[3] = {(cuuint32_t)BK, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstride, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// A row-major matrix [rows, ld] of esize-byte elements (bf16, or int8 codes) as a 3D
// tensor {chunk, ld / chunk, rows} (its own
// memory order, no swizzle), box {chunk, nchunk, box_rows}: one box is box_rows
// consecutive rows of nchunk * chunk columns, landing in shared memory row-major
// (rows of nchunk * chunk elements, nothing between them). Zero fill outside.
bool make_tensor_map_rows(CUtensorMap* m, const void* base, uint64_t rows, uint64_t ld, int chunk,
                          int nchunk, int box_rows, int esize) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || ld % chunk != 0 || (esize != 1 && esize != 2)) return false;
  cuuint64_t gdim[3] = {(cuuint64_t)chunk, (cuuint64_t)(ld / chunk), (cuuint64_t)rows};
  cuuint64_t gstride[2] = {(cuuint64_t)chunk * esize, (cuuint64_t)ld * esize};
  cuuint32_t box[3] = {(cuuint32_t)chunk, (cuuint32_t)nchunk, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
             const_cast<void*>(base), gdim, gstride, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D map over a bf16 row-major matrix [rows, cols] (row stride ld elements),
// box = box_cols x box_rows with the 128-byte swizzle, zero fill outside.
bool make_tensor_map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                        uint64_t ld, int box_cols, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <int BN, int EPI, int EW = 4>
int launch_cfg(const CUtensorMap* mA, const CUtensorMap& mB, const CUtensorMap& mB2,
               const TcGemm& g, const TcTiles& tt, cudaStream_t s) {
  constexpr int smem = TcCfg<BN>::SMEM_BYTES;
  if (set_smem_once((const void*)k_tc_gemm<BN, EPI, EW>, smem)) return TP_ECUDA;
  // with the segment sum a CTA takes every segment of an output tile
  const int units =
      EPI == TC_EPI_SEGSUM_F32 || EPI == TC_EPI_SEGSUM_RELU_BF16 ? tt.ntiles / g.nseg : tt.ntiles;
  const int grid = units < num_sms() ? units : num_sms();
  return launch_pdl(k_tc_gemm<BN, EPI, EW>, dim3(grid), dim3(tc_threads(EW)), smem, s, mA[0], mA[1], mA[2], mB,
                    mB2, g, tt);
}

}  // namespace

int launch_tc_gemm(const TcGemm& g, cudaStream_t s) {
  if (g.nA < 1 || g.nA > 3 || g.N < 1 || g.K < 8 || g.K % 8 != 0 || g.nseg < 1) return TP_EINVAL;
  if (g.lda % 8 != 0 || g.ldb % 8 != 0) return TP_EINVAL;
  if ((int64_t)g.nseg * g.K > g.lda || (int64_t)g.nseg * g.K > g.ldb) return TP_EINVAL;
  const bool swiglu = g.epi == TC_EPI_SWIGLU_BF16;
  const bool trans = g.epi == TC_EPI_STORE_T_F32 || g.epi == TC_EPI_STORE_T_PAIRS_F32;
  if (swiglu && !g.B2) return TP_EINVAL;
  if (!trans && (g.N % 32 != 0 || g.ldo % 8 != 0 || g.nA != 1)) return TP_EINVAL;
  if (trans && g.N > 128) return TP_EINVAL;
  if (g.epi == TC_EPI_STORE_T_PAIRS_F32 && (g.N & 1)) return TP_EINVAL;
  const bool segsum = g.epi == TC_EPI_SEGSUM_F32 || g.epi == TC_EPI_SEGSUM_RELU_BF16;
  // the segment sum keeps a row's BN running sums in registers: 128 columns per tile
  const int BN = trans ? (g.N <= 32 ? 32 : (g.N <= 64 ? 64 : 128)) : (segsum ? 128 : 256);
  CUtensorMap mA[3], mB, mB2;
  TcTiles tt{};
  tt.mt_off[0] = 0;
  for (int j = 0; j < 3; ++j) {
    const int jj = j < g.nA ? j : 0;
    if (g.Am[jj] < 1) return TP_EINVAL;
    if (!make_map(&mA[j], g.A[jj], g.Am[jj], g.nseg, g.K, g.lda, BM)) return TP_ECUDA;
    tt.mt_off[j + 1] = tt.mt_off[j] + (j < g.nA ? (g.Am[j] + BM - 1) / BM : 0);
  }
  const int brows = swiglu ? BN / 2 : BN;
  if (!make_map(&mB, g.B, g.N, g.nseg, g.K, g.ldb, brows) ||
      !make_map(&mB2, swiglu ? g.B2 : g.B, g.N, g.nseg, g.K, g.ldb, brows))
    return TP_ECUDA;
  const int nout = swiglu ? BN / 2 : BN;
  tt.num_n = (g.N + nout - 1) / nout;
  const int64_t nt = (int64_t)tt.mt_off[3] * tt.num_n * g.nseg;
  if (nt > 0x7fffffff) return TP_EINVAL;
  tt.ntiles = (int)nt;
  if (g.epi == TC_EPI_STORE_T_PAIRS_F32) {
    if (BN == 32) return launch_cfg<32, TC_EPI_STORE_T_PAIRS_F32>(mA, mB, mB2, g, tt, s);
    if (BN == 64) return launch_cfg<64, TC_EPI_STORE_T_PAIRS_F32>(mA, mB, mB2, g, tt, s);
    return launch_cfg<128, TC_EPI_STORE_T_PAIRS_F32>(mA, mB, mB2, g, tt, s);
  }
  if (trans) {
    if (BN == 32) return launch_cfg<32, TC_EPI_STORE_T_F32>(mA, mB, mB2, g, tt, s);
    if (BN == 64) return launch_cfg<64, TC_EPI_STORE_T_F32>(mA, mB, mB2, g, tt, s);
    return launch_cfg<128, TC_EPI_STORE_T_F32>(mA, mB, mB2, g, tt, s);
  }
  switch (g.epi) {
    case TC_EPI_STORE_F32: return launch_cfg<256, TC_EPI_STORE_F32>(mA, mB, mB2, g, tt, s);
    case TC_EPI_RELU_BF16: return launch_cfg<256, TC_EPI_RELU_BF16>(mA, mB, mB2, g, tt, s);
    case TC_EPI_SWIGLU_BF16: return launch_cfg<256, TC_EPI_SWIGLU_BF16>(mA, mB, mB2, g, tt, s);
    case TC_EPI_SEGSUM_F32:
      return g.quant ? launch_cfg<128, TC_EPI_SEGSUM_F32, 8>(mA, mB, mB2, g, tt, s)
                     : launch_cfg<128, TC_EPI_SEGSUM_F32>(mA, mB, mB2, g, tt, s);
    case TC_EPI_SEGSUM_RELU_BF16:
      return g.quant ? launch_cfg<128, TC_EPI_SEGSUM_RELU_BF16, 8>(mA, mB, mB2, g, tt, s)
                     : launch_cfg<128, TC_EPI_SEGSUM_RELU_BF16>(mA, mB, mB2, g, tt, s);
    default: return TP_EINVAL;
  }
}

}  // namespace tp
