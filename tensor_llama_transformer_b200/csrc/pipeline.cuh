// Device helpers of the streaming kernels: bounded mbarrier waits, bulk and
// tensor (TMA) copies into shared memory, warp-level bf16 MMA with ldmatrix,
// and the packed float32x2 dot-product step of the GEMVs.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace tp {

constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // every wait gives up after 2 s

TP_DEV uint32_t s2u(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

TP_DEV uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

TP_DEV void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(s2u(b)), "r"(count) : "memory");
}

TP_DEV void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

TP_DEV void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(s2u(b)), "r"(bytes)
               : "memory");
}

TP_DEV void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(s2u(b)) : "memory");
}

TP_DEV bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(s2u(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase of parity `parity` to complete; gives up after
// kWaitTimeoutNs, raising the error word (nullable) instead of hanging.
TP_DEV bool mbar_wait(uint64_t* b, uint32_t parity, int* err) {
  if (mbar_try(b, parity)) return true;
  const uint64_t t0 = gtimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try(b, parity)) return true;
    if ((i & 255) == 0 && gtimer() - t0 > kWaitTimeoutNs) {
      if (err) atomicExch(err, 1);
      return false;
    }
  }
}

// Contiguous global -> shared copy, completion counted on `bar` (16-byte
// aligned addresses, size a multiple of 16).
TP_DEV void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          s2u(dst)),
      "l"(src), "r"(bytes), "r"(s2u(bar))
      : "memory");
}

// L2 policy for data read once per step (weights, the KV cache): evict first,
// so that streaming them does not push the small, reused activations out of L2.
TP_DEV uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// bulk_g2s with an L2 cache policy.
TP_DEV void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(s2u(dst)),
      "l"(src), "r"(bytes), "r"(s2u(bar)), "l"(pol)
      : "memory");
}

// Prefetch of a contiguous global range into L2 (16-byte aligned, size a
// multiple of 16); no completion to wait for.
TP_DEV void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// One box of a 2D tensor map at element coordinates (x, y) -> shared memory.
TP_DEV void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(s2u(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(s2u(bar))
      : "memory");
}

// tma_load_2d with an L2 cache policy.
TP_DEV void tma_load_2d_hint(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                             uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(s2u(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(s2u(bar)), "l"(pol)
      : "memory");
}

// One box of a 3D tensor map at element coordinates (x, y, z) -> shared memory.
TP_DEV void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3, %4}], [%5];" ::"r"(s2u(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(s2u(bar))
      : "memory");
}

// tma_load_3d with an L2 cache policy.
TP_DEV void tma_load_3d_hint(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar,
                             uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(s2u(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(s2u(bar)), "l"(pol)
      : "memory");
}

// Named barrier 1 among the consumer warps of a warp-specialised CTA.
TP_DEV void consumers_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

TP_DEV void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

TP_DEV void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D (16x8 float32) += A (16x16 bf16, row-major) * B (16x8 bf16, column-major)
TP_DEV void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3},"
      " {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

TP_DEV uint32_t pack_bf16x2(uint16_t first, uint16_t second) {
  return (uint32_t)first | ((uint32_t)second << 16);
}

// acc (two float32 lanes as one 64-bit register pair) += the 8 bf16 weights of
// w times the 8 activations (lo = elements 0..3, hi = 4..7), two weights per
// packed fma.rn.f32x2: lane 0 of acc collects the even elements, lane 1 the odd.
TP_DEV void fma8(uint64_t& acc, const uint4 w, const float4 lo, const float4 hi) {
  const uint64_t x01 = ((uint64_t)__float_as_uint(lo.y) << 32) | __float_as_uint(lo.x);
  const uint64_t x23 = ((uint64_t)__float_as_uint(lo.w) << 32) | __float_as_uint(lo.z);
  const uint64_t x45 = ((uint64_t)__float_as_uint(hi.y) << 32) | __float_as_uint(hi.x);
  const uint64_t x67 = ((uint64_t)__float_as_uint(hi.w) << 32) | __float_as_uint(hi.z);
  asm("{\n .reg .b64 w;\n"
      " mov.b64 w, {%5, %6};  fma.rn.f32x2 %0, w, %1, %0;\n"
      " mov.b64 w, {%7, %8};  fma.rn.f32x2 %0, w, %2, %0;\n"
      " mov.b64 w, {%9, %10}; fma.rn.f32x2 %0, w, %3, %0;\n"
      " mov.b64 w, {%11, %12}; fma.rn.f32x2 %0, w, %4, %0;\n}"
      : "+l"(acc)
      : "l"(x01), "l"(x23), "l"(x45), "l"(x67), "r"(w.x << 16), "r"(w.x & 0xFFFF0000u),
        "r"(w.y << 16), "r"(w.y & 0xFFFF0000u), "r"(w.z << 16), "r"(w.z & 0xFFFF0000u),
        "r"(w.w << 16), "r"(w.w & 0xFFFF0000u));
}

// fma8 over two accumulators (elements 0-1 and 4-5 into a, 2-3 and 6-7 into b),
// halving the dependent chain per vector; the caller adds hsum2(a) + hsum2(b).
TP_DEV void fma8_2(uint64_t& a, uint64_t& b, const uint4 w, const float4 lo, const float4 hi) {
  const uint64_t x01 = ((uint64_t)__float_as_uint(lo.y) << 32) | __float_as_uint(lo.x);
  const uint64_t x23 = ((uint64_t)__float_as_uint(lo.w) << 32) | __float_as_uint(lo.z);
  const uint64_t x45 = ((uint64_t)__float_as_uint(hi.y) << 32) | __float_as_uint(hi.x);
  const uint64_t x67 = ((uint64_t)__float_as_uint(hi.w) << 32) | __float_as_uint(hi.z);
  asm("{\n .reg .b64 w;\n"
      " mov.b64 w, {%6, %7};  fma.rn.f32x2 %0, w, %2, %0;\n"
      " mov.b64 w, {%8, %9};  fma.rn.f32x2 %1, w, %3, %1;\n"
      " mov.b64 w, {%10, %11}; fma.rn.f32x2 %0, w, %4, %0;\n"
      " mov.b64 w, {%12, %13}; fma.rn.f32x2 %1, w, %5, %1;\n}"
      : "+l"(a), "+l"(b)
      : "l"(x01), "l"(x23), "l"(x45), "l"(x67), "r"(w.x << 16), "r"(w.x & 0xFFFF0000u),
        "r"(w.y << 16), "r"(w.y & 0xFFFF0000u), "r"(w.z << 16), "r"(w.z & 0xFFFF0000u),
        "r"(w.w << 16), "r"(w.w & 0xFFFF0000u));
}

TP_DEV float hsum2(uint64_t acc) {
  return __uint_as_float((uint32_t)acc) + __uint_as_float((uint32_t)(acc >> 32));
}

// Sums each of R values (R = 2, 4, 8) over the warp's 32 lanes with
// log2(R) exchange steps that halve the values a lane holds, then a butterfly
// over the remaining lanes: 5 + R/2 - 1 shuffles in all instead of 5 R. Lane l
// returns the total of value l / (32 / R).
template <int R>
TP_DEV float warp_sum_multi(float (&v)[R], int lane) {
#pragma unroll
  for (int k = 0; (1 << k) < R; ++k) {
    const int m = 16 >> k, half = R >> (k + 1);
    const bool up = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = up ? v[i] : v[i + half];
      const float keep = up ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
  float t = v[0];
#pragma unroll
  for (int m = 32 / R / 2; m >= 1; m >>= 1) t += __shfl_xor_sync(0xffffffffu, t, m);
  return t;
}

// The GEMV consumer step for one warp and one ring stage (rows cur .. end-1 of
// the CTA's range, stored from `stage`, row_bytes each): with PW = 2, row pairs
// pw and pw + 8 of the stage; with PW = 1, pair pw, or 1/Q of it (vectors
// [vb, ve) of 8 elements) when Q > 1. Each row is dotted with the NB staged
// activation rows (xs: lo halves [NB][nv], then hi halves) with packed FMA, and
// the warp's 2 PW NB sums are reduced in one butterfly:
//   res[((r + row) NB + b) Q + part] = sum.
template <int NB, int PW>
TP_DEV void ring_pairs_dot(const uint8_t* stage, int cur, int end, const float4* xs, float* res,
                           int nv, uint32_t rb, int pw, int part, int Q, int vb, int ve, int lane) {
  constexpr int R = 2 * PW * NB;  // values: (pair j, row, batch row)
  int rr[PW];
  bool valid[PW];
  const uint4* wr[PW];
#pragma unroll
  for (int j = 0; j < PW; ++j) {
    rr[j] = cur + 2 * (pw + 8 * j);
    valid[j] = rr[j] < end;
    wr[j] = reinterpret_cast<const uint4*>(stage + (size_t)(rr[j] - cur) * rb);
  }
  if (!valid[0]) return;  // pairs are filled in order: no pair for this warp
  uint64_t acc[R][2];
#pragma unroll
  for (int i = 0; i < R; ++i) acc[i][0] = acc[i][1] = 0ull;
#pragma unroll 4
  for (int v = vb + lane; v < ve; v += 32) {
    float4 lo[NB], hi[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      lo[b] = xs[b * nv + v];
      hi[b] = xs[(NB + b) * nv + v];
    }
#pragma unroll
    for (int j = 0; j < PW; ++j) {
      if (!valid[j]) continue;
      const uint4 u0 = wr[j][v], u1 = wr[j][nv + v];
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        fma8_2(acc[(2 * j) * NB + b][0], acc[(2 * j) * NB + b][1], u0, lo[b], hi[b]);
        fma8_2(acc[(2 * j + 1) * NB + b][0], acc[(2 * j + 1) * NB + b][1], u1, lo[b], hi[b]);
      }
    }
  }
  float val[R];
#pragma unroll
  for (int i = 0; i < R; ++i) val[i] = hsum2(acc[i][0]) + hsum2(acc[i][1]);
  const float tot = warp_sum_multi<R>(val, lane);
  constexpr int kLanes = 32 / R;  // lanes holding each total
  if ((lane & (kLanes - 1)) == 0) {
    const int i = lane / kLanes, j = i / (2 * NB), row = (i / NB) & 1, b = i % NB;
    if (valid[j]) res[((size_t)(rr[j] + row) * NB + b) * Q + part] = tot;
  }
}

// Shared address of 16-byte chunk c (8 dims, 0..15) of row t of a 64-row K or
// V tile that TMA wrote as two boxes of 64 rows x 64 dims (8 KB each, the first
// for dims 0..63) with the 128-byte swizzle; base must be 1024-byte aligned.
TP_DEV uint32_t kv_tile_addr(uint32_t base, int t, int c) {
  return base + (uint32_t)((c >> 3) * 8192 + t * 128 + (((c & 7) ^ (t & 7)) << 4));
}

}  // namespace tp
