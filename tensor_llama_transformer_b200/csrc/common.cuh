// Shared device helpers for the tensor-parallel block kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/tp_block.h"

#define TP_DEV __device__ __forceinline__

namespace tp {

constexpr int kQ8Block = 32;
constexpr int kHeadDim = 128;

// ---------------------------------------------------------------- bf16 unpack
// A bf16 value is the upper half of a float32, so widening is a shift.
TP_DEV float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
TP_DEV float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

TP_DEV uint16_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

// A float32 value as two bf16 terms, hi = bf16(v) and lo = bf16(v - hi): v - hi
// is exact in float32, so hi + lo carries about 16 significant bits. Operands of
// the tensor-core decode path are fed as such pairs (rows 2b and 2b+1).
TP_DEV void bf16_split(float v, uint16_t& hi, uint16_t& lo) {
  hi = f32_to_bf16_bits(v);
  lo = f32_to_bf16_bits(v - __uint_as_float(((uint32_t)hi) << 16));
}

// 16-byte streaming load that bypasses L1 (weights are read once per launch).
TP_DEV uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ---------------------------------------------------------------- reductions
TP_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
TP_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum; `red` must hold >= 32 floats. All threads get the result.
TP_DEV float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = lane < nw ? red[lane] : 0.f;
  return warp_sum(t);
}
TP_DEV float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = lane < nw ? red[lane] : -INFINITY;
  return warp_max(t);
}

// ---------------------------------------------------------------- Q8 codec
// Int8 block quantisation of a sync buffer, 32 values per block, one float32
// scale (the Quantize*/Dequantize* tasks of the distributed-llama list; the
// format is int8 + fp32 scale, d = amax/127, codes = x/d rounded half away
// from zero). Every step is one IEEE round-to-nearest float32 operation, so
// the codes are reproducible bit for bit on any IEEE machine.
TP_DEV float q8_scale(float amax) { return __fdiv_rn(amax, 127.0f); }

// The correctly rounded quotient, out of line: the codecs below take it only for the
// rare values near a rounding tie (and for scales outside [2^-120, 2^120]), so one copy
// of its code serves every caller instead of one inlined per value of an unrolled loop.
static __device__ __noinline__ float q8_div_rn(float x, float d) { return __fdiv_rn(x, d); }

// The code is round(fl(x / d)) with fl the correctly rounded quotient. The
// quotient is first taken with the fast division __fdividef (at most 2 ulp from
// x / d for d in the normal range, so at most 2.5 ulp from fl(x / d)); since
// |x| <= amax gives |x / d| < 128, that is below 2e-5 in absolute terms, and
// rounding to an integer can only differ from rounding fl(x / d) when the
// quotient lies that close to a tie k + 1/2. Only then (and for d outside
// [2^-120, 2^120]) is the correctly rounded division taken.
TP_DEV int q8_code(float x, float d) {
  if (d == 0.0f) return 0;
  float q;
  if (d > 0x1p-120f && d < 0x1p120f) {
    q = __fdividef(x, d);
    const float a = fabsf(q);
    if (fabsf(a - truncf(a) - 0.5f) < 4e-5f) q = q8_div_rn(x, d);
  } else {
    q = q8_div_rn(x, d);
  }
  float v = roundf(q);  // roundf: halfway cases away from zero
  v = fminf(fmaxf(v, -127.0f), 127.0f);
  return (int)v;
}

TP_DEV float q8_value(int q, float d) { return __fmul_rn((float)q, d); }

// For many values of one block: the block's reciprocal r = 1/d, correctly rounded
// (__frcp_rn), or 0 when d is outside [2^-120, 2^120] (every value of the block then
// takes the division).
TP_DEV float q8_recip(float d) { return d > 0x1p-120f && d < 0x1p120f ? __frcp_rn(d) : 0.f; }

// q8_code(x, d) as an integral float (+0 for a zero code), from q = x * r with
// r = q8_recip(d): two correctly rounded steps put q within 2^-23 relative of the exact
// x / d, and |x / d| <= 127.0001, so q is within 1.6e-5 of x / d and within 2e-5 of
// fl(x / d) (half an ulp below 128 is 3.8e-6). Rounding q and fl(x / d) to an integer
// can then differ only when one of them lies within 2e-5 of a tie k + 1/2, and there
// the correctly rounded division is taken instead (window 4e-5, as in q8_code).
TP_DEV float q8_code_rf(float x, float d, float r) {
  if (d == 0.0f) return 0.f;
  float q;
  if (r != 0.f) {
    q = __fmul_rn(x, r);
    const float a = fabsf(q);
    if (fabsf(a - truncf(a) - 0.5f) < 4e-5f) q = q8_div_rn(x, d);
  } else {
    q = q8_div_rn(x, d);
  }
  // roundf: halfway cases away from zero; + 0 turns a -0 code into +0
  return fminf(fmaxf(roundf(q), -127.0f), 127.0f) + 0.0f;
}

// The Q8 round trip of N values of N different blocks, value i with its block's scale
// d[i] (a merge's slices): one branch for all of them, as in q8_codes below; the result
// is q8_value(q8_code(p[i], d[i]), d[i]) bit for bit.
template <int N>
TP_DEV void q8_roundtrip_each(float* p, const float* d);

// The codes of N values of one block (q8_code_rf of each, bit for bit) without a branch
// per value: every quotient q = x * r is formed first, with one flag for "some q lies
// within 4e-5 of a tie, or the scale is outside [2^-120, 2^120]". Without it (nearly
// always), round half away from zero is trunc(q + copysign(1/2, q)): for |q| < 128 the
// sum is off by at most 3.8e-6, so it cannot cross an integer when q is at least 4e-5
// from a tie. With it, every value takes q8_code_rf. c may be x (codes in place).
template <int N>
TP_DEV void q8_codes(const float* x, float* c, float d, float r) {
  bool near = !(r != 0.f);
  float q[N];
#pragma unroll
  for (int i = 0; i < N; ++i) {
    q[i] = __fmul_rn(x[i], r);
    const float a = fabsf(q[i]);
    near |= fabsf(a - truncf(a) - 0.5f) < 4e-5f;
  }
  if (!near) {
#pragma unroll
    for (int i = 0; i < N; ++i)
      c[i] = fminf(fmaxf(truncf(__fadd_rn(q[i], copysignf(0.5f, q[i]))), -127.0f), 127.0f) + 0.0f;
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) c[i] = q8_code_rf(x[i], d, r);
  }
}

// q8_codes for G blocks at once (block g: x[g N .. g N + N - 1] with scale d[g] and
// reciprocal r[g]), with one near flag over all of them, so that their chains can run
// side by side; the codes are q8_code_rf's, bit for bit, as for q8_codes.
template <int N, int G>
TP_DEV void q8_codes_g(const float* x, float* c, const float* d, const float* r) {
  bool near = false;
  float q[G * N];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    near |= !(r[g] != 0.f);
#pragma unroll
    for (int i = 0; i < N; ++i) {
      q[g * N + i] = __fmul_rn(x[g * N + i], r[g]);
      const float a = fabsf(q[g * N + i]);
      near |= fabsf(a - truncf(a) - 0.5f) < 4e-5f;
    }
  }
  if (!near) {
#pragma unroll
    for (int i = 0; i < G * N; ++i)
      c[i] = fminf(fmaxf(truncf(__fadd_rn(q[i], copysignf(0.5f, q[i]))), -127.0f), 127.0f) + 0.0f;
  } else {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int i = 0; i < N; ++i) c[g * N + i] = q8_code_rf(x[g * N + i], d[g], r[g]);
  }
}

template <int N>
TP_DEV void q8_roundtrip_each(float* p, const float* d) {
  bool near = false;
  float r[N], q[N];
#pragma unroll
  for (int i = 0; i < N; ++i) {
    r[i] = q8_recip(d[i]);
    q[i] = __fmul_rn(p[i], r[i]);
    const float a = fabsf(q[i]);
    near |= !(r[i] != 0.f) || fabsf(a - truncf(a) - 0.5f) < 4e-5f;
  }
  if (!near) {
#pragma unroll
    for (int i = 0; i < N; ++i)
      p[i] = __fmul_rn(
          fminf(fmaxf(truncf(__fadd_rn(q[i], copysignf(0.5f, q[i]))), -127.0f), 127.0f) + 0.0f, d[i]);
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) p[i] = __fmul_rn(q8_code_rf(p[i], d[i], r[i]), d[i]);
  }
}

// Quantise-dequantise of 4 consecutive values held by each of 8 consecutive
// lanes (one 32-value block per 8-lane group). All 32 lanes must call it.
TP_DEV void q8_roundtrip4(float4& v) {
  float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
  const float d = q8_scale(a);
  v.x = q8_value(q8_code(v.x, d), d);
  v.y = q8_value(q8_code(v.y, d), d);
  v.z = q8_value(q8_code(v.z, d), d);
  v.w = q8_value(q8_code(v.w, d), d);
}

// Quantise 4 values per lane (8-lane groups = one block): writes 4 codes; the
// group's first lane writes the scale. Returns the codes packed little-endian.
TP_DEV uint32_t q8_quantize4(float4 v, float* scale_out /* nullable */) {
  float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
  const float d = q8_scale(a), r = q8_recip(d);
  if (scale_out && (threadIdx.x & 7) == 0) *scale_out = d;
  const float xs[4] = {v.x, v.y, v.z, v.w};
  float cf[4];
  q8_codes<4>(xs, cf, d, r);
  const uint32_t c0 = (uint32_t)((int)cf[0] & 0xFF), c1 = (uint32_t)((int)cf[1] & 0xFF);
  const uint32_t c2 = (uint32_t)((int)cf[2] & 0xFF), c3 = (uint32_t)((int)cf[3] & 0xFF);
  return c0 | (c1 << 8) | (c2 << 16) | (c3 << 24);
}

TP_DEV float4 q8_unpack4(uint32_t codes, float d) {
  float4 r;
  r.x = q8_value((int)(int8_t)(codes & 0xFF), d);
  r.y = q8_value((int)(int8_t)((codes >> 8) & 0xFF), d);
  r.z = q8_value((int)(int8_t)((codes >> 16) & 0xFF), d);
  r.w = q8_value((int)(int8_t)((codes >> 24) & 0xFF), d);
  return r;
}

// ---------------------------------------------------------------- PDL
// Programmatic dependent launch: a kernel lets the next kernel of the stream be
// scheduled as soon as all its CTAs have started (launch_dependents), and a
// kernel waits for its predecessor's completion and memory (wait) only where it
// first touches data the predecessor produced. Work before the wait may only
// read inputs no earlier kernel writes (weights, pos, cache rows before pos).
TP_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
TP_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace tp

// ---------------------------------------------------------------- host side
#define TP_CUDA_TRY(expr)                       \
  do {                                          \
    cudaError_t err__ = (expr);                 \
    if (err__ != cudaSuccess) return TP_ECUDA;  \
  } while (0)

#define TP_LAUNCH_CHECK()                                        \
  do {                                                           \
    if (cudaGetLastError() != cudaSuccess) return TP_ECUDA;      \
  } while (0)

namespace tp {
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Whether launches carry the programmatic-serialization attribute (default on;
// the environment variable TP_PDL=0 turns it off, for comparison runs).
bool pdl_enabled();

// Launches `kernel` on `s`, allowing it to overlap its predecessor's tail
// (programmatic dependent launch) when pdl_enabled().
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
               Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess ? TP_OK
                                                                                       : TP_ECUDA;
}
int device_check();   // TP_OK if the current device is sm_100 (cached per device)
int num_sms();        // SM count of the current device (cached)
// Raise a kernel's dynamic shared-memory limit once per (kernel, device); later
// calls are host-only lookups, so launches stay legal inside stream capture.
int set_smem_once(const void* kernel, int bytes);
}  // namespace tp
