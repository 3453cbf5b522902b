// dca_softmax.cuh -- device helpers shared by the tcgen05 attention kernels:
// bf16 packing, the software exp2 of part of the scores, query-row rotation
// into the 128-byte-swizzled operand tile, and the exchange between the two
// threads of a row.
#pragma once
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "dca_plan.cuh"
#include "sm100_ptx.cuh"

// How the two threads of a row wait for each other's half-row maximum:
// polling (no suspension) -- on the critical path of every item.
#ifndef DCA_PAIR_WAIT
#define DCA_PAIR_WAIT wait_poll
#endif

namespace dca {
namespace attn {

constexpr int HALF_BYTES = 16384;  // 128 rows x 64 bf16 (one 128-byte swizzle column block)

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Software 2^x for a pair of arguments x <= 8, on the FMA and ALU pipes, to
// take part of the exponentials off the MUFU pipe (at d = 128 one MUFU ex2
// per score costs as much SM time as the score's tensor-core work).
// Method: x = n + f with n = round(x) (adding 1.5 * 2^23 rounds to an integer
// in fp32) and f in [-1/2, 1/2]; 2^f by a degree-3 polynomial fitted for
// minimum relative error with the Remez exchange (exp2_poly_fit.py next to
// this file: max relative error 7.5e-5, below the 2^-9 half-ulp of the bf16 P);
// 2^n added to the exponent field.  Arguments below -126 are clamped (result
// ~0, as for the hardware path).
constexpr float EXP2_C0 = 0.9999280571937561f;
constexpr float EXP2_C1 = 0.6932609677314758f;
constexpr float EXP2_C2 = 0.2426111251115799f;
constexpr float EXP2_C3 = 0.0551716685295105f;

__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  const float RND = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 t = add2(x, make_float2(RND, RND));
  const float2 n = add2(t, make_float2(-RND, -RND));
  const float2 f = fma2(n, make_float2(-1.0f, -1.0f), x);
  float2 q = fma2(make_float2(EXP2_C3, EXP2_C3), f, make_float2(EXP2_C2, EXP2_C2));
  q = fma2(q, f, make_float2(EXP2_C1, EXP2_C1));
  q = fma2(q, f, make_float2(EXP2_C0, EXP2_C0));
  // the integer n sits in the low mantissa bits of t; shifting by 23 moves it
  // into the exponent field (the constant part of t shifts out)
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

// The same software 2^x for one argument with the constants as instruction
// immediates (no registers held for them; the packed form above keeps six
// constant pairs in registers).
__device__ __forceinline__ float exp2_poly1(float x) {
  x = fmaxf(x, -126.0f);
  const float t = x + 12582912.0f;  // 1.5 * 2^23: rounds x to an integer n in t's low bits
  const float f = x - (t - 12582912.0f);
  float q = fmaf(EXP2_C3, f, EXP2_C2);
  q = fmaf(q, f, EXP2_C1);
  q = fmaf(q, f, EXP2_C0);
  return __uint_as_float(__float_as_uint(q) + (__float_as_uint(t) << 23));
}

// Of every 8 score pairs of a row, this many take the software exp2.
#ifndef DCA_EXP2_POLY_PAIRS
#define DCA_EXP2_POLY_PAIRS 2
#endif

// Rotate one query row by the positions of table row `trow` and write it to
// the 128-byte-swizzled K-major operand tile (two 16 KiB column blocks: dims
// 0-63 and 64-127; RoPE pairs (k, k+64) sit at the same offset of each block).
__device__ __forceinline__ void write_q_row(uint8_t* qb, int r, const __nv_bfloat16* qrow,
                                            const float2* trow, int c0 = 0, int c1 = 8) {
  const uint32_t row_off = static_cast<uint32_t>(r) * 128u;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    if (c < c0 || c >= c1) continue;
    uint4 oa = make_uint4(0, 0, 0, 0), ob = oa;
    if (qrow != nullptr) {
      const uint4 xa = *reinterpret_cast<const uint4*>(qrow + 8 * c);
      const uint4 xb = *reinterpret_cast<const uint4*>(qrow + 64 + 8 * c);
      const float4* t4 = reinterpret_cast<const float4*>(trow + 8 * c);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&xa);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xb);
      uint32_t* pa = reinterpret_cast<uint32_t*>(&oa);
      uint32_t* pb = reinterpret_cast<uint32_t*>(&ob);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 t = t4[e];
        const float2 x = __bfloat1622float2(a2[e]);
        const float2 y = __bfloat1622float2(b2[e]);
        pa[e] = pack_bf16(x.x * t.x - y.x * t.y, x.y * t.z - y.y * t.w);
        pb[e] = pack_bf16(x.x * t.y + y.x * t.x, x.y * t.w + y.y * t.z);
      }
    }
    const uint32_t phys = static_cast<uint32_t>((c ^ (r & 7)) * 16);
    *reinterpret_cast<uint4*>(qb + row_off + phys) = oa;
    *reinterpret_cast<uint4*>(qb + HALF_BYTES + row_off + phys) = ob;
  }
}

// Maximum of 64 scores: eight independent chains of three-input maxima.
__device__ __forceinline__ float max64(const uint32_t* sv) {
  float m8[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) m8[c] = __uint_as_float(sv[c]);
#pragma unroll
  for (int e = 8; e < 64; e += 16) {
#pragma unroll
    for (int c = 0; c < 8; ++c)
      m8[c] = max3f(m8[c], __uint_as_float(sv[e + c]),
                    e + 8 + c < 64 ? __uint_as_float(sv[e + 8 + c]) : m8[c]);
  }
  return max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
}

// Exchange one float with the thread that holds the other half of the same
// row (same lane, warp +/- 4) through shared memory and the pair's mbarrier
// (one arrival per warp).  Phase `ph` alternates two buffers: a thread can be
// at most one exchange ahead of its partner, so a buffer is rewritten only
// after the partner has read it.  Bounded like every wait of the kernel.
struct PairCtx {
  float* xval;      // [2][2][128]
  uint64_t* bar;    // this lane quarter's pair barrier
  uint32_t ph;      // exchanges done so far
  int half, r, lane;
};

__device__ __forceinline__ bool pair_exchange(PairCtx& pc, float mine, float& other,
                                              volatile int* abort, unsigned int* status,
                                              uint64_t timeout_ns, unsigned int code) {
  float* slot = pc.xval + (pc.ph & 1u) * 256u;
  slot[pc.half * 128 + pc.r] = mine;
  __syncwarp();
  if (pc.lane == 0) mbar_arrive(pc.bar);
  bool ok = DCA_PAIR_WAIT(pc.bar, pc.ph & 1u, abort, status, timeout_ns, code);
  ok = __all_sync(0xffffffffu, ok);
  if (ok) other = slot[(1 - pc.half) * 128 + pc.r];
  ++pc.ph;
  return ok;
}

// Exponentials of 64 scores against the reference `mb` (= m_ref * sc):
// P (bf16 pairs) into pk, their sum returned.
__device__ __forceinline__ float exp_pack64(const uint32_t* sv, float sc, float mb, uint32_t* pk) {
  const float2 sc2 = make_float2(sc, sc);
  const float2 nmb2 = make_float2(-mb, -mb);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    float2 x = fma2(make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), sc2,
                    nmb2);
    if ((e & 7) < DCA_EXP2_POLY_PAIRS) {
      x = exp2_poly2(x);
    } else {
      x.x = ex2_approx(x.x);
      x.y = ex2_approx(x.y);
    }
    acc[e & 3] = add2(acc[e & 3], x);
    pk[e] = pack_bf16(x.x, x.y);
  }
  const float2 a = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
  return a.x + a.y;
}

}  // namespace attn
}  // namespace dca
