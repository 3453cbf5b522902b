// dca_prep.cu -- preparation kernels of a DCA prefill call.
//
//  * rope_table_kernel: cos/sin of p * theta_k, theta_k = base^(-2k/d), for
//    every position a query or key can be rotated by.  Angles and sin/cos are
//    evaluated in float64 (positions reach c - 1 ~ 2.6e5 radians at k = 0,
//    where an fp32 product would already be off by ~1e-2 rad) and stored fp32.
//  * rotate_keys_kernel: k'_j = R(j mod s) k_j.  In DCA every key is rotated
//    by its periodic position j mod s whatever the query ("Qwen2.5-1M 不重训
//    外推 1M", section Inter-Chunk Attention; intra-chunk pairs use the same
//    key position), so each key is rotated once per call instead of once per
//    (query tile, head) that reads it.
// Both are memory-bound streaming kernels (grid-stride, 16-byte accesses).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dca_internal.h"

namespace dca {

__global__ void rope_table_kernel(float2* __restrict__ tab, int64_t T, int64_t n_direct,
                                  int64_t c, double base, int d) {
  const int half = d / 2;
  const int64_t total = T * half;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = idx / half;
    const int k = static_cast<int>(idx - row * half);
    const int64_t pos = row < n_direct ? row : c - 1;
    const double theta = pow(base, -2.0 * k / d);
    double sn, cs;
    sincos(static_cast<double>(pos) * theta, &sn, &cs);
    tab[idx] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
  }
}

// One thread per (key row j, KV head g, group of 8 rotation pairs); d = 128.
__global__ void rotate_keys_bf16_kernel(const __nv_bfloat16* __restrict__ k,
                                        __nv_bfloat16* __restrict__ kr,
                                        const float2* __restrict__ tab, int64_t j_begin,
                                        int64_t j_end, int Hkv, int64_t s) {
  constexpr int CH = 8;  // 64 pairs / 8 per 16-byte vector
  const int64_t total = (j_end - j_begin) * Hkv * CH;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int c = static_cast<int>(idx % CH);
    const int64_t rest = idx / CH;
    const int g = static_cast<int>(rest % Hkv);
    const int64_t j = j_begin + rest / Hkv;
    const int64_t pos = j % s;
    const int64_t base_off = (j * Hkv + g) * 128;
    const uint4 xa = *reinterpret_cast<const uint4*>(k + base_off + 8 * c);
    const uint4 xb = *reinterpret_cast<const uint4*>(k + base_off + 64 + 8 * c);
    const float4* t4 = reinterpret_cast<const float4*>(tab + pos * 64 + 8 * c);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&xa);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xb);
    uint4 oa, ob;
    __nv_bfloat162* oa2 = reinterpret_cast<__nv_bfloat162*>(&oa);
    __nv_bfloat162* ob2 = reinterpret_cast<__nv_bfloat162*>(&ob);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float4 t = t4[e];  // (cos, sin) of pairs 2e and 2e+1
      const float2 x = __bfloat1622float2(a2[e]);
      const float2 y = __bfloat1622float2(b2[e]);
      const float xa0 = x.x * t.x - y.x * t.y, xb0 = x.x * t.y + y.x * t.x;
      const float xa1 = x.y * t.z - y.y * t.w, xb1 = x.y * t.w + y.y * t.z;
      oa2[e] = __floats2bfloat162_rn(xa0, xa1);
      ob2[e] = __floats2bfloat162_rn(xb0, xb1);
    }
    *reinterpret_cast<uint4*>(kr + base_off + 8 * c) = oa;
    *reinterpret_cast<uint4*>(kr + base_off + 64 + 8 * c) = ob;
  }
}

__global__ void rotate_keys_f32_kernel(const float* __restrict__ k, float* __restrict__ kr,
                                       const float2* __restrict__ tab, int64_t j_begin,
                                       int64_t j_end, int Hkv, int64_t s) {
  constexpr int CH = 16;  // 64 pairs / 4 per 16-byte vector
  const int64_t total = (j_end - j_begin) * Hkv * CH;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int c = static_cast<int>(idx % CH);
    const int64_t rest = idx / CH;
    const int g = static_cast<int>(rest % Hkv);
    const int64_t j = j_begin + rest / Hkv;
    const int64_t pos = j % s;
    const int64_t base_off = (j * Hkv + g) * 128;
    const float4 x = *reinterpret_cast<const float4*>(k + base_off + 4 * c);
    const float4 y = *reinterpret_cast<const float4*>(k + base_off + 64 + 4 * c);
    const float4* t4 = reinterpret_cast<const float4*>(tab + pos * 64 + 4 * c);
    const float4 t01 = t4[0], t23 = t4[1];
    float4 oa, ob;
    oa.x = x.x * t01.x - y.x * t01.y;  ob.x = x.x * t01.y + y.x * t01.x;
    oa.y = x.y * t01.z - y.y * t01.w;  ob.y = x.y * t01.w + y.y * t01.z;
    oa.z = x.z * t23.x - y.z * t23.y;  ob.z = x.z * t23.y + y.z * t23.x;
    oa.w = x.w * t23.z - y.w * t23.w;  ob.w = x.w * t23.w + y.w * t23.z;
    *reinterpret_cast<float4*>(kr + base_off + 4 * c) = oa;
    *reinterpret_cast<float4*>(kr + base_off + 64 + 4 * c) = ob;
  }
}

static int grid_for(int64_t work, int threads) {
  int64_t blocks = (work + threads - 1) / threads;
  const int64_t cap = 148LL * 16;  // grid-stride beyond 16 blocks per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return static_cast<int>(blocks);
}

cudaError_t launch_rope_table(float2* tab, int64_t T, int64_t n_direct, int64_t c, double base,
                              int d, cudaStream_t st) {
  const int threads = 256;
  rope_table_kernel<<<grid_for(T * (d / 2), threads), threads, 0, st>>>(tab, T, n_direct, c,
                                                                         base, d);
  return cudaGetLastError();
}

cudaError_t launch_rotate_keys(const void* k, void* kr, const float2* tab, int64_t j_begin,
                               int64_t j_end, int Hkv, int64_t s, int dtype, cudaStream_t st) {
  if (j_end <= j_begin) return cudaSuccess;
  const int threads = 256;
  if (dtype == 0) {
    rotate_keys_bf16_kernel<<<grid_for((j_end - j_begin) * Hkv * 8, threads), threads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(k), static_cast<__nv_bfloat16*>(kr), tab, j_begin,
        j_end, Hkv, s);
  } else {
    rotate_keys_f32_kernel<<<grid_for((j_end - j_begin) * Hkv * 16, threads), threads, 0, st>>>(
        static_cast<const float*>(k), static_cast<float*>(kr), tab, j_begin, j_end, Hkv, s);
  }
  return cudaGetLastError();
}

}  // namespace dca
