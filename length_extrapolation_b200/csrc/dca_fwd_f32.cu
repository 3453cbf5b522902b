// dca_fwd_f32.cu -- Dual Chunk Attention forward in fp32 on CUDA cores.
//
// For fp32 inputs the result must hold 1e-4 relative accuracy, which rules
// out the tensor cores (tf32 keeps 10 mantissa bits: ~1e-3 logit error), so
// this kernel is plain FFMA.  Same tile plan as the tensor-core kernel
// (dca_plan.cuh) with 64-row query tiles and 64-key tiles:
//   block = one (64-row query tile, query head); 256 threads; thread t owns
//   rows 4*(t/16)+a (a < 4) and score columns (t%16)+16b (b < 4), output
//   columns (t%16)+16u (u < 8).  Row max / sum reduce over the 16 lanes of a
//   half-warp.
// Query rows are rotated in shared memory at each phase switch
// (INTER -> SUCC -> INTRA); keys arrive pre-rotated by j mod s.
#include <math.h>

#include "dca_internal.h"
#include "dca_plan.cuh"

namespace dca {
namespace f32k {

constexpr int BM = 64, BN = 64, HD = 128, THREADS = 256;
constexpr int KPAD = HD + 1;  // padded key rows: conflict-free column reads
constexpr int PPAD = BN + 1;
constexpr size_t SMEM_BYTES =
    sizeof(float) * (BM * HD + BN * KPAD + BN * HD + BM * PPAD);

struct Params {
  const float* q;
  const float* kr;
  const float* v;
  float* out;
  const float2* tab;
  int64_t q_start, Lq, Lk, s, w, tab_c1;
  int Hq, Hkv, G, n_qtiles;
  int reading;
  float scale_log2;
  float* lse;  // optional [Lq][Hq] natural-log LSE
};

__global__ void __launch_bounds__(THREADS) dca_fwd_f32_kernel(const Params p) {
  extern __shared__ float sm[];
  float* Qs = sm;                 // [BM][HD]
  float* Ks = Qs + BM * HD;       // [BN][KPAD]
  float* Vs = Ks + BN * KPAD;     // [BN][HD]
  float* Ps = Vs + BN * HD;       // [BM][PPAD]

  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x / p.Hq);  // longest first
  const int h = static_cast<int>(blockIdx.x % p.Hq);
  const int g = h / p.G;
  const int64_t i0 = p.q_start + static_cast<int64_t>(qt) * BM;
  const int64_t q_end = p.q_start + p.Lq;
  const int64_t i_last = (i0 + BM - 1 < q_end - 1) ? i0 + BM - 1 : q_end - 1;
  const int64_t i_hi = i0 + BM - 1;
  const TilePlan plan = make_plan(i0, i_last, p.s, p.w, BN, p.reading);

  const int t = threadIdx.x;
  const int rg = t >> 4, cg = t & 15;
  const float sc = p.scale_log2;

  float O[4][8];
  float m_run[4], l_run[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    m_run[a] = -INFINITY;
    l_run[a] = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) O[a][u] = 0.f;
  }

  int cur_cls = -1;
  for (int n = 0; n < plan.n_items; ++n) {
    int kt, cls;
    plan_item(plan, n, kt, cls);
    __syncthreads();  // previous tile fully consumed
    if (cls != cur_cls) {
      // rotate the query rows for this phase
      for (int idx = t; idx < BM * (HD / 2); idx += THREADS) {
        const int row = idx / (HD / 2), k = idx % (HD / 2);
        const int64_t i = i0 + row;
        float ya = 0.f, yb = 0.f;
        if (i <= i_last) {
          const float* qrow = p.q + ((i - p.q_start) * p.Hq + h) * static_cast<int64_t>(HD);
          const float2 cs = p.tab[query_table_row(i, cls, p.s, p.w, p.tab_c1) * (HD / 2) + k];
          const float x = qrow[k], y = qrow[k + HD / 2];
          ya = x * cs.x - y * cs.y;
          yb = x * cs.y + y * cs.x;
        }
        Qs[row * HD + k] = ya;
        Qs[row * HD + k + HD / 2] = yb;
      }
      cur_cls = cls;
    }
    const int64_t j0 = static_cast<int64_t>(kt) * BN;
    for (int idx = t; idx < BN * (HD / 4); idx += THREADS) {
      const int row = idx / (HD / 4), c4 = idx % (HD / 4);
      const int64_t j = j0 + row;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      if (j < p.Lk) {
        const int64_t off = (j * p.Hkv + g) * static_cast<int64_t>(HD) + 4 * c4;
        kv = *reinterpret_cast<const float4*>(p.kr + off);
        vv = *reinterpret_cast<const float4*>(p.v + off);
      }
      float* kd = Ks + row * KPAD + 4 * c4;
      kd[0] = kv.x; kd[1] = kv.y; kd[2] = kv.z; kd[3] = kv.w;
      *reinterpret_cast<float4*>(Vs + row * HD + 4 * c4) = vv;
    }
    __syncthreads();

    float S[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) S[a][b] = 0.f;
#pragma unroll 4
    for (int k = 0; k < HD; ++k) {
      float qa[4], kb[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) qa[a] = Qs[(4 * rg + a) * HD + k];
#pragma unroll
      for (int b = 0; b < 4; ++b) kb[b] = Ks[(cg + 16 * b) * KPAD + k];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) S[a][b] = fmaf(qa[a], kb[b], S[a][b]);
    }

    const bool full = item_is_full(i0, i_hi, j0, j0 + BN - 1, p.s, p.w, cls, p.reading);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int64_t i = i0 + 4 * rg + a;
      if (!full) {
        const int64_t ni = i / p.s;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int64_t j = j0 + cg + 16 * b;
          const bool valid = (j <= i) && (pair_class(ni - j / p.s, i - j, p.w, p.reading) == cls);
          if (!valid) S[a][b] = -INFINITY;
        }
      }
      float mx = fmaxf(fmaxf(S[a][0], S[a][1]), fmaxf(S[a][2], S[a][3]));
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m_run[a], mx);
      const float alpha = (m_new == -INFINITY) ? 1.f : exp2f((m_run[a] - m_new) * sc);
      const float mb = (m_new == -INFINITY) ? 0.f : m_new * sc;
      float rs = 0.f;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float pv = exp2f(fmaf(S[a][b], sc, -mb));
        rs += pv;
        Ps[(4 * rg + a) * PPAD + cg + 16 * b] = pv;
      }
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
      l_run[a] = l_run[a] * alpha + rs;
      m_run[a] = m_new;
#pragma unroll
      for (int u = 0; u < 8; ++u) O[a][u] *= alpha;
    }
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < BN; ++j) {
      float vj[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) vj[u] = Vs[j * HD + cg + 16 * u];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float pa = Ps[(4 * rg + a) * PPAD + j];
#pragma unroll
        for (int u = 0; u < 8; ++u) O[a][u] = fmaf(pa, vj[u], O[a][u]);
      }
    }
  }

#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int64_t i = i0 + 4 * rg + a;
    if (i > i_last) continue;
    float* orow = p.out + ((i - p.q_start) * p.Hq + h) * static_cast<int64_t>(HD);
    const float inv = 1.f / l_run[a];
#pragma unroll
    for (int u = 0; u < 8; ++u) orow[cg + 16 * u] = O[a][u] * inv;
    // p = 2^(S sc - m sc), so ln sum_j e^(z_j) = (m sc + log2 l) ln 2
    if (p.lse != nullptr && cg == 0)
      p.lse[(i - p.q_start) * p.Hq + h] = (m_run[a] * sc + log2f(l_run[a])) * 0.6931471805599453f;
  }
}

}  // namespace f32k

cudaError_t launch_attention_f32(const AttnArgs& a, cudaStream_t st) {
  using namespace f32k;
  if (a.Lq <= 0) return cudaSuccess;
  Params p;
  p.q = static_cast<const float*>(a.q);
  p.kr = static_cast<const float*>(a.kr);
  p.v = static_cast<const float*>(a.v);
  p.out = static_cast<float*>(a.out);
  p.tab = a.tab;
  p.q_start = a.q_start;
  p.Lq = a.Lq;
  p.Lk = a.Lk;
  p.s = a.s;
  p.w = a.w;
  p.tab_c1 = a.tab_c1;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.n_qtiles = static_cast<int>((a.Lq + BM - 1) / BM);
  p.reading = a.reading;
  p.scale_log2 = a.scale_log2;
  p.lse = a.lse;
  const int64_t blocks = static_cast<int64_t>(p.n_qtiles) * p.Hq;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(dca_fwd_f32_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  dca_fwd_f32_kernel<<<static_cast<unsigned>(blocks), THREADS, SMEM_BYTES, st>>>(p);
  return cudaGetLastError();
}

}  // namespace dca
