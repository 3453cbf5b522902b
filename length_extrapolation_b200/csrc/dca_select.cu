// dca_select.cu -- online key selection for the vertical-slash sparse
// attention ("Qwen2.5-1M 不重训外推 1M", section "稀疏注意力 + 核优化": the fix
// restores continuous relative positions at the key-selection stage, since
// DCA's remapped positions break the diagonal pattern).
//
// For the last n_last (<= 64) rows i of the query block and each query head:
// p_ij = softmax over keys j <= i of the logits -- the DCA logits, or RoPE
// logits at the true positions i and j ("continuous");
//     vertical[j] = sum_rows p_ij,     slash[o] = sum_rows p_{i, i-o};
// the n_v keys and n_s offsets of largest score (ties: the smaller index)
// become the head's pattern, written straight into the sparse workspace
// (lists, bitmaps, slash runs) for dca_sparse_attend.
//
// Kernels: query variants (fp64 angles where the table has none), two score
// passes over the keys on the tensor cores (dca_select_mma.cu: row max/sum,
// then the sums of probabilities), a merge of the row statistics, a radix
// select per (head, kind), and the gather of the selected vertical rows.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "dca_internal.h"
#include "dca_plan.cuh"
#include "sm100_ptx.cuh"

namespace dca {
namespace sel {

constexpr int ROWS = 64;     // rows of the estimate (max)
constexpr int KT = 128;      // keys per tile
constexpr int HD = 128;

// Row statistics: max and sum over the key slices' partial (max, sum) (one
// warp per (head, row)).
__global__ void sel_stats_kernel(const float2* __restrict__ part, float2* __restrict__ stats,
                                 int n_tiles, int Hq) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= Hq * ROWS) return;
  const int h = wid / ROWS, r = wid % ROWS;
  const float2* pp = part + static_cast<int64_t>(h) * n_tiles * ROWS + r;
  float m = -INFINITY;
  for (int tt = lane; tt < n_tiles; tt += 32) m = fmaxf(m, pp[static_cast<int64_t>(tt) * ROWS].x);
  for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float l = 0.f;
  if (m != -INFINITY)
    for (int tt = lane; tt < n_tiles; tt += 32) {
      const float2 v = pp[static_cast<int64_t>(tt) * ROWS];
      if (v.x != -INFINITY) l += v.y * exp2f(v.x - m);
    }
  for (int off = 16; off >= 1; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  if (lane == 0) stats[h * ROWS + r] = make_float2(m, l);
}

// Query variants: DCA (3, from the workspace table) or continuous (1, angle
// i * theta_k in fp64); pre-scaled to log2 units.  Also the continuous key
// chunk rotations (cos, sin) of s * n * theta_k.
__global__ void sel_qvar_kernel(const __nv_bfloat16* __restrict__ q, const float2* __restrict__ tab,
                                float* __restrict__ qv, float2* __restrict__ crot, int64_t q_start,
                                int64_t Lq, int n_last, int Hq, int64_t s, int64_t w,
                                int64_t tab_c1, int nvar, int continuous, double base,
                                float scale_log2, int n_chunks) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t n_q = static_cast<int64_t>(Hq) * nvar * ROWS * (HD / 2);
  if (idx < n_q) {
    const int k = static_cast<int>(idx % (HD / 2));
    const int r = static_cast<int>((idx / (HD / 2)) % ROWS);
    const int v = static_cast<int>((idx / (HD / 2 * ROWS)) % nvar);
    const int h = static_cast<int>(idx / (static_cast<int64_t>(HD / 2) * ROWS * nvar));
    float ya = 0.f, yb = 0.f;
    const int64_t tq = Lq - n_last + r;
    const int64_t i = q_start + tq;
    // a row of the first chunk attends intra-chunk keys only (and the table
    // holds the positions s + r only once the cache passes the first chunk)
    if (r < n_last && (continuous || v == CLS_INTRA || i >= s)) {
      const __nv_bfloat16* qr = q + (tq * Hq + h) * static_cast<int64_t>(HD);
      const float xa = __bfloat162float(qr[k]), xb = __bfloat162float(qr[k + HD / 2]);
      float c, sn;
      if (continuous) {
        const double th = pow(base, -2.0 * k / HD);
        double sd, cd;
        sincos(static_cast<double>(i) * th, &sd, &cd);
        c = static_cast<float>(cd);
        sn = static_cast<float>(sd);
      } else {
        const float2 cs = tab[query_table_row(i, v, s, w, tab_c1) * (HD / 2) + k];
        c = cs.x;
        sn = cs.y;
      }
      ya = (xa * c - xb * sn) * scale_log2;
      yb = (xa * sn + xb * c) * scale_log2;
    }
    float* o = qv + ((static_cast<int64_t>(h) * nvar + v) * ROWS + r) * HD;
    o[k] = ya;
    o[k + HD / 2] = yb;
  }
  if (continuous && idx < static_cast<int64_t>(n_chunks) * (HD / 2)) {
    const int k = static_cast<int>(idx % (HD / 2));
    const int64_t n = idx / (HD / 2);
    const double th = pow(base, -2.0 * k / HD);
    double sd, cd;
    sincos(static_cast<double>(s * n) * th, &sd, &cd);
    crot[idx] = make_float2(static_cast<float>(cd), static_cast<float>(sd));
  }
}

// Block-wide exclusive scan of one int per thread (1024 threads); returns
// the prefix and the total through `total`.
__device__ __forceinline__ int block_scan(int v, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += y;
    }
    warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  total = warp_sums[31];
  __syncthreads();
  return before;
}

struct SelectOut {
  int32_t* nv;      // [Hq] counts (kind 0) ...
  int32_t* ns;      // ... and (kind 1)
  int32_t* vidx;    // [Hq][nv_cap]
  int32_t* soff;    // [Hq][s_cap]
  int2* runs;       // [Hq][SPARSE_MAX_RUNS]
  int32_t* nruns;   // [Hq]
  uint32_t* vbit;   // [Hq][wpr] (zeroed before)
  uint32_t* sbit;   // [Hq][wpr] (zeroed before)
  int64_t nv_cap, s_cap, wpr;
};

// Top-k by value (ties: smaller index) of scores[0 .. Lk) (all >= 0), for
// (head, kind) = (blockIdx.x / 2, blockIdx.x % 2): radix select on the float
// bits (order-preserving for non-negative floats) in three histogram passes,
// then an ordered pass writes the selected indices ascending.
__global__ void __launch_bounds__(1024)
    sel_topk_kernel(const float* __restrict__ vert, const float* __restrict__ slash, int64_t Lk,
                    int64_t n_v, int64_t n_s, SelectOut out) {
  __shared__ int hist[4096];
  __shared__ int warp_sums[32];
  __shared__ int sh_bin, sh_above;
  const int h = blockIdx.x >> 1, kind = blockIdx.x & 1;
  const float* sc = (kind ? slash : vert) + static_cast<int64_t>(h) * Lk;
  const int64_t kk = kind ? (n_s < Lk ? n_s : Lk) : (n_v < Lk ? n_v : Lk);
  const int tid = threadIdx.x;

  uint32_t prefix = 0;   // selected high bits so far
  int64_t above = 0;     // elements strictly above the current prefix bucket
  const int shifts[3] = {20, 8, 0};
  const int widths[3] = {12, 12, 8};
  for (int pass = 0; pass < 3 && kk > 0; ++pass) {
    const int nb = 1 << widths[pass];
    for (int b = tid; b < nb; b += 1024) hist[b] = 0;
    __syncthreads();
    const int top = pass == 0 ? 32 : shifts[pass - 1];
    const int lane = tid & 31;
    for (int64_t base = 0; base < Lk; base += 1024) {
      // lanes with the same bin add once (scores crowd into a few bins)
      const int64_t j = base + tid;
      int bin = -1;
      if (j < Lk) {
        const uint32_t bits = __float_as_uint(sc[j]);
        if (pass == 0 || (bits >> top) == prefix) bin = static_cast<int>((bits >> shifts[pass]) & (nb - 1));
      }
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
    }
    __syncthreads();
    if (tid == 0) {
      int64_t cum = above;
      int b = nb - 1;
      for (; b >= 0; --b) {
        if (cum + hist[b] >= kk) break;
        cum += hist[b];
      }
      sh_bin = b < 0 ? 0 : b;
      sh_above = static_cast<int>(cum);
    }
    __syncthreads();
    prefix = (prefix << widths[pass]) | static_cast<uint32_t>(sh_bin);
    above = sh_above;
    __syncthreads();
  }
  const uint32_t T = prefix;                // the k-th largest value's bits
  const int64_t need_eq = kk - above;       // how many equal to T are taken
  int32_t* list = kind ? out.soff + h * out.s_cap : out.vidx + h * out.nv_cap;
  uint32_t* bitrow = (kind ? out.sbit : out.vbit) + h * out.wpr;
  int64_t eq_seen = 0, written = 0;
  for (int64_t base = 0; base < Lk && kk > 0; base += 1024) {
    const int64_t j = base + tid;
    const uint32_t bits = j < Lk ? __float_as_uint(sc[j]) : 0u;
    const int is_eq = (j < Lk && bits == T) ? 1 : 0;
    int eq_total;
    const int eq_before = block_scan(is_eq, warp_sums, eq_total);
    const int sel = (j < Lk) && (bits > T || (is_eq && eq_seen + eq_before < need_eq)) ? 1 : 0;
    int sel_total;
    const int pos = block_scan(sel, warp_sums, sel_total);
    if (sel) {
      list[written + pos] = static_cast<int32_t>(j);
      atomicOr(&bitrow[j >> 5], 1u << (j & 31));
    }
    eq_seen += eq_total;
    written += sel_total;
  }
  __syncthreads();  // the list is complete before one thread reads it
  if (tid == 0) {
    if (kind == 0) {
      out.nv[h] = static_cast<int32_t>(written);
    } else {
      out.ns[h] = static_cast<int32_t>(written);
      // runs of consecutive offsets (the caller keeps n_s <= SPARSE_MAX_RUNS)
      int n = 0;
      int2* rr = out.runs + static_cast<int64_t>(h) * SPARSE_MAX_RUNS;
      for (int64_t e = 0; e < written; ++e) {
        const int32_t o = list[e];
        if (n > 0 && rr[n - 1].y == o) {
          rr[n - 1].y = o + 1;
        } else if (n < SPARSE_MAX_RUNS) {
          rr[n++] = make_int2(o, o + 1);
        }
      }
      out.nruns[h] = n;
    }
  }
}

}  // namespace sel

size_t select_scratch_bytes(int64_t Lk, int Hq, int64_t n_chunks) {
  const int64_t n_tiles = (Lk + sel::KT - 1) / sel::KT;
  size_t b = 0;
  auto add = [&](size_t n) { b += (n + 255) / 256 * 256; };
  add(sizeof(float) * static_cast<size_t>(Hq) * 3 * sel::ROWS * sel::HD);   // query variants
  add(sizeof(float2) * static_cast<size_t>(n_chunks) * (sel::HD / 2));     // chunk rotations
  add(sizeof(float2) * static_cast<size_t>(Hq) * n_tiles * sel::ROWS);     // slice statistics
  add(sizeof(float2) * static_cast<size_t>(Hq) * sel::ROWS);               // row statistics
  add(sizeof(float) * static_cast<size_t>(Hq) * Lk * 2);                   // scores
  return b;
}

cudaError_t launch_select(const SelectArgs& sa, cudaStream_t st) {
  using namespace sel;
  const int64_t n_tiles = (sa.Lk + KT - 1) / KT;
  const int nvar = sa.continuous ? 1 : 3;
  uint8_t* b = static_cast<uint8_t*>(sa.scratch);
  size_t off = 0;
  auto take = [&](size_t n) {
    uint8_t* p = b + off;
    off += (n + 255) / 256 * 256;
    return p;
  };
  float* qv = reinterpret_cast<float*>(take(sizeof(float) * sa.Hq * 3 * ROWS * HD));
  float2* crot = reinterpret_cast<float2*>(take(sizeof(float2) * sa.n_chunks * (HD / 2)));
  float2* part = reinterpret_cast<float2*>(take(sizeof(float2) * sa.Hq * n_tiles * ROWS));
  float2* stats = reinterpret_cast<float2*>(take(sizeof(float2) * sa.Hq * ROWS));
  float* scores = reinterpret_cast<float*>(take(sizeof(float) * sa.Hq * sa.Lk * 2));
  float* vert = scores;
  float* slash = scores + static_cast<int64_t>(sa.Hq) * sa.Lk;

  // vert is stored whole by the second score pass; slash is accumulated
  cudaError_t e = cudaMemsetAsync(slash, 0, sizeof(float) * sa.Hq * sa.Lk, st);
  if (e != cudaSuccess) return e;
  {
    const int64_t n = std::max<int64_t>(static_cast<int64_t>(sa.Hq) * nvar * ROWS * (HD / 2),
                                        sa.n_chunks * (HD / 2));
    sel_qvar_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(sa.q), sa.tab, qv, crot, sa.q_start, sa.Lq, sa.n_last,
        sa.Hq, sa.s, sa.w, sa.tab_c1, nvar, sa.continuous, sa.rope_base, sa.scale_log2,
        static_cast<int>(sa.n_chunks));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const int64_t i_first = sa.q_start + sa.Lq - sa.n_last;
  const int n_slices = select_slices(sa.Lk);
  e = launch_select_scores(sa.kr, qv, crot, part, stats, vert, slash, i_first, sa.Lk, sa.s, sa.w,
                           sa.n_last, sa.Hq, sa.Hkv, sa.reading, sa.continuous, 1, sa.status,
                           sa.timeout_ns, st);
  if (e != cudaSuccess) return e;
  sel_stats_kernel<<<static_cast<unsigned>((sa.Hq * ROWS * 32 + 255) / 256), 256, 0, st>>>(
      part, stats, n_slices, sa.Hq);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  e = launch_select_scores(sa.kr, qv, crot, part, stats, vert, slash, i_first, sa.Lk, sa.s, sa.w,
                           sa.n_last, sa.Hq, sa.Hkv, sa.reading, sa.continuous, 2, sa.status,
                           sa.timeout_ns, st);
  if (e != cudaSuccess) return e;
  SelectOut o;
  o.nv = sa.nv;
  o.ns = sa.ns;
  o.vidx = sa.vidx;
  o.soff = sa.soff;
  o.runs = sa.runs;
  o.nruns = sa.nruns;
  o.vbit = sa.vbit;
  o.sbit = sa.sbit;
  o.nv_cap = sa.nv_cap;
  o.s_cap = sa.s_cap;
  o.wpr = sa.wpr;
  sel_topk_kernel<<<static_cast<unsigned>(2 * sa.Hq), 1024, 0, st>>>(vert, slash, sa.Lk, sa.n_v,
                                                                      sa.n_s, o);
  return cudaGetLastError();
}

}  // namespace dca
