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

// Top-k by value (ties: the smaller index) of each score row (vertical and
// slash of every head, all scores >= 0): a radix select on the float bits
// (order-preserving for non-negative floats), 12 + 12 + 8 bits.  Each pass
// is a histogram over the row's spans (one CTA per span, warp-aggregated
// shared-memory atomics, then the nonzero bins into a global histogram) and
// a pick of the bin holding the k-th largest (a suffix scan over the bins).
// Then per span the count above / equal to the k-th value, and an ordered
// write: the spans' counts place each span's output, equal values are taken
// in index order, so the list comes out ascending.
constexpr int TK_THREADS = 1024;
constexpr int TK_BINS = 4096;

struct TopkState {
  uint32_t prefix;  // the high bits of the k-th largest found so far
  int32_t pad;
  int64_t above;    // elements strictly above the prefix's bucket
};

struct TopkArgs {
  const float* vert;   // [Hq][Lk]
  const float* slash;  // [Hq][Lk]
  int64_t Lk, n_v, n_s, span;
  int nb;              // spans (CTAs) per row; rows = 2 Hq: (head, kind)
  int* hist;           // [rows][TK_BINS]
  TopkState* state;    // [rows]
  int2* cnt;           // [rows][nb]: (above the k-th value, equal to it)
};

// span of one CTA: a multiple of the block, at least 16K, at most 1024 spans per row
inline int64_t topk_span(int64_t Lk) {
  int64_t sp = (Lk + 1023) / 1024;
  if (sp < 16384) sp = 16384;
  return (sp + TK_THREADS - 1) / TK_THREADS * TK_THREADS;
}

__device__ __forceinline__ int64_t topk_k(const TopkArgs& a, int row) {
  const int64_t n = (row & 1) ? a.n_s : a.n_v;
  return n < a.Lk ? n : a.Lk;
}
__device__ __forceinline__ const float* topk_row(const TopkArgs& a, int row) {
  return ((row & 1) ? a.slash : a.vert) + static_cast<int64_t>(row >> 1) * a.Lk;
}

__global__ void __launch_bounds__(TK_THREADS)
    sel_topk_hist_kernel(const TopkArgs a, int pass) {
  __shared__ int hist[TK_BINS];
  const int row = blockIdx.y;
  if (topk_k(a, row) == 0) return;
  const int shift = pass == 0 ? 20 : (pass == 1 ? 8 : 0);
  const int nbin = pass == 2 ? 256 : TK_BINS;
  const int top = pass == 0 ? 32 : (pass == 1 ? 20 : 8);  // bits above this pass
  const uint32_t prefix = pass == 0 ? 0u : a.state[row].prefix;
  const int tid = threadIdx.x, lane = tid & 31;
  for (int b = tid; b < nbin; b += TK_THREADS) hist[b] = 0;
  __syncthreads();
  const float* sc = topk_row(a, row);
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * a.span;
  for (int64_t j = j0 + tid; j < j0 + a.span; j += TK_THREADS) {  // same trip count in every lane
    int bin = -1;
    if (j < a.Lk) {
      const uint32_t bits = __float_as_uint(sc[j]);
      if ((static_cast<uint64_t>(bits) >> top) == prefix) bin = static_cast<int>((bits >> shift) & (nbin - 1));
    }
    // after the first pass few scores match the prefix: most warps skip
    if (__any_sync(0xffffffffu, bin >= 0)) {
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
    }
  }
  __syncthreads();
  int* g = a.hist + static_cast<int64_t>(row) * TK_BINS;
  for (int b = tid; b < nbin; b += TK_THREADS)
    if (hist[b] != 0) atomicAdd(&g[b], hist[b]);
}

// One CTA per row: the bin holding the k-th largest (bins scanned from the
// top), appended to the prefix; clears the histogram for the next pass.
__global__ void __launch_bounds__(TK_THREADS)
    sel_topk_pick_kernel(const TopkArgs a, int pass) {
  __shared__ int warp_sums[32];
  const int row = blockIdx.x;
  const int64_t kk = topk_k(a, row);
  if (kk == 0) return;
  const int nbin = pass == 2 ? 256 : TK_BINS;
  const int width = pass == 2 ? 8 : 12;
  const int per = nbin / TK_THREADS > 0 ? nbin / TK_THREADS : 1;  // bins per thread
  const uint32_t prefix = pass == 0 ? 0u : a.state[row].prefix;
  const int64_t above = pass == 0 ? 0 : a.state[row].above;
  int* g = a.hist + static_cast<int64_t>(row) * TK_BINS;
  const int tid = threadIdx.x;
  int c[4] = {0, 0, 0, 0};
  int sum = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int d = tid * per + e;  // rank of the bin from the top
    if (e < per && d < nbin) c[e] = g[nbin - 1 - d];
    sum += c[e];
  }
  int total;
  int64_t cum = above + block_scan(sum, warp_sums, total);  // elements in higher bins
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int d = tid * per + e;
    if (e < per && d < nbin && cum < kk && cum + c[e] >= kk) {
      a.state[row].prefix = (prefix << width) | static_cast<uint32_t>(nbin - 1 - d);
      a.state[row].above = cum;
    }
    cum += c[e];
  }
  for (int b = tid; b < TK_BINS; b += TK_THREADS) g[b] = 0;  // every read is behind the scan's barriers
}

// Per span: how many scores are above / equal to the k-th value T.
__global__ void __launch_bounds__(TK_THREADS)
    sel_topk_count_kernel(const TopkArgs a) {
  __shared__ int warp_sums[32];
  const int row = blockIdx.y;
  if (topk_k(a, row) == 0) return;
  const uint32_t T = a.state[row].prefix;
  const float* sc = topk_row(a, row);
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * a.span;
  int gt = 0, eq = 0;
  for (int64_t j = j0 + threadIdx.x; j < j0 + a.span && j < a.Lk; j += TK_THREADS) {
    const uint32_t bits = __float_as_uint(sc[j]);
    gt += bits > T;
    eq += bits == T;
  }
  int tg, te;
  block_scan(gt, warp_sums, tg);
  block_scan(eq, warp_sums, te);
  if (threadIdx.x == 0) a.cnt[static_cast<int64_t>(row) * a.nb + blockIdx.x] = make_int2(tg, te);
}

// Ordered write of the selected indices of each span (ascending), their
// bitmap bits; equal values are taken while the row still needs them.  The
// span is walked in blocks of TK_THREADS x TK_PER scores, each thread owning
// TK_PER consecutive ones, so two block scans per block (equal values before
// the thread, selected before the thread) place everything.
constexpr int TK_PER = 16;

__global__ void __launch_bounds__(TK_THREADS)
    sel_topk_write_kernel(const TopkArgs a, SelectOut out) {
  __shared__ int warp_sums[32];
  __shared__ long long sh_start, sh_eq_before;
  const int row = blockIdx.y, kind = row & 1, h = row >> 1;
  const int64_t kk = topk_k(a, row);
  if (kk == 0) return;
  const uint32_t T = a.state[row].prefix;
  const int64_t need_eq = kk - a.state[row].above;
  if (threadIdx.x == 0) {
    const int2* cr = a.cnt + static_cast<int64_t>(row) * a.nb;
    int64_t start = 0, eqb = 0;
    for (int b = 0; b < static_cast<int>(blockIdx.x); ++b) {
      const int2 cb = cr[b];
      int64_t take = need_eq - eqb;
      take = take < 0 ? 0 : (take > cb.y ? cb.y : take);
      start += cb.x + take;
      eqb += cb.y;
    }
    sh_start = start;
    sh_eq_before = eqb;
  }
  __syncthreads();
  int32_t* list = kind ? out.soff + h * out.s_cap : out.vidx + h * out.nv_cap;
  uint32_t* bitrow = (kind ? out.sbit : out.vbit) + h * out.wpr;
  const float* sc = topk_row(a, row);
  const int64_t span0 = static_cast<int64_t>(blockIdx.x) * a.span;
  const int64_t span1 = span0 + a.span < a.Lk ? span0 + a.span : a.Lk;
  // blocks of TK_THREADS x TK_PER scores in order; thread t owns TK_PER
  // consecutive scores of each, so (block, thread, element) is index order
  for (int64_t c0 = span0; c0 < span1; c0 += TK_THREADS * TK_PER) {
    const int64_t jt = c0 + static_cast<int64_t>(threadIdx.x) * TK_PER;
    // this block's starting counts, read before thread 0 advances them
    const int64_t eq_before = sh_eq_before, start = sh_start;
    uint32_t bits[TK_PER];
    int eq = 0;
#pragma unroll
    for (int e = 0; e < TK_PER; ++e) {
      const int64_t j = jt + e;
      bits[e] = j < span1 ? __float_as_uint(sc[j]) : 0u;
      eq += (j < span1 && bits[e] == T) ? 1 : 0;
    }
    int eq_total;
    int64_t eq_seen = eq_before + block_scan(eq, warp_sums, eq_total);
    uint32_t take = 0;  // bit e: element e selected
#pragma unroll
    for (int e = 0; e < TK_PER; ++e) {
      const int64_t j = jt + e;
      if (j < span1 && bits[e] > T) take |= 1u << e;
      if (j < span1 && bits[e] == T) {
        if (eq_seen < need_eq) take |= 1u << e;
        ++eq_seen;
      }
    }
    int sel_total;
    int64_t pos = start + block_scan(__popc(take), warp_sums, sel_total);
#pragma unroll
    for (int e = 0; e < TK_PER; ++e) {
      if (take & (1u << e)) {
        const int64_t j = jt + e;
        list[pos++] = static_cast<int32_t>(j);
        atomicOr(&bitrow[j >> 5], 1u << (j & 31));
      }
    }
    if (threadIdx.x == 0) {  // every thread read the counts before the scans' barriers
      sh_eq_before = eq_before + eq_total;
      sh_start = start + sel_total;
    }
    __syncthreads();
  }
}

// Counts, and the runs of consecutive slash offsets: one CTA per head, one
// thread per list entry (the caller keeps n_s <= SPARSE_MAX_RUNS < 1024); an
// entry starts a run unless it follows its predecessor, a scan of the starts
// numbers the runs.
__global__ void __launch_bounds__(TK_THREADS)
    sel_topk_finish_kernel(const TopkArgs a, SelectOut out) {
  __shared__ int warp_sums[32];
  const int h = blockIdx.x, e = threadIdx.x;
  const int64_t ks = topk_k(a, 2 * h + 1);
  if (e == 0) {
    out.nv[h] = static_cast<int32_t>(topk_k(a, 2 * h));
    out.ns[h] = static_cast<int32_t>(ks);
  }
  const int32_t* list = out.soff + h * out.s_cap;
  const int32_t o = e < ks ? list[e] : 0;
  const int start = (e < ks && (e == 0 || list[e - 1] + 1 != o)) ? 1 : 0;
  const int last = (e < ks && (e + 1 == ks || list[e + 1] != o + 1)) ? 1 : 0;
  int n_runs;
  const int idx = block_scan(start, warp_sums, n_runs) - (start ? 0 : 1);  // this entry's run
  int2* rr = out.runs + static_cast<int64_t>(h) * SPARSE_MAX_RUNS;
  if (start) rr[idx].x = o;
  if (last) rr[idx].y = o + 1;
  if (e == 0) out.nruns[h] = n_runs;
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
  const int64_t nb = (Lk + sel::topk_span(Lk) - 1) / sel::topk_span(Lk);
  add(sizeof(int) * static_cast<size_t>(2 * Hq) * sel::TK_BINS);            // top-k histograms
  add(sizeof(sel::TopkState) * static_cast<size_t>(2 * Hq));                // top-k state
  add(sizeof(int2) * static_cast<size_t>(2 * Hq) * nb);                     // top-k span counts
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
  const int n_slices = select_stat_slices(sa.Lk);
  e = launch_select_row_stats(sa.kr, qv, crot, part, i_first, sa.Lk, sa.s, sa.w, sa.n_last, sa.Hq,
                              sa.Hkv, sa.reading, sa.continuous, sa.status, sa.timeout_ns, st);
  if (e != cudaSuccess) return e;
  sel_stats_kernel<<<static_cast<unsigned>((sa.Hq * ROWS * 32 + 255) / 256), 256, 0, st>>>(
      part, stats, n_slices, sa.Hq);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  e = launch_select_sums(sa.kr, qv, crot, stats, vert, slash, i_first, sa.Lk, sa.s, sa.w,
                         sa.n_last, sa.Hq, sa.Hkv, sa.reading, sa.continuous, sa.status,
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
  TopkArgs ta;
  ta.vert = vert;
  ta.slash = slash;
  ta.Lk = sa.Lk;
  ta.n_v = sa.n_v;
  ta.n_s = sa.n_s;
  ta.span = topk_span(sa.Lk);
  ta.nb = static_cast<int>((sa.Lk + ta.span - 1) / ta.span);
  ta.hist = reinterpret_cast<int*>(take(sizeof(int) * 2 * sa.Hq * TK_BINS));
  ta.state = reinterpret_cast<TopkState*>(take(sizeof(TopkState) * 2 * sa.Hq));
  ta.cnt = reinterpret_cast<int2*>(take(sizeof(int2) * 2 * sa.Hq * ta.nb));
  if ((e = cudaMemsetAsync(ta.hist, 0, sizeof(int) * 2 * sa.Hq * TK_BINS, st)) != cudaSuccess)
    return e;
  const dim3 spans(static_cast<unsigned>(ta.nb), static_cast<unsigned>(2 * sa.Hq));
  for (int pass = 0; pass < 3; ++pass) {
    sel_topk_hist_kernel<<<spans, TK_THREADS, 0, st>>>(ta, pass);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    sel_topk_pick_kernel<<<static_cast<unsigned>(2 * sa.Hq), TK_THREADS, 0, st>>>(ta, pass);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  sel_topk_count_kernel<<<spans, TK_THREADS, 0, st>>>(ta);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  sel_topk_write_kernel<<<spans, TK_THREADS, 0, st>>>(ta, o);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  sel_topk_finish_kernel<<<static_cast<unsigned>(sa.Hq), TK_THREADS, 0, st>>>(ta, o);
  return cudaGetLastError();
}

}  // namespace dca
