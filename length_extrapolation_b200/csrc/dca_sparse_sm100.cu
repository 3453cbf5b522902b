// dca_sparse_sm100.cu -- vertical-slash sparse Dual Chunk Attention for sm_100a.
//
// The Qwen2.5-1M framework runs MInference's vertical-slash sparse attention
// on top of DCA ("Qwen2.5-1M 不重训外推 1M", sections "跟 NSA / 其他稀疏注意力的
// 区别" and "稀疏注意力 + 核优化"): per query head, a few key columns (vertical
// lines) and a few diagonals (slash lines) carry the attention, and only
// those keys are attended.  For head h with vertical keys V_h and slash
// offsets S_h, row i attends exactly
//     M_h(i) = { j <= i : j in V_h } U { i - o : o in S_h, o <= i } U { i }
// (each key once) with the DCA logits of the dense kernel and a softmax over
// M_h(i).
//
// One CTA = one 128-row query tile of one query head (patterns are per head).
// Its work list has two kinds of 128-key items, visited class by class
// (INTER, SUCC, INTRA; dca_plan.cuh):
//   vertical items  tiles of the head's gathered vertical keys (rotated keys
//                   and values copied into a compact [n][Hq][128] array by
//                   the preparation kernels), masked to j <= i and the class;
//   slash items     windows of 128 cache keys covering what the slash
//                   diagonals (and the diagonal j = i) reach from the rows of
//                   the tile, masked per element to the member pairs not
//                   already counted as vertical, and to the class.
// The slash windows come from the head's runs of consecutive offsets, merged
// into key ranges once per CTA in shared memory (dca_sparse_plan.cuh).
//
// Warps (320 threads): warps 0-7 softmax (warp w and w+4 split each row's 128
// keys), warp 8 TMA producer (6-slot K/V ring, no multicast), warp 9 MMA
// issuer.  TMEM holds two S buffers, O and the rotated query tile: S = Q K^T
// takes Q from TMEM and the key tile from shared memory, so S(n+1) runs on
// the tensor cores while the softmax warps work on S(n); P(n) overwrites the
// first 64 columns of its S buffer and feeds O += P V from TMEM.  Where the
// class changes between items n and n+1 the softmax warps rewrite the query
// tile for the new class after S(n) has completed and before they release
// P(n), and S(n+1) is issued after P(n) instead of one item earlier.  Warp 0
// builds the work list at the start (runs staged in shared memory, the
// vertical-list searches done by the whole warp); each softmax thread keeps
// its row's key range and vertical-list positions per class, so an item's
// keep mask is a range test plus the slash and vertical bitmaps.
// Every wait is bounded; on timeout the CTA raises its abort flag, ORs a code
// into the device status word, drains its copies and MMAs and exits.
#include <cuda_bf16.h>
#include <math.h>

#include "dca_internal.h"
#include "dca_plan.cuh"
#include "dca_softmax.cuh"
#include "dca_sparse_plan.cuh"
#include "sm100_ptx.cuh"

namespace dca {
namespace sp {

using namespace attn;

constexpr int BM = 128, BN = 128, HD = 128;
constexpr int NSLOT = 6;                 // K/V ring: the key tile of S(k) reuses the slot of K(k - 3)
static_assert(NSLOT % 2 == 0, "a key tile's slot must have held a key tile");
constexpr int NSBUF = 2;                 // S buffers in TMEM (P aliases their first 64 columns)
constexpr uint32_t COL_O = NSBUF * 128;  // O after them
constexpr uint32_t COL_Q = COL_O + 128;  // the rotated query tile (MMA operand A), 64 columns
constexpr int TILE_BYTES = 32768;
constexpr int NUM_THREADS = 320;
constexpr int WARP_LOAD = 8, WARP_MMA = 9;
constexpr float RESCALE_LOG2 = 8.0f;

constexpr unsigned ST_SOFTMAX = 0x10u, ST_LOAD = 0x100u, ST_MMA = 0x1000u, ST_DRAIN = 0x10000u;

struct SmemCtl {
  uint64_t slot_full[NSLOT];
  uint64_t slot_empty[NSLOT];
  uint64_t s_full[NSBUF];
  uint64_t p_full[NSBUF];
  uint64_t pv_done[2];
  uint64_t q_ready;
  uint64_t o_final;
  uint64_t drain;
  uint64_t pair_bar[4];
  uint32_t tmem_base;
  int abort;
  float xval[2][2][128];
  SparsePlan plan;
};

constexpr size_t SMEM_BYTES = 1024 + NSLOT * TILE_BYTES + sizeof(SmemCtl);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

struct Params {
  const __nv_bfloat16* q;
  __nv_bfloat16* out;
  const float2* tab;
  const int32_t* vidx;    // [Hq][nv_cap] sorted vertical keys
  const int32_t* nv;      // [Hq] vertical key counts
  const int2* runs;       // [Hq][SPARSE_MAX_RUNS] slash offset runs [x, y), ascending
  const int32_t* nruns;   // [Hq]
  const uint32_t* vbit;   // [Hq][wpr] vertical membership bits (bit j)
  const uint32_t* sbit;   // [Hq][wpr] slash offset bits (bit o)
  int64_t wpr;            // words per head row of the bitmaps (>= cap/32 + 2)
  int64_t nv_cap;
  int64_t q_start, Lq, Lk;
  int64_t s, w, tab_c1;
  int Hq, Hkv, G, n_qtiles;
  int reading;
  float scale_log2;
  unsigned int* status;
  unsigned long long timeout_ns;
  int debug;
};

// Bitmap rows are padded with two zero words past their last bit; bits below
// 0 read as 0.
// Columns of this thread's half-row of an item (64 keys) that are attended:
// inside the row's key range [lo, hi) for the item's class (causality
// included), and members -- for a slash window the keys on a slash diagonal
// of the head (or j = i) that are not vertical keys, for a vertical tile the
// row's positions [pa, pb) of the gathered list for the class.  Bit e keeps
// column e.  keep_fetch issues the bitmap loads of the next item before the
// current item's softmax; keep_finish forms the mask after it.
struct KeepFetch {
  uint32_t v[3], s[3];  // vertical bits from key j0, slash bits from offset i - j0 - 63
  int src, a, b;        // slash: kept columns [a, b) of the range; vertical: the same from [pa, pb)
  int sh_v, sh_s, base;
};

__device__ __forceinline__ int clamp64(int x) { return x < 0 ? 0 : (x > 64 ? 64 : x); }

__device__ __forceinline__ void bits_fetch(const uint32_t* row, int lo, uint32_t w[3], int& sh) {
  const int base = lo < 0 ? 0 : lo;
  const int wd = base >> 5;
  sh = base & 31;
  if (lo <= -64) {
    w[0] = w[1] = w[2] = 0u;
    return;
  }
  w[0] = row[wd];
  w[1] = row[wd + 1];
  w[2] = row[wd + 2];
}

__device__ __forceinline__ uint64_t bits_form(const uint32_t w[3], int sh, int lo) {
  uint64_t v = (static_cast<uint64_t>(w[0]) | (static_cast<uint64_t>(w[1]) << 32)) >> sh;
  if (sh) v |= static_cast<uint64_t>(w[2]) << (64 - sh);
  if (lo < 0) v = lo <= -64 ? 0ull : (v << -lo);
  return v;
}

__device__ __forceinline__ KeepFetch keep_fetch(int src, int start, int i, int half, int lo, int hi,
                                                int pa, int pb, const uint32_t* vrow,
                                                const uint32_t* srow) {
  KeepFetch f;
  f.src = src;
  if (src == 1) {
    const int j0 = start + 64 * half;  // first key of the half window
    f.a = clamp64(lo - j0);
    f.b = max(clamp64(hi - j0), f.a);
    f.base = i - j0;  // offset of key e is base - e
    bits_fetch(vrow, j0, f.v, f.sh_v);
    bits_fetch(srow, f.base - 63, f.s, f.sh_s);
  } else {
    const int pos0 = start + 64 * half;  // first gathered position
    f.a = clamp64(pa - pos0);
    f.b = max(clamp64(pb - pos0), f.a);
  }
  return f;
}

__device__ __forceinline__ uint64_t keep_finish(const KeepFetch& f, int start, int half) {
  const uint64_t rng =
      (f.b >= 64 ? ~0ull : ((1ull << f.b) - 1)) & ~(f.a >= 64 ? ~0ull : ((1ull << f.a) - 1));
  if (f.src != 1) return rng;
  const int j0 = start + 64 * half;
  const uint64_t vm = bits_form(f.v, f.sh_v, j0);
  uint64_t sm = __brevll(bits_form(f.s, f.sh_s, f.base - 63));
  if (f.base >= 0 && f.base < 64) sm |= 1ull << f.base;
  return rng & sm & ~vm;
}

// The work list of the CTA, built by one warp: the slash runs staged in
// P.iv (highest offsets first) with coalesced loads, the lower bounds of
// SPARSE_NKEYS keys in the sorted vertical list found together (each round
// samples 32 evenly spaced positions of every key's remaining interval and
// keeps the one sub-interval that can hold the bound; 1024 keys take two
// rounds), lane 0 merges the ranges, and the lanes count the items.
__device__ void plan_build_warp(SparsePlan& P, const int32_t* vk, int nvh, const int2* runs,
                                int nr, int64_t i0, int64_t i_last, int64_t s, int64_t w,
                                int reading, int lane) {
  for (int r = lane; r < nr; r += 32) P.iv[nr - 1 - r] = runs[r];
  int64_t klo[3], khi[3], key[SPARSE_NKEYS];
  if (lane == 0) sparse_plan_ranges(P, i0, i_last, s, w, reading, klo, khi);
  else class_key_ranges(i0, i_last, s, w, reading, klo, khi);
  sparse_plan_keys(i_last, klo, khi, key);
  int lo[SPARSE_NKEYS], len[SPARSE_NKEYS];
#pragma unroll
  for (int e = 0; e < SPARSE_NKEYS; ++e) {
    lo[e] = 0;
    len[e] = nvh;
  }
  for (;;) {
    bool more = false;
#pragma unroll
    for (int e = 0; e < SPARSE_NKEYS; ++e) more |= len[e] > 0;
    if (!more) break;
    int v[SPARSE_NKEYS], st[SPARSE_NKEYS];
#pragma unroll
    for (int e = 0; e < SPARSE_NKEYS; ++e) {
      st[e] = (len[e] + 31) >> 5;
      const int q = lane * st[e];
      v[e] = (len[e] > 0 && q < len[e]) ? vk[lo[e] + q] : 0x7fffffff;
    }
#pragma unroll
    for (int e = 0; e < SPARSE_NKEYS; ++e) {
      if (len[e] == 0) continue;  // uniform across the warp
      const int c = __popc(__ballot_sync(0xffffffffu, static_cast<int64_t>(v[e]) < key[e]));
      if (c == 0) {
        len[e] = 0;
      } else {
        const int end = lo[e] + len[e];
        const int nlo = lo[e] + (c - 1) * st[e] + 1;
        const int nend = min(lo[e] + c * st[e], end);
        lo[e] = nlo;
        len[e] = nend - nlo;
      }
    }
  }
  __syncwarp();
  if (lane == 0) {
    sparse_plan_vertical(P, klo, khi, lo, 128);
    sparse_plan_slash(P, [&](int k) { return P.iv[k]; }, nr, i0, i_last, 128);
  }
  __syncwarp();
  // the item count (sparse_plan_count) with the ranges spread over the lanes
  int cnt = 0;
  for (int r = lane; r < P.n_iv; r += 32) cnt += sparse_range_items(P.iv[r], P.kr);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
  if (lane == 0) P.n_items = cnt + sparse_vertical_items(P);
}

// One online-softmax step for half of a query row (see the dense kernel):
// columns outside `keep` masked, half-row max exchanged with the partner
// thread, exponentials into P (bf16, first 64 columns of the S buffer), O
// rescaled when the reference moves (after the previous item's P.V
// completed).
__device__ __forceinline__ bool sparse_half_step(
    uint32_t tS, uint32_t tO, int n, uint64_t keep, const Params& p, float sc, float& m_ref,
    float& l_sum, PairCtx& pc, SmemCtl* ctl, volatile int* abort, unsigned int* status) {
  const int half = pc.half;
  uint32_t sv[64];
  tmem_ld64(tS + 64u * half, sv);
  if (keep != ~0ull) {
#pragma unroll
    for (int e = 0; e < 64; ++e)
      if (!((keep >> e) & 1ull)) sv[e] = 0xff800000u;  // -inf
  }
  // at most one attended key in each half-row of the warp (a window that a
  // lone diagonal crosses): its score is the half-row maximum, and one
  // exponential per thread replaces 64
  const bool one_key = __all_sync(0xffffffffu, __popcll(keep) <= 1);
  const int e1 = keep ? __ffsll(static_cast<long long>(keep)) - 1 : -1;
  const float mx_half = max64(sv);
  float mx_other = -INFINITY;
  if (!pair_exchange(pc, mx_half, mx_other, abort, status, p.timeout_ns, ST_SOFTMAX)) return false;
  const float mx = fmaxf(mx_half, mx_other);

  const float m_new = fmaxf(m_ref, mx);
  const bool need =
      (m_new > m_ref) && (m_ref == -INFINITY || (m_new - m_ref) * sc > RESCALE_LOG2);
  float alpha = 1.f;
  if (need) {
    alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx((m_ref - m_new) * sc);
    m_ref = m_new;
    l_sum *= alpha;
  }
  uint32_t pk[32];
  const float mb = (m_ref == -INFINITY) ? 0.f : m_ref * sc;
  if (one_key) {
    const float pv = e1 >= 0 ? ex2_approx(fmaf(mx_half, sc, -mb)) : 0.f;
    l_sum += pv;
    const uint32_t b = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(pv)));
    const uint32_t word = (e1 & 1) ? (b << 16) : b;
#pragma unroll
    for (int w2 = 0; w2 < 32; ++w2) pk[w2] = (w2 == (e1 >> 1)) ? word : 0u;
  } else {
    l_sum += exp_pack64(sv, sc, mb, pk);
  }
  tmem_st32(tS + 32u * half, pk);
  // O holds items < n; the P.V of item n - 1 must have landed before a rescale
  if (n > 0 && __any_sync(0xffffffffu, need)) {
    const int m = n - 1;
    bool ok = wait_bounded(&ctl->pv_done[m & 1], static_cast<uint32_t>((m >> 1) & 1), abort,
                           status, p.timeout_ns, ST_SOFTMAX);
    if (!__all_sync(0xffffffffu, ok)) return false;
    tc_fence_after();
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t o[32];
      tmem_ld32(tO + 64u * half + 32u * c, o);
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
      tmem_st32(tO + 64u * half + 32u * c, o);
    }
  }
  tmem_st_wait();
  return true;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    dca_sparse_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_gk,
                      const __grid_constant__ CUtensorMap tm_gv, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* slots = smem;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(slots + NSLOT * TILE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: the G heads of a KV group next to each other (they cross
  // the same slash tiles of the cache), longest query tiles first
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x / p.Hq);
  const int h = static_cast<int>(blockIdx.x % p.Hq);
  const int g = h / p.G;
  const int64_t i0 = p.q_start + static_cast<int64_t>(qt) * BM;
  const int64_t q_end = p.q_start + p.Lq;
  const int64_t i_last = (i0 + BM - 1 < q_end - 1) ? i0 + BM - 1 : q_end - 1;

  if (threadIdx.x == 0) {
    for (int k = 0; k < NSLOT; ++k) {
      mbar_init(&ctl->slot_full[k], 1);
      mbar_init(&ctl->slot_empty[k], 1);
    }
    for (int st = 0; st < NSBUF; ++st) {
      mbar_init(&ctl->s_full[st], 1);
      mbar_init(&ctl->p_full[st], 8);
    }
    for (int st = 0; st < 2; ++st) mbar_init(&ctl->pv_done[st], 1);
    mbar_init(&ctl->q_ready, 8);
    mbar_init(&ctl->o_final, 1);
    mbar_init(&ctl->drain, 1);
    for (int k = 0; k < 4; ++k) mbar_init(&ctl->pair_bar[k], 2);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    // ---- the CTA's work list
    plan_build_warp(ctl->plan, p.vidx + static_cast<int64_t>(h) * p.nv_cap, p.nv[h],
                    p.runs + static_cast<int64_t>(h) * SPARSE_MAX_RUNS, p.nruns[h], i0, i_last,
                    p.s, p.w, p.reading, lane);
  }
  if (warp == WARP_MMA) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == WARP_LOAD && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_gk);
    tma_prefetch_desc(&tm_gv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = ctl->tmem_base;
  volatile int* abort_flag = &ctl->abort;
  const SparsePlan& plan = ctl->plan;
  const int N = plan.n_items;

  if (warp < 8) {
    // =========================================================== softmax
    const int half = warp >> 2;
    const int sub = warp & 3;
    const int r = sub * 32 + lane;
    PairCtx pc;
    pc.xval = &ctl->xval[0][0][0];
    pc.bar = &ctl->pair_bar[sub];
    pc.ph = 0;
    pc.half = half;
    pc.r = r;
    pc.lane = lane;
    const int64_t i = i0 + r;
    const bool real = i <= i_last;
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const float sc = p.scale_log2;
    const __nv_bfloat16* qrow =
        real ? p.q + ((i - p.q_start) * p.Hq + h) * static_cast<int64_t>(HD) : nullptr;
    // the row's key range per class (a padding row past the block keeps none)
    int klo[3], khi[3];
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      klo[c] = khi[c] = 0;
      if (real)
        row_key_range<int>(static_cast<int>(i), c, static_cast<int>(p.s), static_cast<int>(p.w),
                           p.reading, klo[c], khi[c]);
    }
    const uint32_t* vrow = p.vbit + static_cast<int64_t>(h) * p.wpr;
    const uint32_t* srow = p.sbit + static_cast<int64_t>(h) * p.wpr;
    const int32_t* vk = p.vidx + static_cast<int64_t>(h) * p.nv_cap;
    const int ii = static_cast<int>(i);
    // the row's positions [vpa, vpb) in the sorted vertical list per class:
    // six lower bounds searched together (branch-free halving)
    int vpa[3], vpb[3];
    {
      const int nvh = plan.nv_eff;
      int pos[6];
#pragma unroll
      for (int e = 0; e < 6; ++e) pos[e] = 0;
      int len = nvh;
      while (len > 1) {
        const int hl = len >> 1;
#pragma unroll
        for (int e = 0; e < 6; ++e) {
          const int key = (e & 1) ? khi[e >> 1] : klo[e >> 1];
          if (vk[pos[e] + hl - 1] < key) pos[e] += hl;
        }
        len -= hl;
      }
#pragma unroll
      for (int e = 0; e < 6; ++e) {
        const int key = (e & 1) ? khi[e >> 1] : klo[e >> 1];
        if (len == 1 && vk[pos[e]] < key) ++pos[e];
      }
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        vpa[c] = pos[2 * c];
        vpb[c] = pos[2 * c + 1];
      }
    }
    auto fetch = [&](int src_, int start_, int cls_) {
      const int lo = cls_ == 0 ? klo[0] : (cls_ == 1 ? klo[1] : klo[2]);
      const int hi = cls_ == 0 ? khi[0] : (cls_ == 1 ? khi[1] : khi[2]);
      const int pa = cls_ == 0 ? vpa[0] : (cls_ == 1 ? vpa[1] : vpa[2]);
      const int pb = cls_ == 0 ? vpb[0] : (cls_ == 1 ? vpb[1] : vpb[2]);
      return keep_fetch(src_, start_, ii, half, lo, hi, pa, pb, vrow, srow);
    };
    // the row rotated for a class, into the query operand in TMEM (column c
    // holds dims 2c, 2c + 1; this thread: dims 32 half .. +31 and 64 + the same)
    auto write_q = [&](int cls_) {
      uint32_t wa[16], wb[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) wa[e] = wb[e] = 0u;
      if (real) {
        const float2* trow = p.tab + query_table_row(i, cls_, p.s, p.w, p.tab_c1) * 64;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int d0 = 32 * half + 8 * c;
          const uint4 xa = *reinterpret_cast<const uint4*>(qrow + d0);
          const uint4 xb = *reinterpret_cast<const uint4*>(qrow + 64 + d0);
          const float4* t4 = reinterpret_cast<const float4*>(trow + d0);
          const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&xa);
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xb);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float4 t = t4[e];
            const float2 x = __bfloat1622float2(a2[e]);
            const float2 y = __bfloat1622float2(b2[e]);
            wa[4 * c + e] = pack_bf16(x.x * t.x - y.x * t.y, x.y * t.z - y.y * t.w);
            wb[4 * c + e] = pack_bf16(x.x * t.y + y.x * t.x, x.y * t.w + y.y * t.z);
          }
        }
      }
      const uint32_t tq = tbase + lane_off + COL_Q + 16u * half;
      tmem_st16(tq, wa);
      tmem_st16(tq + 32u, wb);
      tmem_st_wait();
    };

    SparseIter it;
    sparse_iter_init(it);
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    int src = 0, start = 0, cls = CLS_INTRA;
    uint64_t keep = 0;
    if (N > 0) {
      sparse_iter_next(it, plan, src, start, cls);
      keep = keep_finish(fetch(src, start, cls), start, half);
      write_q(cls);  // the first class's query operand
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->q_ready);

    int st = 0;             // S buffer of item n (n mod NSBUF)
    uint32_t ph = 0u;       // its phase bits, one per buffer
    for (int n = 0; n < N && ok; ++n) {
      ok = wait_poll(&ctl->s_full[st], (ph >> st) & 1u, abort_flag, p.status, p.timeout_ns,
                     ST_SOFTMAX);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // the next item: its mask's loads are in flight during this item's softmax
      int src1 = src, start1 = start, cls1 = cls;
      KeepFetch kf;
      kf.src = 0;
      kf.a = kf.b = 0;
      if (n + 1 < N) {
        sparse_iter_next(it, plan, src1, start1, cls1);
        kf = fetch(src1, start1, cls1);
      }
      const uint32_t tS = tbase + lane_off + static_cast<uint32_t>(st * 128);
      const uint32_t tO = tbase + lane_off + COL_O;
      ok = sparse_half_step(tS, tO, n, keep, p, sc, m_ref, l_sum, pc, ctl, abort_flag, p.status);
      if (!ok) break;
      const uint64_t keep1 = keep_finish(kf, start1, half);
      // a class change: S(n) has completed, S(n + 1) waits for P(n), so the
      // operand tile is free for the next class's rotation
      if (n + 1 < N && cls1 != cls) write_q(cls1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[st]);
      ph ^= 1u << st;
      st = st == NSBUF - 1 ? 0 : st + 1;
      src = src1;
      start = start1;
      cls = cls1;
      keep = keep1;
    }
    // epilogue: O / (l_half0 + l_half1) -> bf16 -> out
    if (ok && N > 0) {
      ok = wait_bounded(&ctl->o_final, 0u, abort_flag, p.status, p.timeout_ns, ST_SOFTMAX);
      ok = __all_sync(0xffffffffu, ok);
    }
    float l_other = 0.f;
    if (ok) ok = pair_exchange(pc, l_sum, l_other, abort_flag, p.status, p.timeout_ns, ST_SOFTMAX);
    if (ok && N > 0) {
      const float l_tot = l_sum + l_other;
      tc_fence_after();
      const uint32_t tO = tbase + lane_off + COL_O + 64u * half;
      const float inv = 1.f / l_tot;
      __nv_bfloat16* orow =
          real ? p.out + ((i - p.q_start) * p.Hq + h) * static_cast<int64_t>(HD) + 64 * half
               : nullptr;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32u * c, o);
        if (real) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w4;
            w4.x = pack_bf16(__uint_as_float(o[8 * v4 + 0]) * inv, __uint_as_float(o[8 * v4 + 1]) * inv);
            w4.y = pack_bf16(__uint_as_float(o[8 * v4 + 2]) * inv, __uint_as_float(o[8 * v4 + 3]) * inv);
            w4.z = pack_bf16(__uint_as_float(o[8 * v4 + 4]) * inv, __uint_as_float(o[8 * v4 + 5]) * inv);
            w4.w = pack_bf16(__uint_as_float(o[8 * v4 + 6]) * inv, __uint_as_float(o[8 * v4 + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + 32 * c + 8 * v4) = w4;
          }
        }
      }
    }
  } else if (warp == WARP_LOAD) {
    // =========================================================== TMA producer
    if (lane == 0) {
      int last_li[NSLOT];
#pragma unroll
      for (int k = 0; k < NSLOT; ++k) last_li[k] = -1;
      SparseIter it;
      sparse_iter_init(it);
      bool ok = true;
      int src, start, cls;
      for (int n = 0; n < N && ok; ++n) {
        sparse_iter_next(it, plan, src, start, cls);
        for (int which = 0; which < 2; ++which) {  // 0: keys, 1: values
          const int li = 2 * n + which;
          const int slot = li % NSLOT;
          const int use = li / NSLOT;
          if (use > 0) {
            ok = wait_bounded(&ctl->slot_empty[slot], static_cast<uint32_t>((use - 1) & 1),
                              abort_flag, p.status, p.timeout_ns, ST_LOAD);
            if (!ok) break;
          }
          if ((p.debug & 1) && li == 0) continue;  // test hook: withhold the first key tile
          uint8_t* dst = slots + slot * TILE_BYTES;
          const CUtensorMap* tm = src == 1 ? (which ? &tm_v : &tm_k) : (which ? &tm_gv : &tm_gk);
          const int head_coord = src == 1 ? g : h;
          mbar_arrive_expect_tx(&ctl->slot_full[slot], TILE_BYTES);
          // rows from the item's first key (slash) or first position (vertical)
          tma_load_3d(dst, tm, &ctl->slot_full[slot], 0, head_coord, start);
          tma_load_3d(dst + HALF_BYTES, tm, &ctl->slot_full[slot], 64, head_coord, start);
          last_li[slot] = li;
        }
      }
      for (int k = 0; k < NSLOT; ++k)
        if (last_li[k] >= 0)
          wait_drain(&ctl->slot_full[k], static_cast<uint32_t>((last_li[k] / NSLOT) & 1),
                     p.status, p.timeout_ns, ST_DRAIN);
    }
    __syncwarp();
  } else if (warp == WARP_MMA) {
    // =========================================================== MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(BM, BN, false);
      const uint32_t id_o = idesc_bf16_f32(BM, HD, true);
      const uint64_t dk0 = sdesc_sw128(smem_u32(slots), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(slots), HALF_BYTES, 1024);
      auto full_wait = [&](int li) {
        return wait_spin(&ctl->slot_full[li % NSLOT], static_cast<uint32_t>((li / NSLOT) & 1),
                         abort_flag, p.status, p.timeout_ns, ST_MMA);
      };
      // S(k) = Q K^T into buffer k mod NSBUF (Q from TMEM, the key tile from
      // shared memory); the cursor stands after item `issued`,
      // cls_next its class, cls_prev the class of the last S issued
      SparseIter it;
      sparse_iter_init(it);
      int src_, start_, cls_next = -1, cls_prev = -1;
      int issued = 0, sb = 0;
      if (N > 0) sparse_iter_next(it, plan, src_, start_, cls_next);
      auto issue_s = [&]() {
        const int li = 2 * issued;
        const uint64_t dk = dk0 + static_cast<uint64_t>(((li % NSLOT) * TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4);
          mma_ts(tbase + static_cast<uint32_t>(sb * 128), tbase + COL_Q + static_cast<uint32_t>(kk * 8),
                 dk + off, id_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&ctl->s_full[sb]);
        mma_commit(&ctl->slot_empty[li % NSLOT]);
        ++issued;
        sb = sb == NSBUF - 1 ? 0 : sb + 1;
        cls_prev = cls_next;
        if (issued < N) sparse_iter_next(it, plan, src_, start_, cls_next);
      };
      // S(k) may go once P.V(k - NSBUF) is issued (its buffer), and, where
      // the class changes, once P(k - 1) is released (the query operand)
      auto can_issue = [&](int n_done) {  // P.V issued for items < n_done
        return issued < N && issued <= n_done + NSBUF - 1 &&
               (issued <= n_done || cls_next == cls_prev);
      };
      auto tile_landed = [&](int li) {
        return mbar_test_wait(&ctl->slot_full[li % NSLOT], static_cast<uint32_t>((li / NSLOT) & 1));
      };
      bool ok = wait_bounded(&ctl->q_ready, 0u, abort_flag, p.status, p.timeout_ns, ST_MMA);
      while (ok && can_issue(0)) {
        ok = full_wait(2 * issued);
        if (!ok) break;
        tc_fence_after();
        issue_s();
      }
      int pb = 0;        // buffer of P(n)
      uint32_t pph = 0;  // p_full phase bits, one per buffer
      // The key tile of S(k) lands in the slot that S(k - 3) frees, so no key
      // tile waits for a P.V.
      for (int n = 0; n < N && ok; ++n) {
        const int lv = 2 * n + 1;
        ok = full_wait(lv);
        // S ahead of P.V(n) where its key tile has already landed
        while (ok && can_issue(n) && tile_landed(2 * issued)) {
          tc_fence_after();
          issue_s();
        }
        // the key tile of the S that follows P.V(n): a wait between the P.V
        // and the S MMAs would leave the tensor pipe idle
        if (ok && can_issue(n + 1)) ok = full_wait(2 * issued);
        if (!ok) break;
        ok = wait_spin(&ctl->p_full[pb], (pph >> pb) & 1u, abort_flag, p.status, p.timeout_ns,
                       ST_MMA);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dv = dv0 + static_cast<uint64_t>(((lv % NSLOT) * TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          mma_ts(tbase + COL_O, tbase + static_cast<uint32_t>(pb * 128 + kk * 8),
                 dv + static_cast<uint64_t>((kk * 2048) >> 4), id_o, (n > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&ctl->pv_done[n & 1]);
        mma_commit(&ctl->slot_empty[lv % NSLOT]);
        pph ^= 1u << pb;
        pb = pb == NSBUF - 1 ? 0 : pb + 1;
        while (ok && can_issue(n + 1)) {
          ok = full_wait(2 * issued);
          if (!ok) break;
          tc_fence_after();
          issue_s();
        }
      }
      if (ok && N > 0) mma_commit(&ctl->o_final);
      mma_commit(&ctl->drain);
      wait_drain(&ctl->drain, 0u, p.status, p.timeout_ns, ST_DRAIN);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace sp

cudaError_t launch_sparse_sm100(const AttnArgs& a, const SparseArgs& sa, cudaStream_t st) {
  using namespace sp;
  if (a.Lq <= 0) return cudaSuccess;
  CUtensorMap tm_k, tm_v, tm_gk, tm_gv;
  if (!encode_kv_map(&tm_k, a.kr, a.Lk, a.Hkv) || !encode_kv_map(&tm_v, a.v, a.Lk, a.Hkv) ||
      !encode_kv_map(&tm_gk, sa.gk, sa.nv_cap, a.Hq) ||
      !encode_kv_map(&tm_gv, sa.gv, sa.nv_cap, a.Hq))
    return cudaErrorInvalidValue;
  Params p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.tab = a.tab;
  p.vidx = sa.vidx;
  p.nv = sa.nv;
  p.runs = sa.runs;
  p.nruns = sa.nruns;
  p.vbit = sa.vbit;
  p.sbit = sa.sbit;
  p.wpr = sa.wpr;
  p.nv_cap = sa.nv_cap;
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
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  p.debug = a.debug;
  const int64_t blocks = static_cast<int64_t>(p.n_qtiles) * p.Hq;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(dca_sparse_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  dca_sparse_kernel<<<static_cast<unsigned>(blocks), NUM_THREADS, SMEM_BYTES, st>>>(
      tm_k, tm_v, tm_gk, tm_gv, p);
  return cudaGetLastError();
}

}  // namespace dca
