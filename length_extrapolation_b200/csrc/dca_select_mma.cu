// dca_select_mma.cu -- the score passes of the key selection on the tensor
// cores (dca_select.cu holds the rest of the selection and states what it
// computes: vertical and slash sums of the last rows' softmax).
//
// One CTA = one query head x one slice of 4096 keys.  The 64 estimate rows
// are the MMA N: S^T = K' Q_v^T (M = 128 keys, N = 64 rows, K = 128 dims,
// tcgen05.mma kind::f16, fp32 accumulators in TMEM), so TMEM lane t holds
// key t's logits for all rows and each softmax thread owns one key.
//
// The query operand is the fp32 rotated query row (log2 units) split into
// bf16 hi + lo parts, two MMAs accumulating into one S^T, so the logits keep
// the precision of an fp32 dot product with the bf16 cached keys.  DCA: one
// operand per pair class (INTER, SUCC, INTRA ranges, as in dca_plan.cuh).
// Continuous positions: <R(i) q, R(j) k> = <R(-s n_j) R(i) q, R(j mod s) k>,
// so the cached keys are used as they are and the operand is the query
// rotated back by its key chunk's angle; a work item is (key tile, chunk)
// and two operand buffers alternate as the chunk advances.
//
// Two passes over the same items:
//   1  per thread and row an online (max, sum of 2^(x - max)) over its keys,
//      merged over the CTA's 128 threads and written per (head, slice, row);
//      sel_stats_kernel merges the slices;
//   2  p = 2^(x - M) / L: the per-key sum over the rows (vertical) into a
//      shared-memory bin per key of the slice; the sums along the diagonals
//      i - j (slash) in registers, one lane per diagonal class mod 32 fed by a
//      rotating shuffle, then into a bin per offset; the bins are stored /
//      added to the score arrays once per CTA.
// The rows of an item's class (and of causality) are one contiguous range
// per key (class_row_range), so masking is a range test.
// Warps: 0-3 softmax, 4 TMA producer (ring of 3 -- continuous positions: 4 --
// 32 KiB key tiles, no multicast), 5 MMA issuer.  Every mbarrier wait is bounded; on timeout the
// CTA raises its abort flag, ORs a code into the status word, drains its
// copies and MMAs, frees TMEM and exits.  The softmax warps' own barriers
// (bar.sync 1, 128) are reached by all four warps on every path.
#include <cuda_bf16.h>
#include <math.h>

#include <type_traits>

#include "dca_internal.h"
#include "dca_plan.cuh"
#include "sm100_ptx.cuh"

namespace dca {
namespace selm {

constexpr int ROWS = 64, BN = 128, HD = 128;
constexpr int SLICE = 4096;               // keys per CTA
constexpr int NSLOT = 3;                  // key-tile ring (DCA)
constexpr int NSLOT_MAX = 4;              // continuous: a 4th slot in the unused operand space
constexpr int TILE_BYTES = 32768, HALF_BYTES = 16384;
constexpr int QOP = ROWS * HD * 2;        // 16 KiB: one bf16 query operand
constexpr int QOP_HALF = ROWS * 128;      // its 64-column block
constexpr int NOPND = 6;                  // DCA: 3 classes x (hi, lo); continuous: 2 x (hi, lo)
constexpr int THREADS = 192;
constexpr int WARP_LOAD = 4, WARP_MMA = 5;
constexpr uint32_t TMEM_COLS = 128;       // two S^T buffers of 64 columns
constexpr int SBINS = SLICE + ROWS;       // offsets i - j met by a slice
constexpr int MSTRIDE = 136;              // row stride of the merge buffers (conflict-free)
constexpr int MROWS = 16;                 // rows per merge round
// pass 2: vertical bins [SLICE] (key j is always updated by one thread) and
// the slash bins [SBINS] (each lane adds its three diagonal sums once per
// item, atomically: the warps' diagonal ranges overlap)
constexpr int BIN_FLOATS =
    (SLICE + SBINS) > 2 * MROWS * MSTRIDE ? (SLICE + SBINS) : 2 * MROWS * MSTRIDE;
constexpr float NEG_BIG = -1e30f;         // finite "no value yet" maximum

constexpr unsigned ST_SOFTMAX = 0x10u, ST_LOAD = 0x100u, ST_MMA = 0x1000u, ST_DRAIN = 0x10000u;

struct SmemCtl {
  uint64_t slot_full[NSLOT_MAX];
  uint64_t slot_empty[NSLOT_MAX];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t op_full[2];      // a query operand buffer is written (4 warp arrivals)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int n_items;
  int lo[3], hi[3];         // DCA: k-tile range per class, clipped to the slice
  int kt0;                  // continuous: first k-tile of the slice
  int64_t kend;             // continuous: end of the slice's causal keys
  int64_t c_first, c_last;  // continuous: key chunks met
};

constexpr size_t SMEM_BYTES =
    1024 + NSLOT * TILE_BYTES + NOPND * QOP + sizeof(float) * BIN_FLOATS + sizeof(SmemCtl);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

struct Params {
  const float* qv;          // [Hq][nvar][ROWS][HD] rotated query rows, log2 units
  const float2* crot;       // continuous: (cos, sin) of s*n*theta_k [n_chunks][64]
  float2* part;             // pass 1 out: [Hq][n_slices][ROWS] (max, sum)
  const float2* stats;      // pass 2 in: [Hq][ROWS] (max, sum)
  float* vert;              // pass 2 out: [Hq][Lk]
  float* slash;             // pass 2 out: [Hq][Lk] (accumulated)
  int64_t i_first, Lk, s, w;
  int n_last, Hq, Hkv, G, n_slices, reading, continuous;
  unsigned int* status;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// The work item cursor: DCA walks the class ranges (INTER, SUCC, INTRA), the
// continuous mode the (k-tile, chunk) pairs of the slice in key order.
struct Cursor {
  int n;       // item index
  int kt;      // k-tile
  int v;       // DCA: class; continuous: chunk - c_first
  int64_t c;   // continuous: key chunk
};

__device__ __forceinline__ void dca_item(const SmemCtl* ctl, Cursor& it) {
  const int c2 = ctl->hi[CLS_INTER] - ctl->lo[CLS_INTER];
  const int c1 = ctl->hi[CLS_SUCC] - ctl->lo[CLS_SUCC];
  if (it.n < c2) {
    it.v = CLS_INTER;
    it.kt = ctl->lo[CLS_INTER] + it.n;
  } else if (it.n < c2 + c1) {
    it.v = CLS_SUCC;
    it.kt = ctl->lo[CLS_SUCC] + (it.n - c2);
  } else {
    it.v = CLS_INTRA;
    it.kt = ctl->lo[CLS_INTRA] + (it.n - c2 - c1);
  }
}

__device__ __forceinline__ Cursor first_item(const SmemCtl* ctl, const Params& p) {
  Cursor it;
  it.n = 0;
  if (p.continuous) {
    it.kt = ctl->kt0;
    it.c = ctl->c_first;
    it.v = 0;
  } else {
    dca_item(ctl, it);
    it.c = 0;
  }
  return it;
}

__device__ __forceinline__ void next_item(const SmemCtl* ctl, const Params& p, Cursor& it) {
  ++it.n;
  if (p.continuous) {
    const int64_t tile_end = static_cast<int64_t>(it.kt) * BN + BN;
    const int64_t last = (tile_end < ctl->kend ? tile_end : ctl->kend) - 1;
    const uint32_t s32 = static_cast<uint32_t>(p.s);
    if (it.c < static_cast<uint32_t>(last) / s32) {
      ++it.c;
    } else {
      ++it.kt;
      it.c = static_cast<uint32_t>(it.kt * BN) / s32;
    }
    it.v = static_cast<int>(it.c - ctl->c_first);
  } else {
    dca_item(ctl, it);
  }
}

// bf16 hi + lo of the fp32 row values (a, b): the lo parts carry the rounding
// error of the hi parts.
__device__ __forceinline__ void split_pack(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Query operand pair (hi at op_hi, lo at op_hi + QOP): K-major, 128-byte
// swizzle, from the fp32 rows `src` [ROWS][HD], rotated back by the chunk
// angles `cs` (continuous) or as they are (cs == nullptr).  128 threads.
__device__ __forceinline__ void build_operand(uint8_t* op_hi, const float* __restrict__ src,
                                              const float2* __restrict__ cs, int tau) {
#pragma unroll
  for (int task = tau; task < ROWS * 8; task += 128) {  // all loads issued together
    const int r = task >> 3, c = task & 7;
    const float* row = src + r * HD;
    const float4 a0 = *reinterpret_cast<const float4*>(row + 8 * c);
    const float4 a1 = *reinterpret_cast<const float4*>(row + 8 * c + 4);
    const float4 b0 = *reinterpret_cast<const float4*>(row + 64 + 8 * c);
    const float4 b1 = *reinterpret_cast<const float4*>(row + 64 + 8 * c + 4);
    float xa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    float xb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
    if (cs != nullptr) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float2 t = cs[8 * c + e];  // R(-phi): (a cos + b sin, b cos - a sin)
        const float ra = xa[e] * t.x + xb[e] * t.y;
        const float rb = xb[e] * t.x - xa[e] * t.y;
        xa[e] = ra;
        xb[e] = rb;
      }
    }
    uint4 ha, la, hb, lb;
    uint32_t* pha = reinterpret_cast<uint32_t*>(&ha);
    uint32_t* pla = reinterpret_cast<uint32_t*>(&la);
    uint32_t* phb = reinterpret_cast<uint32_t*>(&hb);
    uint32_t* plb = reinterpret_cast<uint32_t*>(&lb);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      split_pack(xa[2 * e], xa[2 * e + 1], pha[e], pla[e]);
      split_pack(xb[2 * e], xb[2 * e + 1], phb[e], plb[e]);
    }
    uint8_t* d = op_hi + r * 128 + ((c ^ (r & 7)) << 4);
    *reinterpret_cast<uint4*>(d) = ha;
    *reinterpret_cast<uint4*>(d + QOP_HALF) = hb;
    *reinterpret_cast<uint4*>(d + QOP) = la;
    *reinterpret_cast<uint4*>(d + QOP + QOP_HALF) = lb;
  }
}

// (max, sum) merge of two partial row statistics (maxima finite).
__device__ __forceinline__ float2 merge_stat(float2 a, float2 b) {
  const float m = fmaxf(a.x, b.x);
  return make_float2(m, a.y * exp2f(a.x - m) + b.y * exp2f(b.x - m));
}

template <int PASS>
__global__ void __launch_bounds__(THREADS, 1)
    sel_mma_kernel(const __grid_constant__ CUtensorMap tm_k, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* slots = smem;
  uint8_t* opnd = slots + NSLOT * TILE_BYTES;
  float* bins = reinterpret_cast<float*>(opnd + NOPND * QOP);
  float* vbin = bins;            // [SLICE]     pass 2
  float* sbin = bins + SLICE;    // [SBINS]     pass 2
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(bins + BIN_FLOATS);

  // key-tile ring: 3 slots, and in continuous mode (4 operands, not 6) a
  // fourth slot in the operand space it leaves free
  const int nslot = p.continuous ? NSLOT_MAX : NSLOT;
  auto slot_at = [&](int k) { return k < NSLOT ? slots + k * TILE_BYTES : opnd + 4 * QOP; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the G heads of one KV group and slice are adjacent: they read the same keys
  const int hh = static_cast<int>(blockIdx.x) % p.G;
  const int rest = static_cast<int>(blockIdx.x) / p.G;
  const int sl = rest % p.n_slices;
  const int g = rest / p.n_slices;
  const int h = g * p.G + hh;
  const int64_t ka = static_cast<int64_t>(sl) * SLICE;
  const int64_t i_last = p.i_first + p.n_last - 1;

  if (threadIdx.x == 0) {
    for (int k = 0; k < NSLOT_MAX; ++k) {
      mbar_init(&ctl->slot_full[k], 1);
      mbar_init(&ctl->slot_empty[k], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&ctl->s_full[k], 1);
      mbar_init(&ctl->s_free[k], 4);
      mbar_init(&ctl->op_full[k], 4);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    int n = 0;
    if (p.continuous) {
      int64_t kend = ka + SLICE;
      if (kend > i_last + 1) kend = i_last + 1;
      if (kend > p.Lk) kend = p.Lk;
      ctl->kend = kend;
      ctl->kt0 = static_cast<int>(ka / BN);
      if (kend > ka) {
        ctl->c_first = ka / p.s;
        ctl->c_last = (kend - 1) / p.s;
        // items: per k-tile, the chunks its causal keys meet
        for (int64_t t0 = ka; t0 < kend; t0 += BN) {
          const int64_t t1 = (t0 + BN < kend ? t0 + BN : kend) - 1;
          n += static_cast<int>(t1 / p.s - t0 / p.s + 1);
        }
      } else {
        ctl->c_first = ctl->c_last = 0;
      }
    } else {
      const TilePlan P = make_plan(p.i_first, i_last, p.s, p.w, BN, p.reading);
      const int t0 = static_cast<int>(ka / BN), t1 = static_cast<int>((ka + SLICE) / BN);
      for (int c = 0; c < 3; ++c) {
        const int a = P.lo[c] > t0 ? P.lo[c] : t0;
        int b = P.hi[c] < t1 ? P.hi[c] : t1;
        if (b < a) b = a;
        ctl->lo[c] = a;
        ctl->hi[c] = b;
        n += b - a;
      }
    }
    ctl->n_items = n;
    fence_barrier_init();
  }
  if (PASS == 2)
    for (int e = threadIdx.x; e < SLICE + SBINS; e += THREADS) bins[e] = 0.f;
  if (warp == WARP_MMA) {
    tmem_alloc(&ctl->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == WARP_LOAD && lane == 0) tma_prefetch_desc(&tm_k);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = ctl->tmem_base;
  volatile int* abort_flag = &ctl->abort;
  const int N = ctl->n_items;

  if (warp < 4) {
    // =========================================================== softmax warps
    const int tau = warp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float* qh = p.qv + static_cast<int64_t>(h) * (p.continuous ? 1 : 3) * ROWS * HD;
    if (N > 0) {
      if (p.continuous) {
        build_operand(opnd, qh, p.crot + ctl->c_first * (HD / 2), tau);
        if (ctl->c_first + 1 <= ctl->c_last)
          build_operand(opnd + 2 * QOP, qh, p.crot + (ctl->c_first + 1) * (HD / 2), tau);
      } else {
        for (int v = 0; v < 3; ++v)
          build_operand(opnd + 2 * v * QOP, qh + v * ROWS * HD, nullptr, tau);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ctl->op_full[0]);
        if (p.continuous && ctl->c_first + 1 <= ctl->c_last) mbar_arrive(&ctl->op_full[1]);
      }
    }

    // pass 1: running (max, sum) per row; pass 2: C_r = M_r + log2 L_r, so
    // p = 2^(x - C_r)
    constexpr int NR1 = PASS == 1 ? ROWS : 1, NR2 = PASS == 2 ? ROWS : 1;
    float m[NR1], l[NR1], C[NR2];
#pragma unroll
    for (int r = 0; r < NR1; ++r) {
      m[r] = NEG_BIG;
      l[r] = 0.f;
    }
    if (PASS == 2) {
#pragma unroll
      for (int r = 0; r < NR2; ++r) {
        const float2 st = p.stats[h * ROWS + r];
        C[r] = st.y > 0.f ? st.x + __log2f(st.y) : 0.f;
      }
    }
    Cursor it = first_item(ctl, p);
    for (int n = 0; n < N; ++n) {
      const int buf = n & 1;
      if (!wait_warp(&ctl->s_full[buf], static_cast<uint32_t>((n >> 1) & 1), abort_flag, p.status,
                     p.timeout_ns, ST_SOFTMAX, lane))
        break;
      tc_fence_after();
      const int64_t j = static_cast<int64_t>(it.kt) * BN + tau;
      int ra, rb;
      class_row_range(j, p.i_first, p.n_last, p.Lk, p.s, p.w, p.reading,
                      p.continuous ? -1 : it.v, p.continuous ? it.c : -1, &ra, &rb);
      // every row of every lane valid: no masks (the common case)
      const bool full = __all_sync(0xffffffffu, ra == 0 && rb == ROWS);
      float vsum = 0.f;
      // slash: the warp's 32 keys and 64 rows meet the diagonals d = r - t,
      // t = lane of the key; lane L owns those with d = L (mod 32), d in
      // [-31, 63]: a0 (d = L - 32), a1 (d = L), a2 (d = L + 32).  At row r the
      // value p(r, (r - L) mod 32) is on one of lane L's diagonals.
      float a0 = 0.f, a1 = 0.f, a2 = 0.f;
      // the rows of one half of S^T: online stats (pass 1) or probabilities,
      // their vertical and diagonal sums (pass 2); MASKED applies [ra, rb)
      auto rows_of_half = [&](const uint32_t* sv, const int half, auto masked) {
        constexpr bool MASKED = decltype(masked)::value;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int r = half * 32 + e;
          if (PASS == 1) {
            float x = __uint_as_float(sv[e]);
            if (MASKED) x = (r >= ra && r < rb) ? x : -INFINITY;
            const float d = x - m[r];  // m is finite: a masked x gives -inf, t = 0
            const float t = ex2_approx(-fabsf(d));
            const bool up = d > 0.f;
            l[r] = up ? fmaf(l[r], t, 1.f) : l[r] + t;
            m[r] = up ? x : m[r];
          } else {
            float pr = ex2_approx(__uint_as_float(sv[e]) - C[r]);
            if (MASKED) pr = (r >= ra && r < rb) ? pr : 0.f;
            vsum += pr;
            // source lane (r - L) mod 32: the shuffle takes the index mod 32
            const float v = __shfl_sync(0xffffffffu, pr, r - lane);
            if (r < 32) {
              if (lane <= r) a1 += v; else a0 += v;
            } else {
              if (lane <= r - 32) a2 += v; else a1 += v;
            }
          }
        }
      };
      // one version per case, so no branch sits between the rows
      auto item_rows = [&](auto masked) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t sv[32];
          tmem_ld32(tbase + lane_off + static_cast<uint32_t>(buf * ROWS + half * 32), sv);
          if (half == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->s_free[buf]);
          }
          rows_of_half(sv, half, masked);
        }
      };
      if (full)
        item_rows(std::false_type{});
      else
        item_rows(std::true_type{});
      if (PASS == 2) {
        vbin[j - ka] += vsum;  // key j is always this thread's
        // bin of diagonal d: offset i - j minus the slice's smallest offset,
        // (ka + SLICE - 1 - j_t) + r = (ka + SLICE - 1 - j_0) + d
        float* bw = sbin + (ka + SLICE - 1 - (static_cast<int64_t>(it.kt) * BN + warp * 32));
        if (lane > 0) atomicAdd(&bw[lane - 32], a0);
        atomicAdd(&bw[lane], a1);
        atomicAdd(&bw[lane + 32], a2);
      }

      // continuous: the last item of chunk c frees its operand buffer for c + 2
      if (p.continuous) {
        const int64_t c = it.c;
        next_item(ctl, p, it);
        if ((n + 1 == N || it.c != c) && c + 2 <= ctl->c_last) {
          build_operand(opnd + 2 * static_cast<int>((c - ctl->c_first) & 1) * QOP, qh,
                        p.crot + (c + 2) * (HD / 2), tau);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->op_full[(c - ctl->c_first) & 1]);
        }
      } else {
        next_item(ctl, p, it);
      }
    }

    // ---- per-CTA results (every softmax warp runs this, whatever happened)
    if (PASS == 1) {
      float* mb = bins;
      float* lb = bins + MROWS * MSTRIDE;
      const int rr = tau >> 3, q = tau & 7;
#pragma unroll
      for (int round = 0; round < ROWS / MROWS; ++round) {
        if (round > 0) softmax_bar();  // the previous round's reads are done
#pragma unroll
        for (int e = 0; e < MROWS; ++e) {
          mb[e * MSTRIDE + tau] = m[round * MROWS + e];
          lb[e * MSTRIDE + tau] = l[round * MROWS + e];
        }
        softmax_bar();
        float2 acc = make_float2(NEG_BIG, 0.f);
#pragma unroll
        for (int e = 0; e < 128 / 8; ++e)
          acc = merge_stat(acc, make_float2(mb[rr * MSTRIDE + q + 8 * e], lb[rr * MSTRIDE + q + 8 * e]));
#pragma unroll
        for (int off = 1; off < 8; off <<= 1)
          acc = merge_stat(acc, make_float2(__shfl_xor_sync(0xffffffffu, acc.x, off),
                                            __shfl_xor_sync(0xffffffffu, acc.y, off)));
        if (q == 0)
          p.part[(static_cast<int64_t>(h) * p.n_slices + sl) * ROWS + round * MROWS + rr] = acc;
      }
    } else {
      softmax_bar();  // every bin update is done
      float* vrow = p.vert + static_cast<int64_t>(h) * p.Lk;
      float* srow = p.slash + static_cast<int64_t>(h) * p.Lk;
      for (int e = tau; e < SLICE; e += 128) {
        const int64_t jj = ka + e;
        if (jj < p.Lk) vrow[jj] = vbin[e];
      }
      const int64_t o0 = p.i_first - (ka + SLICE - 1);
      for (int e = tau; e < SBINS; e += 128) {
        const float v = sbin[e];
        const int64_t o = o0 + e;
        if (v != 0.f && o >= 0 && o < p.Lk) atomicAdd(&srow[o], v);
      }
    }
  } else if (warp == WARP_LOAD) {
    // =========================================================== TMA producer
    if (lane == 0) {
      int last[NSLOT_MAX];
#pragma unroll
      for (int k = 0; k < NSLOT_MAX; ++k) last[k] = -1;
      Cursor it = first_item(ctl, p);
      for (int n = 0; n < N; ++n) {
        const int slot = n % nslot, use = n / nslot;
        if (use > 0 &&
            !wait_bounded(&ctl->slot_empty[slot], static_cast<uint32_t>((use - 1) & 1),
                          abort_flag, p.status, p.timeout_ns, ST_LOAD))
          break;
        uint8_t* dst = slot_at(slot);
        mbar_arrive_expect_tx(&ctl->slot_full[slot], TILE_BYTES);
        tma_load_3d(dst, &tm_k, &ctl->slot_full[slot], 0, g, it.kt * BN);
        tma_load_3d(dst + HALF_BYTES, &tm_k, &ctl->slot_full[slot], 64, g, it.kt * BN);
        last[slot] = n;
        next_item(ctl, p, it);
      }
      for (int k = 0; k < nslot; ++k)
        if (last[k] >= 0)
          wait_drain(&ctl->slot_full[k], static_cast<uint32_t>((last[k] / nslot) & 1), p.status,
                     p.timeout_ns, ST_DRAIN);
    }
    __syncwarp();
  } else if (warp == WARP_MMA) {
    // =========================================================== MMA issuer
    if (lane == 0) {
      const uint32_t id = idesc_bf16_f32_major(BN, ROWS, false, false);
      const uint64_t dq0 = sdesc_sw128(smem_u32(opnd), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(slots), 16, 1024);
      bool ok = true;
      Cursor it = first_item(ctl, p);
      int64_t have = -1;  // the operand (class set or chunk) known to be written
      for (int n = 0; n < N && ok; ++n) {
        const int slot = n % nslot;
        // operand readiness: DCA once; continuous once per chunk
        const int64_t need = p.continuous ? it.c : 0;
        if (need != have) {
          const int ci = p.continuous ? it.v : 0;
          ok = wait_spin(&ctl->op_full[ci & 1], static_cast<uint32_t>((ci >> 1) & 1), abort_flag,
                         p.status, p.timeout_ns, ST_MMA);
          if (!ok) break;
          have = need;
        }
        ok = wait_spin(&ctl->slot_full[slot], static_cast<uint32_t>((n / nslot) & 1), abort_flag,
                       p.status, p.timeout_ns, ST_MMA);
        if (!ok) break;
        if (n >= 2) {
          ok = wait_spin(&ctl->s_free[n & 1], static_cast<uint32_t>(((n - 2) >> 1) & 1),
                         abort_flag, p.status, p.timeout_ns, ST_MMA);
          if (!ok) break;
        }
        tc_fence_after();
        const int op = p.continuous ? 2 * (it.v & 1) : 2 * it.v;
        const uint64_t dk = dk0 + static_cast<uint64_t>((slot_at(slot) - slots) >> 4);
        const uint32_t d_tmem = tbase + static_cast<uint32_t>((n & 1) * ROWS);
#pragma unroll
        for (int part = 0; part < 2; ++part) {  // hi, then lo
          const uint64_t dq = dq0 + static_cast<uint64_t>(((op + part) * QOP) >> 4);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint64_t a_off = static_cast<uint64_t>(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4);
            const uint64_t b_off = static_cast<uint64_t>(((kk >> 2) * QOP_HALF + (kk & 3) * 32) >> 4);
            mma_ss(d_tmem, dk + a_off, dq + b_off, id, (part > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(&ctl->s_full[n & 1]);
        mma_commit(&ctl->slot_empty[slot]);
        next_item(ctl, p, it);
      }
      mma_commit(&ctl->drain);
      wait_drain(&ctl->drain, 0u, p.status, p.timeout_ns, ST_DRAIN);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tbase, TMEM_COLS);
  }
}

}  // namespace selm

int select_slices(int64_t Lk) { return static_cast<int>((Lk + selm::SLICE - 1) / selm::SLICE); }

cudaError_t launch_select_scores(const void* kr, const float* qv, const float2* crot, float2* part,
                                 const float2* stats, float* vert, float* slash, int64_t i_first,
                                 int64_t Lk, int64_t s, int64_t w, int n_last, int Hq, int Hkv,
                                 int reading, int continuous, int pass, unsigned int* status,
                                 unsigned long long timeout_ns, cudaStream_t st) {
  using namespace selm;
  CUtensorMap tm_k;
  if (!encode_kv_map(&tm_k, kr, Lk, Hkv)) return cudaErrorInvalidValue;
  Params p;
  p.qv = qv;
  p.crot = crot;
  p.part = part;
  p.stats = stats;
  p.vert = vert;
  p.slash = slash;
  p.i_first = i_first;
  p.Lk = Lk;
  p.s = s;
  p.w = w;
  p.n_last = n_last;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_slices = select_slices(Lk);
  p.reading = reading;
  p.continuous = continuous;
  p.status = status;
  p.timeout_ns = timeout_ns;
  const int64_t blocks = static_cast<int64_t>(p.n_slices) * Hq;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  auto kern = pass == 1 ? sel_mma_kernel<1> : sel_mma_kernel<2>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(blocks), THREADS, SMEM_BYTES, st>>>(tm_k, p);
  return cudaGetLastError();
}

}  // namespace dca
