// dca_select_mma.cu -- the score passes of the key selection on the tensor
// cores (dca_select.cu holds the rest of the selection and states what it
// computes: vertical and slash sums of the last rows' softmax).
//
// The query operand is the fp32 rotated query row (log2 units) split into
// bf16 hi + lo parts, two MMAs accumulating into one S, so the logits keep
// the precision of an fp32 dot product with the bf16 cached keys.  DCA: one
// operand per pair class (INTER, SUCC, INTRA ranges, as in dca_plan.cuh).
// Continuous positions: <R(i) q, R(j) k> = <R(-s n_j) R(i) q, R(j mod s) k>,
// so the cached keys are used as they are and the operand is the query
// rotated back by its key chunk's angle; a work item is (key tile, chunk).
//
// Pass 1 (sel_rows_kernel, the row statistics) is described at its kernel.
// Pass 2 (sel_sums_kernel): one CTA = one query head x one slice of 4096
// keys.  The 64 estimate rows are the MMA N: S^T = K' Q_v^T (M = 128 keys,
// N = 64 rows, K = 128 dims, fp32 accumulators in TMEM), so TMEM lane t holds
// key t's logits for all rows and each softmax thread owns one key.
// p = 2^(x - M) / L: the per-key sum over the rows (vertical) goes into a
// shared-memory bin per key of the slice; the sums along the diagonals i - j
// (slash) into registers, one lane per diagonal class mod 32 fed by a
// rotating shuffle, then once per item into a bin per offset; the bins are
// stored / added to the score arrays once per CTA.  The rows of an item's
// class (and of causality) are one contiguous range per key
// (class_row_range), so masking is a range test.  Warps: 0-7 softmax (two per
// SMSP: warp w reads the TMEM lane quarter w % 4, i.e. 32 keys, and rows
// 32 (w / 4) .. + 31), 8 TMA producer (ring of 3 -- continuous positions: 4
// -- 32 KiB key tiles, no multicast), 9 MMA issuer; DCA keeps the three
// class operands, continuous positions two chunk operands that alternate as
// the chunk advances.  Every mbarrier wait is bounded; on timeout the CTA
// raises its abort flag, ORs a code into the status word, drains its copies
// and MMAs, frees TMEM and exits.  The softmax warps' own barriers
// (bar.sync 1, 256) are reached by all eight warps on every path.
#include <cuda_bf16.h>
#include <math.h>

#include <type_traits>

#include "dca_internal.h"
#include "dca_plan.cuh"
#include "dca_select_rows.cuh"
#include "dca_softmax.cuh"
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
constexpr int SM_WARPS = 8;               // softmax warps: 2 per SMSP
constexpr int SM_THREADS = 32 * SM_WARPS;
constexpr int THREADS = SM_THREADS + 64;
constexpr int WARP_LOAD = SM_WARPS, WARP_MMA = SM_WARPS + 1;
constexpr int NSBUF = 4;                  // S^T buffers in TMEM (the MMA runs up to 3 items ahead)
constexpr uint32_t TMEM_COLS = NSBUF * ROWS;
constexpr int SBINS = SLICE + ROWS;       // offsets i - j met by a slice
// vertical bins [SLICE] (key j: one atomic add per row half) and slash bins
// [SBINS] (each lane adds its two diagonal sums once per item, atomically:
// the warps' diagonal ranges overlap)
constexpr int BIN_FLOATS = SLICE + SBINS;
constexpr float NEG_BIG = -1e30f;         // finite "no value yet" maximum

constexpr unsigned ST_SOFTMAX = 0x10u, ST_LOAD = 0x100u, ST_MMA = 0x1000u, ST_DRAIN = 0x10000u;

struct SmemCtl {
  uint64_t slot_full[NSLOT_MAX];
  uint64_t slot_empty[NSLOT_MAX];
  uint64_t s_full[NSBUF];
  uint64_t s_free[NSBUF];
  uint64_t op_full[2];      // a query operand buffer is written (one arrival per softmax warp)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int n_items;
  int rot;                  // item order rotation (see phys_item)
  int lo[3], hi[3];         // DCA: k-tile range per class, clipped to the slice
  int kt0;                  // continuous: first k-tile of the slice
  int64_t kend;             // continuous: end of the slice's causal keys
  int64_t c_first, c_last;  // continuous: key chunks met
};

constexpr size_t SMEM_BYTES =
    1024 + NSLOT * TILE_BYTES + NOPND * QOP + sizeof(float) * BIN_FLOATS + sizeof(SmemCtl);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(SLICE % BN == 0 && SLICE / BN <= 32, "one counting lane per k-tile of a slice");

struct Params {
  const float* qv;          // [Hq][nvar][ROWS][HD] rotated query rows, log2 units
  const float2* crot;       // continuous: (cos, sin) of s*n*theta_k [n_chunks][64]
  const float2* stats;      // [Hq][ROWS] (max, sum) over all keys
  float* vert;              // out: [Hq][Lk]
  float* slash;             // out: [Hq][Lk] (accumulated)
  int64_t i_first, Lk, s, w;
  int n_last, Hq, Hkv, G, n_slices, reading, continuous;
  unsigned int* status;
  unsigned long long timeout_ns;
};


// How the score passes wait: the softmax warps for S and the MMA thread for
// its inputs.  DCA_SEL_POLL = 1 polls without sleeping, as the attention
// kernels do (measured 11% faster over a 1M-key selection than backing off
// with __nanosleep between polls, 0).
#ifndef DCA_SEL_POLL
#define DCA_SEL_POLL 1
#endif
__device__ __forceinline__ bool sel_sm_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                            unsigned int* status, uint64_t timeout_ns,
                                            unsigned int code, int lane) {
#if DCA_SEL_POLL
  (void)lane;
  return __all_sync(0xffffffffu, wait_poll(bar, parity, abort, status, timeout_ns, code));
#else
  return wait_warp(bar, parity, abort, status, timeout_ns, code, lane);
#endif
}
__device__ __forceinline__ bool sel_mma_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                             unsigned int* status, uint64_t timeout_ns,
                                             unsigned int code) {
#if DCA_SEL_POLL
  return wait_poll(bar, parity, abort, status, timeout_ns, code);
#else
  return wait_spin(bar, parity, abort, status, timeout_ns, code);
#endif
}

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// The work item cursor: DCA walks the class ranges (INTER, SUCC, INTRA), the
// continuous mode the (k-tile, chunk) pairs of the slice in key order.
struct Cursor {
  int n;       // item index
  int kt;      // k-tile
  int v;       // DCA: class; continuous: chunk - c_first
  int64_t c;   // continuous: key chunk
};

// The G CTAs of a KV group walk the slice's items from different starting
// points (item n is the list's item (n + rot) mod N, rot = hh N / G), so
// they do not all ask L2 for the same key tile at once.  Continuous
// positions rotate only a single-chunk slice (the operand buffers need the
// chunks in order).
template <class Ctl>
__device__ __forceinline__ int phys_item(const Ctl* ctl, int n) {
  const int q = n + ctl->rot;
  return q >= ctl->n_items ? q - ctl->n_items : q;
}

template <class Ctl>
__device__ __forceinline__ void dca_item(const Ctl* ctl, Cursor& it) {
  const int c2 = ctl->hi[CLS_INTER] - ctl->lo[CLS_INTER];
  const int c1 = ctl->hi[CLS_SUCC] - ctl->lo[CLS_SUCC];
  const int q = phys_item(ctl, it.n);
  if (q < c2) {
    it.v = CLS_INTER;
    it.kt = ctl->lo[CLS_INTER] + q;
  } else if (q < c2 + c1) {
    it.v = CLS_SUCC;
    it.kt = ctl->lo[CLS_SUCC] + (q - c2);
  } else {
    it.v = CLS_INTRA;
    it.kt = ctl->lo[CLS_INTRA] + (q - c2 - c1);
  }
}

template <class Ctl, class Prm>
__device__ __forceinline__ Cursor first_item(const Ctl* ctl, const Prm& p) {
  Cursor it;
  it.n = 0;
  if (p.continuous) {
    it.kt = ctl->kt0 + (ctl->c_first == ctl->c_last ? phys_item(ctl, 0) : 0);
    it.c = ctl->c_first;
    it.v = 0;
  } else {
    dca_item(ctl, it);
    it.c = 0;
  }
  return it;
}

template <class Ctl, class Prm>
__device__ __forceinline__ void next_item(const Ctl* ctl, const Prm& p, Cursor& it) {
  ++it.n;
  if (p.continuous && ctl->c_first == ctl->c_last) {
    it.kt = ctl->kt0 + phys_item(ctl, it.n);  // one item per k-tile
  } else if (p.continuous) {
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
// angles `cs` (continuous) or as they are (cs == nullptr).  The softmax warps'
// 256 threads.
__device__ __forceinline__ void build_operand(uint8_t* op_hi, const float* __restrict__ src,
                                              const float2* __restrict__ cs, int t) {
#pragma unroll
  for (int task = t; task < ROWS * 8; task += SM_THREADS) {  // all loads issued together
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

__global__ void __launch_bounds__(THREADS, 1)
    sel_sums_kernel(const __grid_constant__ CUtensorMap tm_k, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* slots = smem;
  uint8_t* opnd = slots + NSLOT * TILE_BYTES;
  float* bins = reinterpret_cast<float*>(opnd + NOPND * QOP);
  float* vbin = bins;            // [SLICE]
  float* sbin = bins + SLICE;    // [SBINS]
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

  if (warp == 0) {
    // work list of the slice; continuous: per k-tile (one lane each) the
    // chunks its causal keys meet, summed over the warp
    int n = 0;
    if (p.continuous) {
      int64_t kend = ka + SLICE;
      if (kend > i_last + 1) kend = i_last + 1;
      if (kend > p.Lk) kend = p.Lk;
      const uint32_t s32 = static_cast<uint32_t>(p.s);
      const int64_t t0 = ka + static_cast<int64_t>(lane) * BN;
      if (lane < SLICE / BN && t0 < kend) {
        const int64_t t1 = (t0 + BN < kend ? t0 + BN : kend) - 1;
        n = static_cast<int>(static_cast<uint32_t>(t1) / s32 - static_cast<uint32_t>(t0) / s32 + 1);
      }
      n = __reduce_add_sync(0xffffffffu, n);
      if (lane == 0) {
        ctl->kend = kend;
        ctl->kt0 = static_cast<int>(ka / BN);
        ctl->c_first = kend > ka ? ka / p.s : 0;
        ctl->c_last = kend > ka ? (kend - 1) / p.s : 0;
      }
    } else if (lane == 0) {
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
    if (lane == 0) {
      for (int k = 0; k < NSLOT_MAX; ++k) {
        mbar_init(&ctl->slot_full[k], 1);
        mbar_init(&ctl->slot_empty[k], 1);
      }
      for (int k = 0; k < NSBUF; ++k) {
        mbar_init(&ctl->s_full[k], 1);
        mbar_init(&ctl->s_free[k], SM_WARPS);
      }
      for (int k = 0; k < 2; ++k) mbar_init(&ctl->op_full[k], SM_WARPS);
      mbar_init(&ctl->drain, 1);
      ctl->abort = 0;
      ctl->n_items = n;
      ctl->rot = (n == 0 || (p.continuous && ctl->c_first != ctl->c_last)) ? 0 : (hh * n) / p.G;
      fence_barrier_init();
    }
  }
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

  if (warp < SM_WARPS) {
    // =========================================================== softmax warps
    // warp w: keys 32 (w % 4) + lane of each tile (its TMEM lane quarter) and
    // rows r0 = 32 (w / 4) .. r0 + 31 of the estimate; two warps per SMSP
    const int kq = warp & 3, r0 = (warp >> 2) * 32;
    const int tau = kq * 32 + lane;  // key within the tile
    const int stid = threadIdx.x;    // 0 .. 255
    const uint32_t lane_off = static_cast<uint32_t>(kq * 32) << 16;
    const float* qh = p.qv + static_cast<int64_t>(h) * (p.continuous ? 1 : 3) * ROWS * HD;
    if (N > 0) {
      if (p.continuous) {
        build_operand(opnd, qh, p.crot + ctl->c_first * (HD / 2), stid);
        if (ctl->c_first + 1 <= ctl->c_last)
          build_operand(opnd + 2 * QOP, qh, p.crot + (ctl->c_first + 1) * (HD / 2), stid);
      } else {
        for (int v = 0; v < 3; ++v)
          build_operand(opnd + 2 * v * QOP, qh + v * ROWS * HD, nullptr, stid);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ctl->op_full[0]);
        if (p.continuous && ctl->c_first + 1 <= ctl->c_last) mbar_arrive(&ctl->op_full[1]);
      }
    }

    // C_r = M_r + log2 L_r, so p = 2^(x - C_r)
    float C[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float2 st = p.stats[h * ROWS + r0 + e];
      C[e] = st.y > 0.f ? st.x + __log2f(st.y) : 0.f;
    }
    Cursor it = first_item(ctl, p);
    for (int n = 0; n < N; ++n) {
      const int buf = n % NSBUF;
      if (!sel_sm_wait(&ctl->s_full[buf], static_cast<uint32_t>((n / NSBUF) & 1), abort_flag,
                     p.status, p.timeout_ns, ST_SOFTMAX, lane))
        break;
      tc_fence_after();
      uint32_t sv[32];
      tmem_ld32(tbase + lane_off + static_cast<uint32_t>(buf * ROWS + r0), sv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->s_free[buf]);

      const int64_t j = static_cast<int64_t>(it.kt) * BN + tau;
      int ra, rb;
      class_row_range(j, p.i_first, p.n_last, p.Lk, p.s, p.w, p.reading,
                      p.continuous ? -1 : it.v, p.continuous ? it.c : -1, &ra, &rb);
      // every row of the warp valid in every lane: no masks (the common case)
      const bool full = __all_sync(0xffffffffu, ra <= r0 && rb >= r0 + 32);
      float vsum = 0.f;
      // slash: the warp's 32 keys and 32 rows meet the diagonals d = r - t
      // (t = lane of the key); lane L owns d = r0 + L - 32 (a0) and r0 + L
      // (a1).  At local row e the value p(r0 + e, (e - L) mod 32) is on one of
      // them: a1 when L <= e.
      float a0 = 0.f, a1 = 0.f;
      auto rows = [&](auto masked) {
        constexpr bool MASKED = decltype(masked)::value;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int r = r0 + e;
          float pr = ex2_approx(__uint_as_float(sv[e]) - C[e]);
          if (MASKED) pr = (r >= ra && r < rb) ? pr : 0.f;
          vsum += pr;
          // source lane (e - L) mod 32: the shuffle takes the index mod 32
          const float v = __shfl_sync(0xffffffffu, pr, e - lane);
          if (lane <= e) a1 += v; else a0 += v;
        }
      };
      // one version per case, so no branch sits between the rows
      if (full)
        rows(std::false_type{});
      else
        rows(std::true_type{});
      atomicAdd(&vbin[j - ka], vsum);  // the two row halves of key j
      // bin of diagonal d: offset i - j minus the slice's smallest offset,
      // (ka + SLICE - 1 - j_t) + r = (ka + SLICE - 1 - j_0) + d
      float* bw = sbin + (ka + SLICE - 1 - (static_cast<int64_t>(it.kt) * BN + kq * 32)) + r0;
      if (lane > 0) atomicAdd(&bw[lane - 32], a0);
      atomicAdd(&bw[lane], a1);

      // continuous: the last item of chunk c frees its operand buffer for c + 2
      if (p.continuous) {
        const int64_t c = it.c;
        next_item(ctl, p, it);
        if ((n + 1 == N || it.c != c) && c + 2 <= ctl->c_last) {
          build_operand(opnd + 2 * static_cast<int>((c - ctl->c_first) & 1) * QOP, qh,
                        p.crot + (c + 2) * (HD / 2), stid);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->op_full[(c - ctl->c_first) & 1]);
        }
      } else {
        next_item(ctl, p, it);
      }
    }

    // ---- per-CTA results (every softmax warp runs this, whatever happened)
    {
      softmax_bar();  // every bin update is done
      float* vrow = p.vert + static_cast<int64_t>(h) * p.Lk;
      float* srow = p.slash + static_cast<int64_t>(h) * p.Lk;
      for (int e = stid; e < SLICE; e += SM_THREADS) {
        const int64_t jj = ka + e;
        if (jj < p.Lk) vrow[jj] = vbin[e];
      }
      const int64_t o0 = p.i_first - (ka + SLICE - 1);
      for (int e = stid; e < SBINS; e += SM_THREADS) {
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
          ok = sel_mma_wait(&ctl->op_full[ci & 1], static_cast<uint32_t>((ci >> 1) & 1), abort_flag,
                         p.status, p.timeout_ns, ST_MMA);
          if (!ok) break;
          have = need;
        }
        ok = sel_mma_wait(&ctl->slot_full[slot], static_cast<uint32_t>((n / nslot) & 1), abort_flag,
                       p.status, p.timeout_ns, ST_MMA);
        if (!ok) break;
        if (n >= NSBUF) {
          ok = sel_mma_wait(&ctl->s_free[n % NSBUF], static_cast<uint32_t>(((n - NSBUF) / NSBUF) & 1),
                         abort_flag, p.status, p.timeout_ns, ST_MMA);
          if (!ok) break;
        }
        tc_fence_after();
        const int op = p.continuous ? 2 * (it.v & 1) : 2 * it.v;
        const uint64_t dk = dk0 + static_cast<uint64_t>((slot_at(slot) - slots) >> 4);
        const uint32_t d_tmem = tbase + static_cast<uint32_t>((n % NSBUF) * ROWS);
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
        mma_commit(&ctl->s_full[n % NSBUF]);
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


// ---------------------------------------------------------------------------
// Pass 1 with the estimate rows as the MMA M.  The row statistics need, per
// row, only a running (max, sum) over the keys, which is one register pair
// when the thread owns the row: S = Q K'^T with M = 128 rows -- the 64
// estimate rows of two heads of a KV group -- and N = 128 keys, so each key
// tile serves two heads and each softmax thread keeps its row's statistics
// the way the attention kernels do.  The query operand (bf16 hi + lo of the
// fp32 rows, in log2 units) sits in TMEM as the MMA A operand; shared memory
// holds a 6-slot key-tile ring; three S buffers let the MMA run two items
// ahead.  The operand is rewritten where the item's variant (DCA: the pair
// class; continuous: the key chunk) changes, after the last S that read it
// has completed.  Warps: 0-3 softmax (thread = row = TMEM lane), 4 TMA
// producer (no multicast), 5 MMA issuer.  One CTA = (KV group, pair of its
// heads, slice of 16384 keys); its (max, sum) per row goes to the slice's
// entry of `part`, which sel_stats_kernel merges.
constexpr int R_ROWS = 128;               // two heads x 64 estimate rows
constexpr int R_SLICE = 16384;            // keys per CTA
constexpr int R_NSLOT = 6;                // key-tile ring
constexpr int R_NSB = 3;                  // S buffers in TMEM
constexpr uint32_t R_COL_QHI = R_NSB * 128, R_COL_QLO = R_COL_QHI + 64;
constexpr int R_THREADS = 192;
constexpr int R_WARP_LOAD = 4, R_WARP_MMA = 5;
constexpr float R_RESCALE_LOG2 = 8.0f;    // the running max moves only when it grows by more

struct RowCtl {
  uint64_t slot_full[R_NSLOT];
  uint64_t slot_empty[R_NSLOT];
  uint64_t s_full[R_NSB];
  uint64_t s_free[R_NSB];
  uint64_t q_ready;         // the operand of the next variant is written (one arrival per warp)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int n_items;
  int rot;                  // 0: items in list order
  int lo[3], hi[3];         // DCA: k-tile range per class, clipped to the slice
  int kt0;                  // continuous: first k-tile of the slice
  int64_t kend;             // continuous: end of the slice's causal keys
  int64_t c_first, c_last;  // continuous: key chunks met
};

constexpr size_t R_SMEM_BYTES = 1024 + R_NSLOT * TILE_BYTES + sizeof(RowCtl);
static_assert(R_SMEM_BYTES <= 232448, "shared memory budget");

struct RowParams {
  const float* qv;          // [Hq][nvar][ROWS][HD] rotated query rows, log2 units
  const float2* crot;       // continuous: (cos, sin) of s*n*theta_k [n_chunks][64]
  float2* part;             // out: [Hq][n_slices][ROWS] (max, sum)
  int64_t i_first, Lk, s, w;
  int n_last, Hq, Hkv, G, n_pairs, n_slices, reading, continuous;
  unsigned int* status;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ int64_t item_variant(const RowParams& p, const Cursor& it) {
  return p.continuous ? it.c : static_cast<int64_t>(it.v);
}

__global__ void __launch_bounds__(R_THREADS, 1)
    sel_rows_kernel(const __grid_constant__ CUtensorMap tm_k, const RowParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* slots = smem;
  RowCtl* ctl = reinterpret_cast<RowCtl*>(slots + R_NSLOT * TILE_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the head pairs of one KV group and slice are adjacent: they read the same keys
  const int hp = static_cast<int>(blockIdx.x) % p.n_pairs;
  const int rest = static_cast<int>(blockIdx.x) / p.n_pairs;
  const int sl = rest % p.n_slices;
  const int g = rest / p.n_slices;
  const int64_t ka = static_cast<int64_t>(sl) * R_SLICE;
  const int64_t i_last = p.i_first + p.n_last - 1;

  if (warp == 0) {
    // work list of the slice; continuous: per k-tile the chunks its causal
    // keys meet, counted by the lanes and summed over the warp
    int n = 0;
    if (p.continuous) {
      int64_t kend = ka + R_SLICE;
      if (kend > i_last + 1) kend = i_last + 1;
      if (kend > p.Lk) kend = p.Lk;
      const uint32_t s32 = static_cast<uint32_t>(p.s);
      for (int t = lane; t < R_SLICE / BN; t += 32) {
        const int64_t t0 = ka + static_cast<int64_t>(t) * BN;
        if (t0 < kend) {
          const int64_t t1 = (t0 + BN < kend ? t0 + BN : kend) - 1;
          n += static_cast<int>(static_cast<uint32_t>(t1) / s32 - static_cast<uint32_t>(t0) / s32 + 1);
        }
      }
      n = __reduce_add_sync(0xffffffffu, n);
      if (lane == 0) {
        ctl->kend = kend;
        ctl->kt0 = static_cast<int>(ka / BN);
        ctl->c_first = kend > ka ? ka / p.s : 0;
        ctl->c_last = kend > ka ? (kend - 1) / p.s : 0;
      }
    } else if (lane == 0) {
      const TilePlan P = make_plan(p.i_first, i_last, p.s, p.w, BN, p.reading);
      const int t0 = static_cast<int>(ka / BN), t1 = static_cast<int>((ka + R_SLICE) / BN);
      for (int c = 0; c < 3; ++c) {
        const int a = P.lo[c] > t0 ? P.lo[c] : t0;
        int b = P.hi[c] < t1 ? P.hi[c] : t1;
        if (b < a) b = a;
        ctl->lo[c] = a;
        ctl->hi[c] = b;
        n += b - a;
      }
    }
    if (lane == 0) {
      for (int k = 0; k < R_NSLOT; ++k) {
        mbar_init(&ctl->slot_full[k], 1);
        mbar_init(&ctl->slot_empty[k], 1);
      }
      for (int k = 0; k < R_NSB; ++k) {
        mbar_init(&ctl->s_full[k], 1);
        mbar_init(&ctl->s_free[k], 4);
      }
      mbar_init(&ctl->q_ready, 4);
      mbar_init(&ctl->drain, 1);
      ctl->abort = 0;
      ctl->n_items = n;
      ctl->rot = 0;
      fence_barrier_init();
    }
  }
  if (warp == R_WARP_MMA) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == R_WARP_LOAD && lane == 0) tma_prefetch_desc(&tm_k);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = ctl->tmem_base;
  volatile int* abort_flag = &ctl->abort;
  const int N = ctl->n_items;

  if (warp < 4) {
    // =========================================================== softmax warps
    const int r = warp * 32 + lane;  // TMEM lane = row of the MMA
    const int hh = r >> 6, rr = r & 63;
    const bool head_ok = 2 * hp + hh < p.G;
    const int h = g * p.G + (head_ok ? 2 * hp + hh : 0);
    const bool row_ok = head_ok && rr < p.n_last;
    const int64_t i = p.i_first + rr;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int nvar = p.continuous ? 1 : 3;
    // the row's operand for the item's variant: hi and lo bf16 parts, column
    // c holding dims 2c, 2c + 1; continuous: rotated back by the chunk angle
    auto write_q = [&](const Cursor& c) {
      uint32_t qh[64], ql[64];
#pragma unroll
      for (int e = 0; e < 64; ++e) qh[e] = ql[e] = 0u;
      if (row_ok) {
        const int v = p.continuous ? 0 : c.v;
        const float* src = p.qv + ((static_cast<int64_t>(h) * nvar + v) * ROWS + rr) * HD;
        const float2* cs = p.continuous ? p.crot + c.c * (HD / 2) : nullptr;
#pragma unroll
        for (int k = 0; k < HD / 2; k += 2) {
          float a0 = src[k], a1 = src[k + 1], b0 = src[HD / 2 + k], b1 = src[HD / 2 + k + 1];
          if (cs != nullptr) {  // R(-phi): (a cos + b sin, b cos - a sin)
            const float2 t0 = cs[k], t1 = cs[k + 1];
            const float ra0 = a0 * t0.x + b0 * t0.y, rb0 = b0 * t0.x - a0 * t0.y;
            const float ra1 = a1 * t1.x + b1 * t1.y, rb1 = b1 * t1.x - a1 * t1.y;
            a0 = ra0; b0 = rb0; a1 = ra1; b1 = rb1;
          }
          split_pack(a0, a1, qh[k / 2], ql[k / 2]);
          split_pack(b0, b1, qh[32 + k / 2], ql[32 + k / 2]);
        }
      }
      tmem_st64(tbase + lane_off + R_COL_QHI, qh);
      tmem_st64(tbase + lane_off + R_COL_QLO, ql);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->q_ready);
    };

    float m_ref = NEG_BIG, l_sum = 0.f;
    Cursor it = first_item(ctl, p);
    if (N > 0) write_q(it);
    for (int n = 0; n < N; ++n) {
      const int buf = n % R_NSB;
      if (!sel_sm_wait(&ctl->s_full[buf], static_cast<uint32_t>((n / R_NSB) & 1), abort_flag,
                     p.status, p.timeout_ns, ST_SOFTMAX, lane))
        break;
      tc_fence_after();
      // S(n) has completed, and with it every S that read this operand: where
      // the next item has another variant, rewrite the operand now
      Cursor nx = it;
      if (n + 1 < N) {
        next_item(ctl, p, nx);
        if (item_variant(p, nx) != item_variant(p, it)) write_q(nx);
      }
      uint32_t sv[128];
      tmem_ld128(tbase + lane_off + static_cast<uint32_t>(buf * 128), sv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->s_free[buf]);
      // the row's keys of this item: its class (or chunk), causal, j < Lk
      int64_t lo = 0, hi = 0;
      if (row_ok) {
        if (p.continuous) {
          lo = it.c * p.s;
          hi = lo + p.s < i + 1 ? lo + p.s : i + 1;
        } else {
          row_key_range<int64_t>(i, it.v, p.s, p.w, p.reading, lo, hi);
        }
        if (hi > p.Lk) hi = p.Lk;
      }
      const int64_t j0 = static_cast<int64_t>(it.kt) * BN;
      const int ea = lo - j0 < 0 ? 0 : (lo - j0 > BN ? BN : static_cast<int>(lo - j0));
      const int eb = hi - j0 < ea ? ea : (hi - j0 > BN ? BN : static_cast<int>(hi - j0));
      if (ea > 0 || eb < BN) {
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (e < ea || e >= eb) sv[e] = 0xff800000u;  // -inf
      }
      float m8[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) m8[c] = __uint_as_float(sv[c]);
#pragma unroll
      for (int e = 8; e < BN; e += 8)
#pragma unroll
        for (int c = 0; c < 8; ++c) m8[c] = fmaxf(m8[c], __uint_as_float(sv[e + c]));
      const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      if (mx > m_ref + R_RESCALE_LOG2) {  // m_ref = NEG_BIG: l_sum is 0 and stays 0
        l_sum *= ex2_approx(m_ref - mx);
        m_ref = mx;
      }
      it = nx;
      if (mx == -INFINITY) continue;  // no key of the row in this item
      // 2^(x - m_ref) <= 2^8; one pair in eight on the FMA pipe
      const float2 nm = make_float2(-m_ref, -m_ref);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
      for (int e = 0; e < BN / 2; ++e) {
        float2 x = add2(make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), nm);
        if ((e & 7) == 0) {
          x.x = attn::exp2_poly1(x.x);
          x.y = attn::exp2_poly1(x.y);
        } else {
          x.x = ex2_approx(x.x);
          x.y = ex2_approx(x.y);
        }
        acc[e & 3] = add2(acc[e & 3], x);
      }
      const float2 a = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
      l_sum += a.x + a.y;
    }
    if (head_ok)
      p.part[(static_cast<int64_t>(h) * p.n_slices + sl) * ROWS + rr] = make_float2(m_ref, l_sum);
  } else if (warp == R_WARP_LOAD) {
    // =========================================================== TMA producer
    if (lane == 0) {
      int last[R_NSLOT];
#pragma unroll
      for (int k = 0; k < R_NSLOT; ++k) last[k] = -1;
      Cursor it = first_item(ctl, p);
      for (int n = 0; n < N; ++n) {
        const int slot = n % R_NSLOT, use = n / R_NSLOT;
        if (use > 0 &&
            !wait_bounded(&ctl->slot_empty[slot], static_cast<uint32_t>((use - 1) & 1),
                          abort_flag, p.status, p.timeout_ns, ST_LOAD))
          break;
        uint8_t* dst = slots + slot * TILE_BYTES;
        mbar_arrive_expect_tx(&ctl->slot_full[slot], TILE_BYTES);
        tma_load_3d(dst, &tm_k, &ctl->slot_full[slot], 0, g, it.kt * BN);
        tma_load_3d(dst + HALF_BYTES, &tm_k, &ctl->slot_full[slot], 64, g, it.kt * BN);
        last[slot] = n;
        next_item(ctl, p, it);
      }
      for (int k = 0; k < R_NSLOT; ++k)
        if (last[k] >= 0)
          wait_drain(&ctl->slot_full[k], static_cast<uint32_t>((last[k] / R_NSLOT) & 1), p.status,
                     p.timeout_ns, ST_DRAIN);
    }
    __syncwarp();
  } else if (warp == R_WARP_MMA) {
    // =========================================================== MMA issuer
    if (lane == 0) {
      const uint32_t id = idesc_bf16_f32(R_ROWS, BN, false);
      const uint64_t dk0 = sdesc_sw128(smem_u32(slots), 16, 1024);
      bool ok = true;
      Cursor it = first_item(ctl, p);
      int64_t have = -1;  // the variant whose operand is known to be written
      uint32_t qph = 0;   // operand writes waited for
      for (int n = 0; n < N && ok; ++n) {
        const int64_t var = item_variant(p, it);
        if (n == 0 || var != have) {
          ok = sel_mma_wait(&ctl->q_ready, qph & 1u, abort_flag, p.status, p.timeout_ns, ST_MMA);
          if (!ok) break;
          ++qph;
          have = var;
        }
        if (n >= R_NSB) {
          ok = sel_mma_wait(&ctl->s_free[n % R_NSB], static_cast<uint32_t>(((n - R_NSB) / R_NSB) & 1),
                         abort_flag, p.status, p.timeout_ns, ST_MMA);
          if (!ok) break;
        }
        const int slot = n % R_NSLOT;
        ok = sel_mma_wait(&ctl->slot_full[slot], static_cast<uint32_t>((n / R_NSLOT) & 1), abort_flag,
                       p.status, p.timeout_ns, ST_MMA);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dk = dk0 + static_cast<uint64_t>((slot * TILE_BYTES) >> 4);
        const uint32_t d_tmem = tbase + static_cast<uint32_t>((n % R_NSB) * 128);
#pragma unroll
        for (int part = 0; part < 2; ++part) {  // hi, then lo
          const uint32_t tq = tbase + (part ? R_COL_QLO : R_COL_QHI);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4);
            mma_ts(d_tmem, tq + static_cast<uint32_t>(kk * 8), dk + off, id,
                   (part > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(&ctl->s_full[n % R_NSB]);
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
  if (warp == R_WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace selm

int select_slices(int64_t Lk) { return static_cast<int>((Lk + selm::SLICE - 1) / selm::SLICE); }

int select_stat_slices(int64_t Lk) {
  return static_cast<int>((Lk + selm::R_SLICE - 1) / selm::R_SLICE);
}

cudaError_t launch_select_sums(const void* kr, const float* qv, const float2* crot,
                               const float2* stats, float* vert, float* slash, int64_t i_first,
                               int64_t Lk, int64_t s, int64_t w, int n_last, int Hq, int Hkv,
                               int reading, int continuous, unsigned int* status,
                               unsigned long long timeout_ns, cudaStream_t st) {
  using namespace selm;
  CUtensorMap tm_k;
  if (!encode_kv_map(&tm_k, kr, Lk, Hkv)) return cudaErrorInvalidValue;
  Params p;
  p.qv = qv;
  p.crot = crot;
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
  cudaError_t e = cudaFuncSetAttribute(sel_sums_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  sel_sums_kernel<<<static_cast<unsigned>(blocks), THREADS, SMEM_BYTES, st>>>(tm_k, p);
  return cudaGetLastError();
}

cudaError_t launch_select_row_stats(const void* kr, const float* qv, const float2* crot,
                                    float2* part, int64_t i_first, int64_t Lk, int64_t s, int64_t w,
                                    int n_last, int Hq, int Hkv, int reading, int continuous,
                                    unsigned int* status, unsigned long long timeout_ns,
                                    cudaStream_t st) {
  using namespace selm;
  CUtensorMap tm_k;
  if (!encode_kv_map(&tm_k, kr, Lk, Hkv)) return cudaErrorInvalidValue;
  RowParams p;
  p.qv = qv;
  p.crot = crot;
  p.part = part;
  p.i_first = i_first;
  p.Lk = Lk;
  p.s = s;
  p.w = w;
  p.n_last = n_last;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_pairs = (p.G + 1) / 2;
  p.n_slices = select_stat_slices(Lk);
  p.reading = reading;
  p.continuous = continuous;
  p.status = status;
  p.timeout_ns = timeout_ns;
  const int64_t blocks = static_cast<int64_t>(Hkv) * p.n_slices * p.n_pairs;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(sel_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(R_SMEM_BYTES));
  if (e != cudaSuccess) return e;
  sel_rows_kernel<<<static_cast<unsigned>(blocks), R_THREADS, R_SMEM_BYTES, st>>>(tm_k, p);
  return cudaGetLastError();
}

}  // namespace dca
