// dca_fwd_sm100.cu -- fused Dual Chunk Attention forward for sm_100a.
//
// One CTA computes two (query tile, query head) units that read the same KV
// head (GQA: the K/V tiles it streams are shared by both): two heads of one
// KV group on the same 128-row query tile, or -- for the last head of a group
// of odd size -- that head on two consecutive query tiles, whose key tiles
// are then visited in ascending order (the shorter tile's list is a prefix of
// the longer one's).  Warp roles (320 threads):
//   warps 0-3  softmax of unit A: one query row per thread (TMEM lane), all
//              128 keys of the row, so no exchange between threads
//   warps 4-7  softmax of unit B; an A warp and a B warp share each SM
//              sub-partition, so one unit's exponentials run while the tensor
//              cores run the other unit's MMAs (ping-pong)
//   warp  8    TMA producer: K'/V tiles (128 keys x 128 dims, bf16, 128-byte
//              swizzle) into a ring of shared-memory slots (no multicast)
//   warp  9    MMA issuer (one thread): S = Q K'^T and O += P V with
//              tcgen05.mma kind::f16 (bf16 in, fp32 accumulate in TMEM)
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512);
// P (bf16) overwrites the first 64 columns of its S and is the TMEM A operand
// of the P.V MMA.  MMA order per item: P.V(A), S(A, next), P.V(B), S(B, next);
// MMAs of one thread execute in order, so S(next) never overwrites P before
// P.V has read it.
//
// DCA ("Qwen2.5-1M 不重训外推 1M", sections 核心思想 / Intra / Successive /
// Inter-Chunk Attention): keys arrive pre-rotated by j mod s; each query row is
// rotated in-kernel by the position of the current phase (INTER: c-1, SUCC:
// s + r_i or c-1 outside the local window, INTRA: r_i).  The work list visits
// INTER k-tiles, then SUCC, then INTRA (dca_plan.cuh), so the softmax threads
// rewrite their Q row only twice per tile.  Tiles wholly inside one class and
// below the diagonal run unmasked; others are masked per element.
// YaRN temperature: logits * m^2/sqrt(d), folded into the exp2 argument.
//
// Online softmax: the row's reference max is updated (and O, l rescaled) only
// when the max grows by more than 2^8; the final O / l uses the same reference.
// A share of the exponentials runs on the FMA pipe (exp2_poly1) to relieve the
// MUFU pipe, which at d = 128 needs as many SM cycles per score as the tensor
// cores.
//
// Every wait is bounded (globaltimer); on timeout the CTA raises a shared
// abort flag, ORs a code into the device status word, drains its own TMA
// copies and MMAs, frees TMEM and exits.
#include <cuda_bf16.h>
#include <math.h>

#include <mutex>

#include "dca_internal.h"
#include "dca_plan.cuh"
#include "dca_softmax.cuh"
#include "sm100_ptx.cuh"

namespace dca {
namespace sm100 {

using namespace attn;

constexpr int BM = 128;            // query rows per tile
constexpr int BN = 128;            // keys per tile
constexpr int HD = 128;            // head dim
#ifndef DCA_NSLOT
#define DCA_NSLOT 5
#endif
constexpr int NSLOT = DCA_NSLOT;   // K/V ring slots
constexpr int TILE_BYTES = 32768;  // 128 x 128 bf16
// 10 warps: 8 softmax (warps 0-3 unit A, 4-7 unit B; one query row per
// thread), TMA producer, MMA issuer.
constexpr int NUM_THREADS = 320;
constexpr int WARP_LOAD = 8;
constexpr int WARP_MMA = 9;
constexpr float RESCALE_LOG2 = 8.0f;
// How the softmax threads wait for S: polling (no suspension; a suspended
// thread wakes up hundreds of cycles after the phase completes), optionally
// with a short back-off so that the waiting unit's warps leave issue slots to
// the other unit's warps of the same sub-partition.
#ifndef DCA_S_WAIT
#define DCA_S_WAIT wait_poll
#endif
// How the MMA issuer waits: polling (wait_poll) or polling with a short
// back-off (wait_spin).  Its waits sit outside the MMA bursts where they can:
// a poll between two groups of MMAs leaves the tensor pipe idle for ~160
// cycles (measured on B200), so a unit's P.V and next S go out back to back.
#ifndef DCA_MMA_WAIT
#define DCA_MMA_WAIT wait_poll
#endif

// Of every 8 score pairs of a row, this many take the software exp2 (the
// rest the MUFU ex2); measured best at 1 (12.5%) with one row per thread.
#ifndef DCA_FWD_POLY_PAIRS
#define DCA_FWD_POLY_PAIRS 1
#endif

// status codes (bits) for timeouts, by role
constexpr unsigned ST_SOFTMAX = 0x10u, ST_LOAD = 0x100u, ST_MMA = 0x1000u, ST_DRAIN = 0x10000u;

struct SmemCtl {
  uint64_t slot_full[NSLOT];
  uint64_t slot_empty[NSLOT];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t q_ready[2];
  uint64_t o_final[2];
  uint64_t drain;
  uint64_t p_half[2];  // P of keys 0..63 of the unit's current item stored
  uint32_t tmem_base;
  int abort;
  // each unit's work list and unmasked k-tile ranges, read per item from here
  // rather than held in registers next to the 128 scores of a row
  TilePlan plan[2];
  FullRanges full[2];
};

constexpr size_t SMEM_BYTES = 1024 + 2 * TILE_BYTES + NSLOT * TILE_BYTES + sizeof(SmemCtl);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

struct Params {
  const __nv_bfloat16* q;
  __nv_bfloat16* out;
  const float2* tab;
  int64_t q_start, Lq, Lk;
  int64_t s, w, tab_c1;
  int Hq, Hkv, G, n_two, n_lone, n_qtiles;
  int lone_pairs;  // the lone head of a group runs on two consecutive q-tiles per CTA
  int reading;     // READING_A or READING_B
  float scale_log2;
  unsigned int* status;
  unsigned long long timeout_ns;
  int debug;
};

// The two units of a CTA.  Unit u covers query tile qt[u] of head h[u]; the
// work list of the CTA is that of unit B (the longer), unit A's is a prefix.
struct Units {
  int g;         // KV head
  int qt[2];
  int h[2];
  bool two;      // unit B exists
};

// CTA -> units.  KV-group-major order: the CTAs running together stream the
// same group's K'/V tiles (shared in L2).  Within a group the CTAs with two
// heads on one q-tile come first, then those of the group's last head (odd
// G); within each set the longest query tiles go first, so CTAs with equal
// work run side by side and stay in step along the key stream.
__device__ __forceinline__ Units decode_units(const Params& p) {
  Units u;
  const int per_group = p.n_qtiles * p.n_two + p.n_lone;
  u.g = static_cast<int>(blockIdx.x) / per_group;
  const int c = static_cast<int>(blockIdx.x) % per_group;
  if (c < p.n_qtiles * p.n_two) {
    const int qt = p.n_qtiles - 1 - c / p.n_two;
    const int pr = c % p.n_two;
    u.qt[0] = u.qt[1] = qt;
    u.h[0] = u.g * p.G + 2 * pr;
    u.h[1] = u.h[0] + 1;
    u.two = true;
  } else {
    const int lc = c - p.n_qtiles * p.n_two;
    u.h[0] = u.h[1] = u.g * p.G + p.G - 1;
    if (p.lone_pairs) {
      u.qt[1] = p.n_qtiles - 1 - 2 * lc;
      u.qt[0] = u.qt[1] - 1;
      u.two = u.qt[0] >= 0;
      if (!u.two) u.qt[0] = u.qt[1];
    } else {
      u.qt[0] = u.qt[1] = p.n_qtiles - 1 - lc;
      u.two = false;
    }
    if (!u.two) {  // a lone unit is unit A (warps 0-3), B idles
      u.qt[1] = u.qt[0];
    }
  }
  return u;
}

// plan_item / is_full on a work list kept in shared memory.
__device__ __forceinline__ void plan_item_v(const volatile TilePlan& P, int n, int& kt, int& cls) {
  const int c2 = P.hi[CLS_INTER] - P.lo[CLS_INTER];
  const int c1 = P.hi[CLS_SUCC] - P.lo[CLS_SUCC];
  if (n < c2) {
    cls = CLS_INTER;
    kt = P.lo[CLS_INTER] + n;
  } else if (n < c2 + c1) {
    cls = CLS_SUCC;
    kt = P.lo[CLS_SUCC] + (n - c2);
  } else {
    cls = CLS_INTRA;
    kt = P.lo[CLS_INTRA] + (n - c2 - c1);
  }
}
__device__ __forceinline__ bool is_full_v(const volatile FullRanges& F, int kt, int cls) {
  return kt >= F.lo[cls] && kt < F.hi[cls];
}

// Maximum of 128 scores: eight independent chains of three-input maxima.
__device__ __forceinline__ float max128(const uint32_t* sv) {
  float m8[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) m8[c] = __uint_as_float(sv[c]);
#pragma unroll
  for (int e = 8; e < 128; e += 16) {
#pragma unroll
    for (int c = 0; c < 8; ++c)
      m8[c] = max3f(m8[c], __uint_as_float(sv[e + c]),
                    e + 8 + c < 128 ? __uint_as_float(sv[e + 8 + c]) : m8[c]);
  }
  return max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
}

// Exponentials of 16 scores against the reference `mb` (= m_ref * sc): P
// (bf16 pairs) into pk[8], their sum added to acc0 / acc1.
__device__ __forceinline__ void exp_pack16(const uint32_t* sv, float2 sc2, float2 nmb2,
                                           uint32_t* pk, float2& acc0, float2& acc1) {
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    float2 x = fma2(make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), sc2,
                    nmb2);
    if (e < DCA_FWD_POLY_PAIRS) {
      x.x = exp2_poly1(x.x);
      x.y = exp2_poly1(x.y);
    } else {
      x.x = ex2_approx(x.x);
      x.y = ex2_approx(x.y);
    }
    if (e & 1)
      acc1 = add2(acc1, x);
    else
      acc0 = add2(acc0, x);
    pk[e] = pack_bf16(x.x, x.y);
  }
}

// One online-softmax step of a full query row (this thread's TMEM lane):
// scores in columns tS..tS+127, P (bf16) written to columns tS..tS+63 (all
// scores are in registers before the first store), partial row sum kept in
// l_sum; O (columns tO..tO+127) rescaled when the row maximum moved more than
// 2^RESCALE_LOG2 above the reference (otherwise P may reach 2^8, exact in
// fp32 and in bf16's exponent range; the final O / l uses the same
// reference).  O holds items < n: their MMAs completed before S(n) did (one
// commit tracks all earlier MMAs).
// `before_exp` / `after_exp` bracket the exponentials (the hand-over of the
// exponential units between the CTA's two units).
// Columns outside [ea, eb) are masked (the row's keys of the item's class
// within the tile; [0, 128) for an unmasked tile).
template <class HalfDone>
__device__ __forceinline__ void softmax_row_step(uint32_t tS, uint32_t tO, int n, int ea, int eb,
                                                 float sc, float& m_ref, float& l_sum,
                                                 HalfDone&& half_done) {
  uint32_t sv[128];
  tmem_ld128(tS, sv);
  if (ea > 0 || eb < 128) {
#pragma unroll
    for (int e = 0; e < 128; ++e)
      if (e < ea || e >= eb) sv[e] = 0xff800000u;  // -inf
  }
  const float mx = max128(sv);
  const float m_new = fmaxf(m_ref, mx);
  const bool need =
      (m_new > m_ref) && (m_ref == -INFINITY || (m_new - m_ref) * sc > RESCALE_LOG2);
  float alpha = 1.f;
  if (need) {
    alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx((m_ref - m_new) * sc);
    m_ref = m_new;
    l_sum *= alpha;
  }
  // TMEM access is warp-collective: rescale O when any row of the warp needs
  // it (rows whose max did not move use alpha = 1), before any P of this item
  // is handed to the P.V MMAs
  if (n > 0 && __any_sync(0xffffffffu, need)) {
    // in chunks of 16 columns: the 128 scores of the row are live here
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      uint32_t o[16];
      tmem_ld16(tO + 16u * c, o);
#pragma unroll
      for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
      tmem_st16(tO + 16u * c, o);
    }
    tmem_st_wait();
  }
  const float mb = (m_ref == -INFINITY) ? 0.f : m_ref * sc;
  const float2 sc2 = make_float2(sc, sc);
  const float2 nmb2 = make_float2(-mb, -mb);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t pk[8];
    exp_pack16(sv + 16 * c, sc2, nmb2, pk, acc0, acc1);
    tmem_st8(tS + 8u * c, pk);
    if (c == 3) {  // P of keys 0..63 stored: the first half of P.V may start
      tmem_st_wait();
      half_done();
    }
  }
  const float2 a = add2(acc0, acc1);
  l_sum += a.x + a.y;
  tmem_st_wait();
}

#ifndef DCA_FWD_BOUNDS
#define DCA_FWD_BOUNDS __launch_bounds__(NUM_THREADS, 1)
#endif
__global__ void DCA_FWD_BOUNDS
    dca_fwd_kernel(const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* q_bufs = smem;  // [2][TILE_BYTES]
  uint8_t* slots = smem + 2 * TILE_BYTES;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(slots + NSLOT * TILE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work units
  const Units U = decode_units(p);
  const int g = U.g;
  const bool two = U.two;
  const int64_t q_end = p.q_start + p.Lq;
  // the CTA's work list is unit B's (or A's alone); unit A's is a prefix of it
  const int64_t i0A = p.q_start + static_cast<int64_t>(U.qt[0]) * BM;
  const int64_t i0B = p.q_start + static_cast<int64_t>(U.qt[1]) * BM;
  const TilePlan wplan = make_plan(i0B, (i0B + BM - 1 < q_end - 1) ? i0B + BM - 1 : q_end - 1,
                                   p.s, p.w, BN, p.reading);
  const int N = wplan.n_items;
  // unit A's items: a prefix of the work list
  const int NA =
      two ? make_plan(i0A, (i0A + BM - 1 < q_end - 1) ? i0A + BM - 1 : q_end - 1, p.s, p.w, BN,
                      p.reading)
                .n_items
          : N;

  if (threadIdx.x == 0) {
    for (int k = 0; k < NSLOT; ++k) {
      mbar_init(&ctl->slot_full[k], 1);
      mbar_init(&ctl->slot_empty[k], 1);
    }
    for (int st = 0; st < 2; ++st) {
      mbar_init(&ctl->s_full[st], 1);
      mbar_init(&ctl->p_full[st], 4);   // one arrival per softmax warp of the unit
      mbar_init(&ctl->q_ready[st], 4);
      mbar_init(&ctl->o_final[st], 1);
    }
    mbar_init(&ctl->drain, 1);
    mbar_init(&ctl->p_half[0], 4);
    mbar_init(&ctl->p_half[1], 4);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == WARP_LOAD && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = ctl->tmem_base;
  volatile int* abort_flag = &ctl->abort;

  if (warp < 8) {
    // =========================================================== softmax
    const int st = warp >> 2;   // unit
    const int sub = warp & 3;   // TMEM lane quarter
    const int r = sub * 32 + lane;
    if (st == 0 || two) {
      const int64_t i0 = st ? i0B : i0A;
      const int64_t i_last = (i0 + BM - 1 < q_end - 1) ? i0 + BM - 1 : q_end - 1;
      if (sub == 0 && lane == 0) {
        ctl->plan[st] = make_plan(i0, i_last, p.s, p.w, BN, p.reading);
        ctl->full[st] = make_full_ranges(i0, i0 + BM - 1, p.s, p.w, BN, p.reading);
      }
      if (st) named_bar_sync(2, 128); else named_bar_sync(1, 128);  // the unit's four warps
      const volatile TilePlan& P = ctl->plan[st];
      const volatile FullRanges& fullr = ctl->full[st];
      const int Nst = P.n_items;
      const int head = st ? U.h[1] : U.h[0];
      // row arithmetic in 32 bits: i < Lk <= 2^31 - 1; s and w clamped (a chunk
      // longer than the cache is the same as one of 2^31 - 1 keys)
      const int i = static_cast<int>(i0) + r;
      const int s32 = p.s < 0x7fffffff ? static_cast<int>(p.s) : 0x7fffffff;
      const int w32 = p.w < 0x7fffffff ? static_cast<int>(p.w) : 0x7fffffff;
      const bool real = i <= i_last;
      const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
      const float sc = p.scale_log2;
      uint8_t* qb = q_bufs + st * TILE_BYTES;
      const uint32_t tS = tbase + lane_off + static_cast<uint32_t>(st * 128);
      const uint32_t tO = tbase + lane_off + 256u + static_cast<uint32_t>(st * 128);
      // rotate this row of the query by the position of class `c` into the operand tile
      auto rotate_q = [&](int c) {
        const __nv_bfloat16* qrow =
            real ? p.q + ((static_cast<int64_t>(i) - p.q_start) * p.Hq + head) *
                             static_cast<int64_t>(HD)
                 : nullptr;
        const float2* trow =
            real ? p.tab + query_table_row(static_cast<int64_t>(i), c, p.s, p.w, p.tab_c1) * 64
                 : nullptr;
        write_q_row(qb, r, qrow, trow);
        fence_proxy_async_smem();
      };

      int kt, cls;
      plan_item_v(P, 0, kt, cls);
      rotate_q(cls);
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->q_ready[st]);

      float m_ref = -INFINITY;
      float l_sum = 0.f;
      bool ok = true;
      for (int n = 0; n < Nst && ok; ++n) {
        plan_item_v(P, n, kt, cls);
        int ea = 0, eb = BN;
        if (!is_full_v(fullr, kt, cls)) {
          int lo, hi;
          row_key_range<int>(i, cls, s32, w32, p.reading, lo, hi);
          const int j0 = kt * BN;
          ea = lo - j0 < 0 ? 0 : (lo - j0 > BN ? BN : lo - j0);
          eb = hi - j0 < ea ? ea : (hi - j0 > BN ? BN : hi - j0);
        }
        int cls_next = cls;
        if (n + 1 < Nst) {
          int kt_next;
          plan_item_v(P, n + 1, kt_next, cls_next);
        }
        ok = DCA_S_WAIT(&ctl->s_full[st], static_cast<uint32_t>(n & 1), abort_flag, p.status,
                        p.timeout_ns, ST_SOFTMAX << st);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        auto half_done = [&]() {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->p_half[st]);
        };
        softmax_row_step(tS, tO, n, ea, eb, sc, m_ref, l_sum, half_done);
        if (cls_next != cls) rotate_q(cls_next);  // phase switch: another query rotation
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->p_full[st]);
      }
      // epilogue: O / l -> bf16 -> out (each thread writes its row, 256 bytes)
      if (ok) {
        ok = wait_bounded(&ctl->o_final[st], 0u, abort_flag, p.status, p.timeout_ns,
                          ST_SOFTMAX << st);
        ok = __all_sync(0xffffffffu, ok);
      }
      if (ok) {
        tc_fence_after();
        const float inv = 1.f / l_sum;
        __nv_bfloat16* orow =
            real ? p.out + ((static_cast<int64_t>(i) - p.q_start) * p.Hq + head) *
                               static_cast<int64_t>(HD)
                 : nullptr;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
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
    }
  } else if (warp == WARP_LOAD) {
    // =========================================================== TMA producer
    if (lane == 0) {
      int last_li[NSLOT];
#pragma unroll
      for (int k = 0; k < NSLOT; ++k) last_li[k] = -1;
      bool ok = true;
      for (int n = 0; n < N && ok; ++n) {
        int kt, cls;
        plan_item(wplan, n, kt, cls);
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
          const CUtensorMap* tm = which ? &tm_v : &tm_k;
          mbar_arrive_expect_tx(&ctl->slot_full[slot], TILE_BYTES);
          tma_load_3d(dst, tm, &ctl->slot_full[slot], 0, g, kt * BN);
          tma_load_3d(dst + HALF_BYTES, tm, &ctl->slot_full[slot], 64, g, kt * BN);
          last_li[slot] = li;
        }
      }
      // every copy this CTA started must land before the CTA exits
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
      const uint32_t slot_addr0 = smem_u32(slots);
      // Descriptors are built once; a k-step only adds its byte offset / 16 to
      // the start-address field (no carry out of the 14-bit field: shared
      // memory addresses stay below 256 KiB).
      const uint64_t dq0 = sdesc_sw128(smem_u32(q_bufs), 16, 1024);
      const uint64_t dq1 = sdesc_sw128(smem_u32(q_bufs + TILE_BYTES), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(slot_addr0, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(slot_addr0, HALF_BYTES, 1024);
      auto issue_s = [&](int st, int li) {
        const uint64_t dk = dk0 + static_cast<uint64_t>(((li % NSLOT) * TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4);
          mma_ss(tbase + static_cast<uint32_t>(st * 128), (st ? dq1 : dq0) + off, dk + off, id_s,
                 kk > 0 ? 1u : 0u);
        }
      };
      // P.V over keys 64*h .. 64*h + 63 (K steps 4h .. 4h + 3)
      auto issue_pv = [&](int st, int li, bool acc, int h) {
        const uint64_t dv = dv0 + static_cast<uint64_t>(((li % NSLOT) * TILE_BYTES) >> 4);
#pragma unroll
        for (int k4 = 0; k4 < BN / 32; ++k4) {
          const int kk = 4 * h + k4;
          mma_ts(tbase + 256u + static_cast<uint32_t>(st * 128),
                 tbase + static_cast<uint32_t>(st * 128 + kk * 8),
                 dv + static_cast<uint64_t>((kk * 2048) >> 4), id_o, (acc || kk > 0) ? 1u : 0u);
        }
      };
      // P.V of unit st: the first half once its P is stored, then the second
      auto pv_unit = [&](int st, int n, int lv) {
        bool w = DCA_MMA_WAIT(&ctl->p_half[st], static_cast<uint32_t>(n & 1), abort_flag,
                              p.status, p.timeout_ns, ST_MMA);
        if (!w) return false;
        tc_fence_after();
        issue_pv(st, lv, n > 0, 0);
        w = DCA_MMA_WAIT(&ctl->p_full[st], static_cast<uint32_t>(n & 1), abort_flag, p.status,
                         p.timeout_ns, ST_MMA);
        if (!w) return false;
        tc_fence_after();
        issue_pv(st, lv, true, 1);
        return true;
      };
      auto full_wait = [&](int li) {
        return DCA_MMA_WAIT(&ctl->slot_full[li % NSLOT], static_cast<uint32_t>((li / NSLOT) & 1),
                            abort_flag, p.status, p.timeout_ns, ST_MMA);
      };

      bool ok = wait_bounded(&ctl->q_ready[0], 0u, abort_flag, p.status, p.timeout_ns, ST_MMA);
      if (ok && two)
        ok = wait_bounded(&ctl->q_ready[1], 0u, abort_flag, p.status, p.timeout_ns, ST_MMA);
      if (ok) ok = full_wait(0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        mma_commit(&ctl->s_full[0]);
        if (two) {
          issue_s(1, 0);
          mma_commit(&ctl->s_full[1]);
        }
        mma_commit(&ctl->slot_empty[0]);
      }
      for (int n = 0; n < N && ok; ++n) {
        const int lv = 2 * n + 1, lk = 2 * n + 2;
        const bool more = n + 1 < N;
        ok = full_wait(lv);
        if (!ok) break;
        // the next key tile is normally resident long before it is needed;
        // waiting for it here keeps the waits out of the unit's MMA burst
        if (more) {
          ok = full_wait(lk);
          if (!ok) break;
        }
        if (n < NA) {
          ok = pv_unit(0, n, lv);
          if (!ok) break;
          if (n + 1 == NA) mma_commit(&ctl->o_final[0]);
        }
        if (more) {
          tc_fence_after();
          if (n + 1 < NA) {
            issue_s(0, lk);
            mma_commit(&ctl->s_full[0]);
          }
        }
        if (two) {
          ok = pv_unit(1, n, lv);
          if (!ok) break;
          if (!more) mma_commit(&ctl->o_final[1]);
        }
        mma_commit(&ctl->slot_empty[lv % NSLOT]);
        if (more) {
          if (two) {
            issue_s(1, lk);
            mma_commit(&ctl->s_full[1]);
          }
          mma_commit(&ctl->slot_empty[lk % NSLOT]);
        }
      }
      // no MMA may still be running when TMEM is released
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

}  // namespace sm100

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [rows][Hkv][128] bf16 as a 3-D tensor (dims, Hkv, rows); boxes of 64 dims x
// 1 head x 128 rows with 128-byte swizzle; rows >= n_rows read as zeros.
bool encode_kv_map(CUtensorMap* m, const void* base, int64_t n_rows, int Hkv) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {128u, static_cast<cuuint64_t>(Hkv), static_cast<cuuint64_t>(n_rows)};
  const cuuint64_t strides[2] = {128u * 2u, static_cast<cuuint64_t>(Hkv) * 128u * 2u};
  const cuuint32_t box[3] = {64u, 1u, 128u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_attention_sm100(const AttnArgs& a, cudaStream_t st) {
  using namespace sm100;
  if (a.Lq <= 0) return cudaSuccess;
  CUtensorMap tm_k, tm_v;
  if (!encode_kv_map(&tm_k, a.kr, a.Lk, a.Hkv) || !encode_kv_map(&tm_v, a.v, a.Lk, a.Hkv))
    return cudaErrorInvalidValue;
  Params p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.out = static_cast<__nv_bfloat16*>(a.out);
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
  p.n_two = p.G / 2;
  p.n_qtiles = static_cast<int>((a.Lq + BM - 1) / BM);
  // The last head of an odd group runs on two consecutive q-tiles per CTA when
  // every q-tile lies in one chunk and every (q-tile, k-tile) pair has one
  // class: then a q-tile's work list is its k-tiles in ascending order, and
  // the shorter tile's list is a prefix of the longer one's.
  p.lone_pairs = (p.G % 2 == 1) && a.reading == READING_A && a.s % BN == 0 &&
                 a.q_start % BM == 0;
  p.n_lone = p.G % 2 == 0 ? 0 : (p.lone_pairs ? (p.n_qtiles + 1) / 2 : p.n_qtiles);
  p.reading = a.reading;
  p.scale_log2 = a.scale_log2;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  p.debug = a.debug;
  const int64_t blocks =
      static_cast<int64_t>(p.Hkv) * (static_cast<int64_t>(p.n_qtiles) * p.n_two + p.n_lone);
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(dca_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  dca_fwd_kernel<<<static_cast<unsigned>(blocks), NUM_THREADS, SMEM_BYTES, st>>>(tm_k, tm_v, p);
  return cudaGetLastError();
}

}  // namespace dca
