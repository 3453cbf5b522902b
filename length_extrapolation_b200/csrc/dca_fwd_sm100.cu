// dca_fwd_sm100.cu -- fused Dual Chunk Attention forward for sm_100a.
//
// One CTA computes one 128-row query tile for two query heads of the same KV
// group (GQA: the K/V tiles it streams are shared by both heads; when the group
// size is odd the last head runs alone).  Warp roles (320 threads):
//   warps 0-7  softmax.  Warp w and warp w+4 share TMEM lanes 32*(w%4)..+31
//              (one query row per lane) and split each row's 128 keys in two
//              halves; every work item they process head A's scores, then
//              head B's, so two warps per SM sub-partition work on the head
//              whose scores are ready while the tensor cores run the other
//              head's MMAs (ping-pong).
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
// A share of the exponentials runs on the FMA pipe (exp2_poly2) to relieve the
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
#define DCA_NSLOT 4
#endif
constexpr int NSLOT = DCA_NSLOT;   // K/V ring slots
constexpr int TILE_BYTES = 32768;  // 128 x 128 bf16
constexpr int HALF_BYTES = 16384;  // 128 rows x 64 bf16 (one 128-byte swizzle column block)
// 10 warps: 8 softmax (warps 0-3 head A, 4-7 head B; one query row per
// thread), TMA producer, MMA issuer.
constexpr int NUM_THREADS = 320;
constexpr int WARP_LOAD = 8;
constexpr int WARP_MMA = 9;
constexpr float RESCALE_LOG2 = 8.0f;
// How the softmax threads wait for the partner's half-row maximum and for S:
// polling (no suspension) -- both are on the critical path of every item, and
// a suspended thread wakes up hundreds of cycles after the phase completes.
#ifndef DCA_PAIR_WAIT
#define DCA_PAIR_WAIT wait_poll
#endif
#ifndef DCA_S_WAIT
#define DCA_S_WAIT wait_poll
#endif
// How the MMA issuer waits: polling with a short back-off (wait_spin) or a
// suspending try_wait (wait_bounded).
#ifndef DCA_MMA_WAIT
#define DCA_MMA_WAIT wait_spin
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
  uint32_t tmem_base;
  int abort;
  // values exchanged between the two threads of a row: [phase parity][half][row]
  float xval[2][2][128];
  uint64_t pair_bar[4];  // one per TMEM lane quarter (its two warps arrive)
};

constexpr size_t SMEM_BYTES = 1024 + 2 * TILE_BYTES + NSLOT * TILE_BYTES + sizeof(SmemCtl);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

struct Params {
  const __nv_bfloat16* q;
  __nv_bfloat16* out;
  const float2* tab;
  int64_t q_start, Lq, Lk;
  int64_t s, w, tab_c1;
  int Hq, Hkv, G, n_pairs, n_qtiles;
  int reading;  // READING_A or READING_B
  float scale_log2;
  unsigned int* status;
  unsigned long long timeout_ns;
  int debug;
};

// One online-softmax step for HALF of a query row: this thread owns keys
// [64*half, 64*half + 64) of the scores in TMEM columns tS..tS+127; the thread
// holding the other half (same TMEM lane, warp +/- 4) exchanges its partial
// maximum through pair_exchange.  Writes P (bf16) for its keys into columns
// tS + 32*half .. +31 (scores both halves have read: the exchange orders both
// loads before either store), keeps its partial row sum, and rescales its half
// of O (tO) when the row maximum moved more than 2^RESCALE_LOG2 above the
// reference (otherwise P may reach 2^8, exact in fp32 and in bf16's exponent
// range; the final O / l uses the same reference).  O holds items < n: their
// MMAs completed before S(n) did (one commit tracks all earlier MMAs).
__device__ __forceinline__ bool softmax_half_step(uint32_t tS, uint32_t tO, int n, bool full,
                                                  int64_t i, int kt, int cls, int64_t s, int64_t w,
                                                  int reading, float sc,
                                                  float& m_ref, float& l_sum, PairCtx& pc,
                                                  volatile int* abort, unsigned int* status,
                                                  uint64_t timeout_ns, unsigned int code) {
  const int half = pc.half;
  uint32_t sv[64];
  tmem_ld64(tS + 64u * half, sv);
  if (!full) mask_cols<64>(sv, i, static_cast<int64_t>(kt) * BN + 64 * half, cls, s, w, reading);
  float mx = max64(sv);
  float mx_other = -INFINITY;
  if (!pair_exchange(pc, mx, mx_other, abort, status, timeout_ns, code)) return false;
  mx = fmaxf(mx, mx_other);

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
  l_sum += exp_pack64(sv, sc, (m_ref == -INFINITY) ? 0.f : m_ref * sc, pk);
  tmem_st32(tS + 32u * half, pk);
  // TMEM access is warp-collective: rescale when any row of the warp needs it
  // (rows whose max did not move use alpha = 1)
  if (n > 0 && __any_sync(0xffffffffu, need)) {
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
    dca_fwd_kernel(const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* q_buf0 = smem;
  uint8_t* q_buf1 = smem + TILE_BYTES;
  uint8_t* slots = smem + 2 * TILE_BYTES;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(slots + NSLOT * TILE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit
  // KV-group-major order: the CTAs running together stream the same group's
  // K'/V tiles (shared in L2); within a group, longest query tiles first.
  // Within a group the CTAs with two heads come first and a lone head (odd
  // G) after them: CTAs with equal work run side by side and stay in step
  // along the key stream, so the tiles they read are still in L2.
  const int per_group = p.n_qtiles * p.n_pairs;
  const int g = static_cast<int>(blockIdx.x) / per_group;
  const int c = static_cast<int>(blockIdx.x) % per_group;
  const int n_two = p.G / 2;  // pairs with two heads
  int qt_idx, pr;
  if (c < p.n_qtiles * n_two) {
    qt_idx = c / n_two;
    pr = c % n_two;
  } else {
    qt_idx = c - p.n_qtiles * n_two;
    pr = n_two;
  }
  const int qt = p.n_qtiles - 1 - qt_idx;
  const int h0 = g * p.G + 2 * pr;
  const bool two = (2 * pr + 1) < p.G;
  const int64_t i0 = p.q_start + static_cast<int64_t>(qt) * BM;
  const int64_t q_end = p.q_start + p.Lq;
  const int64_t i_last = (i0 + BM - 1 < q_end - 1) ? i0 + BM - 1 : q_end - 1;
  const int64_t i_hi = i0 + BM - 1;
  const TilePlan plan = make_plan(i0, i_last, p.s, p.w, BN, p.reading);
  const FullRanges fullr = make_full_ranges(i0, i_hi, p.s, p.w, BN, p.reading);
  const int N = plan.n_items;

  if (threadIdx.x == 0) {
    for (int k = 0; k < NSLOT; ++k) {
      mbar_init(&ctl->slot_full[k], 1);
      mbar_init(&ctl->slot_empty[k], 1);
    }
    for (int st = 0; st < 2; ++st) {
      mbar_init(&ctl->s_full[st], 1);
      mbar_init(&ctl->p_full[st], 8);   // one arrival per softmax warp
      mbar_init(&ctl->q_ready[st], 8);
      mbar_init(&ctl->o_final[st], 1);
    }
    mbar_init(&ctl->drain, 1);
    for (int k = 0; k < 4; ++k) mbar_init(&ctl->pair_bar[k], 2);
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
    // All 8 warps work on head A's scores, then on head B's, for every item:
    // warp w and warp w+4 share TMEM lanes 32*(w%4).. (one query row per lane)
    // and split each row's 128 keys in two halves.  Two warps per SM
    // sub-partition keep its MUFU/FMA pipes busy on the current head while the
    // tensor cores run the other head's MMAs.
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
    const __nv_bfloat16* qrow0 =
        real ? p.q + ((i - p.q_start) * p.Hq + h0) * static_cast<int64_t>(HD) : nullptr;
    const __nv_bfloat16* qrow1 = (real && two) ? qrow0 + HD : nullptr;  // head h0 + 1
    const int c0 = 4 * half, c1 = 4 * half + 4;  // this thread's share of the Q row

    int kt, cls;
    plan_item(plan, 0, kt, cls);
    {
      const float2* trow = real ? p.tab + query_table_row(i, cls, p.s, p.w, p.tab_c1) * 64 : nullptr;
      write_q_row(q_buf0, r, qrow0, trow, c0, c1);
      if (two) write_q_row(q_buf1, r, qrow1, trow, c0, c1);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ctl->q_ready[0]);
        if (two) mbar_arrive(&ctl->q_ready[1]);
      }
    }

    float m_ref[2] = {-INFINITY, -INFINITY};
    float l_sum[2] = {0.f, 0.f};
    bool ok = true;
    for (int n = 0; n < N && ok; ++n) {
      plan_item(plan, n, kt, cls);
      const bool full = is_full(fullr, kt, cls);
      int cls_next = cls;
      if (n + 1 < N) {
        int kt_next;
        plan_item(plan, n + 1, kt_next, cls_next);
      }
#pragma unroll
      for (int st = 0; st < 2; ++st) {
        if (st == 1 && !two) break;
        ok = DCA_S_WAIT(&ctl->s_full[st], static_cast<uint32_t>(n & 1), abort_flag, p.status,
                        p.timeout_ns, ST_SOFTMAX << st);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tbase + lane_off + static_cast<uint32_t>(st * 128);
        const uint32_t tO = tbase + lane_off + 256u + static_cast<uint32_t>(st * 128);
        ok = softmax_half_step(tS, tO, n, full, i, kt, cls, p.s, p.w, p.reading, sc, m_ref[st],
                               l_sum[st], pc,
                               abort_flag, p.status, p.timeout_ns, ST_SOFTMAX << st);
        if (!ok) break;
        if (cls_next != cls) {  // phase switch: the next items need another query rotation
          write_q_row(st ? q_buf1 : q_buf0, r, st ? qrow1 : qrow0,
                      real ? p.tab + query_table_row(i, cls_next, p.s, p.w, p.tab_c1) * 64
                           : nullptr,
                      c0, c1);
          fence_proxy_async_smem();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->p_full[st]);
      }
    }
    // epilogue: O / (l_half0 + l_half1) -> bf16 -> out (each thread writes its 64 columns)
#pragma unroll
    for (int st = 0; st < 2; ++st) {
      if (st == 1 && !two) break;
      if (ok) {
        ok = wait_bounded(&ctl->o_final[st], 0u, abort_flag, p.status, p.timeout_ns,
                          ST_SOFTMAX << st);
        ok = __all_sync(0xffffffffu, ok);
      }
      if (!ok) break;
      float l_other = 0.f;
      ok = pair_exchange(pc, l_sum[st], l_other, abort_flag, p.status, p.timeout_ns,
                         ST_SOFTMAX << st);
      if (!ok) break;
      const float l_tot = l_sum[st] + l_other;
      tc_fence_after();
      const uint32_t tO = tbase + lane_off + 256u + static_cast<uint32_t>(st * 128) + 64u * half;
      const float inv = 1.f / l_tot;
      __nv_bfloat16* orow =
          real ? p.out + ((i - p.q_start) * p.Hq + h0 + st) * static_cast<int64_t>(HD) + 64 * half
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
      bool ok = true;
      for (int n = 0; n < N && ok; ++n) {
        int kt, cls;
        plan_item(plan, n, kt, cls);
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
      const uint32_t q_addr[2] = {smem_u32(q_buf0), smem_u32(q_buf1)};
      const uint32_t slot_addr0 = smem_u32(slots);
      // Descriptors are built once; a k-step only adds its byte offset / 16 to
      // the start-address field (no carry out of the 14-bit field: shared
      // memory addresses stay below 256 KiB).
      const uint64_t dq[2] = {sdesc_sw128(q_addr[0], 16, 1024), sdesc_sw128(q_addr[1], 16, 1024)};
      const uint64_t dk0 = sdesc_sw128(slot_addr0, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(slot_addr0, HALF_BYTES, 1024);
      auto issue_s = [&](int st, int li) {
        const uint64_t dk = dk0 + static_cast<uint64_t>(((li % NSLOT) * TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4);
          mma_ss(tbase + static_cast<uint32_t>(st * 128), dq[st] + off, dk + off, id_s,
                 kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int st, int li, bool acc) {
        const uint64_t dv = dv0 + static_cast<uint64_t>(((li % NSLOT) * TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          mma_ts(tbase + 256u + static_cast<uint32_t>(st * 128),
                 tbase + static_cast<uint32_t>(st * 128 + kk * 8),
                 dv + static_cast<uint64_t>((kk * 2048) >> 4), id_o, (acc || kk > 0) ? 1u : 0u);
        }
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
        ok = DCA_MMA_WAIT(&ctl->p_full[0], static_cast<uint32_t>(n & 1), abort_flag, p.status,
                          p.timeout_ns, ST_MMA);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, lv, n > 0);
        if (more) {
          ok = full_wait(lk);
          if (!ok) break;
          tc_fence_after();
          issue_s(0, lk);
          mma_commit(&ctl->s_full[0]);
        }
        if (two) {
          ok = DCA_MMA_WAIT(&ctl->p_full[1], static_cast<uint32_t>(n & 1), abort_flag, p.status,
                            p.timeout_ns, ST_MMA);
          if (!ok) break;
          tc_fence_after();
          issue_pv(1, lv, n > 0);
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
      if (ok) {
        mma_commit(&ctl->o_final[0]);
        if (two) mma_commit(&ctl->o_final[1]);
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
  p.n_pairs = (p.G + 1) / 2;
  p.n_qtiles = static_cast<int>((a.Lq + BM - 1) / BM);
  p.reading = a.reading;
  p.scale_log2 = a.scale_log2;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  p.debug = a.debug;
  const int64_t blocks = static_cast<int64_t>(p.n_qtiles) * p.Hkv * p.n_pairs;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(dca_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  dca_fwd_kernel<<<static_cast<unsigned>(blocks), NUM_THREADS, SMEM_BYTES, st>>>(tm_k, tm_v, p);
  return cudaGetLastError();
}

}  // namespace dca
