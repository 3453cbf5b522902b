// dca_decode_sm100.cu -- Dual Chunk Attention for a few query rows against a
// long KV cache (the decode step that follows a chunked prefill), sm_100a.
//
// Same position map as the prefill kernel ("Qwen2.5-1M 不重训外推 1M",
// sections Intra / Successive / Inter-Chunk Attention): keys pre-rotated by
// j mod s in the workspace, each query row rotated by r_i, s + r_i (or c - 1
// outside the local window) or c - 1 according to the class of the key tile.
// With one or a few query rows per KV head the work is a stream over the
// whole cache (2 x 256 bytes per key and KV head) and HBM-bound, so the
// kernel is split-KV: the work list of the query block (dca_plan.cuh) is cut
// into contiguous slices, one CTA per (KV head, row group, slice), and a
// merge kernel combines the slices' partial softmax states.
//
// A row group is NR = 16 or 32 (token, head) rows of one KV head: the MMA N.
// One CTA (SW = NR/4 softmax warps + 2):
//   softmax warps  warp w owns TMEM lane quarter w % 4 -- key 32(w%4) + lane
//                  of the current 128-key tile in S^T, the same dim of O^T --
//                  and rows 16(w/4) .. +15 of the group
//   warp SW        TMA producer: K'/V tiles (128 keys x 128 dims, bf16,
//                  128-byte swizzle) into a ring of 32 KiB slots (no multicast)
//   warp SW+1      MMA issuer: S^T = K' Q_cls^T (M = 128 keys, N = NR rows)
//                  and O^T += V^T P^T (M = 128 dims, A = the V tile read
//                  MN-major, B = P^T in shared memory), tcgen05.mma kind::f16,
//                  fp32 accumulators in TMEM
// Query rows are rotated once per class at the start (three operand tiles).
// Online softmax per row: the four warps of a row half exchange their tile
// maxima through shared memory; the reference max moves (and O^T, l rescale)
// only when it grows by more than 2^8, as in the prefill kernel.
// Every wait is bounded (globaltimer); on timeout the CTA raises its abort
// flag, ORs a code into the device status word, drains its copies and MMAs,
// frees TMEM and exits.
#include <cuda_bf16.h>
#include <math.h>

#include "dca_internal.h"
#include "dca_plan.cuh"
#include "sm100_ptx.cuh"

namespace dca {
namespace dec {

constexpr int BN = 128;                  // keys per tile (MMA M of S^T)
constexpr int HD = 128;
constexpr int TILE_BYTES = 32768;        // 128 x 128 bf16
constexpr int HALF_BYTES = 16384;        // 128 rows x 64 bf16 (one swizzle column block)
constexpr float RESCALE_LOG2 = 8.0f;

constexpr unsigned ST_SOFTMAX = 0x10u, ST_LOAD = 0x100u, ST_MMA = 0x1000u, ST_DRAIN = 0x10000u;

template <int NR>
struct Cfg {
  static_assert(NR == 16 || NR == 32, "row group of 16 or 32");
  static constexpr int SW = NR / 4;                     // softmax warps
  // K'/V tile ring: 3 items in flight for 16 rows, 2.5 for 32 (shared-memory
  // budget; a 6-slot ring with one P^T buffer measured no faster for 32)
  static constexpr int NTILE = NR == 16 ? 6 : 5;
  static constexpr int NPB = 2;                         // P^T buffers
  static constexpr int OPB = NR * HD * 2;               // an NR-row operand (Q variant or P^T)
  static constexpr int OPB_HALF = NR * 128;             // its 64-column block
  static constexpr int THREADS = 32 * (SW + 2);
  static constexpr int WARP_LOAD = SW;
  static constexpr int WARP_MMA = SW + 1;
  static constexpr uint32_t TMEM_COLS = NR == 16 ? 64 : 128;  // S^T x2, O^T (NR cols each)
  static constexpr uint32_t COL_O = 2 * NR;
};

template <int NR>
struct SmemCtl {
  static constexpr int SW = Cfg<NR>::SW;
  uint64_t tile_full[Cfg<NR>::NTILE];
  uint64_t tile_empty[Cfg<NR>::NTILE];
  uint64_t s_full[2];
  uint64_t s_free[2];   // the softmax warps have read S^T
  uint64_t p_full[2];   // the softmax warps have written P^T
  uint64_t pv_done[2];  // O^T += V^T P^T of the item with this parity completed
  uint64_t max_bar[2];  // the warps' row maxima are in wmax
  uint64_t q_ready;
  uint64_t o_final;
  uint64_t epi_bar;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  alignas(16) float wmax[2][SW][16];  // read as float4
  float lsum[SW][16];
};

template <int NR>
constexpr size_t smem_bytes() {
  return 1024 + Cfg<NR>::NTILE * TILE_BYTES + (3 + Cfg<NR>::NPB) * Cfg<NR>::OPB +
         sizeof(SmemCtl<NR>);
}
static_assert(smem_bytes<16>() <= 232448 && smem_bytes<32>() <= 232448, "shared memory budget");

struct Params {
  const __nv_bfloat16* q;   // [Lq][Hq][128]
  const float2* tab;
  float* part;              // partial O [cta][NR][HD], m [cta][NR], l [cta][NR]
  int64_t q_start, Lq, Lk, s, w, tab_c1;
  int Hq, Hkv, G, n_rg, n_splits, n_cta;
  int reading;
  float scale_log2;
  TilePlan plan;            // work list of the query block [q_start, q_start + Lq)
  FullRanges fullr;         // its unmasked k-tiles per class
  unsigned int* status;
  unsigned long long timeout_ns;
  int debug;
};

// float -> int with the same order (for the integer warp max reduction); an involution.
__device__ __forceinline__ int ordered(int x) { return x >= 0 ? x : x ^ 0x7fffffff; }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Absolute position of row rho of row group rg (padding rows repeat the last row).
template <int NR>
__device__ __forceinline__ int64_t row_pos(const Params& p, int rg, int rho) {
  int64_t t = (static_cast<int64_t>(rg) * NR + rho) / p.G;
  if (t > p.Lq - 1) t = p.Lq - 1;
  return p.q_start + t;
}

template <int NR>
__global__ void __launch_bounds__(Cfg<NR>::THREADS, 1)
    dca_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<NR>;
  constexpr int SW = C::SW, NTILE = C::NTILE, OPB = C::OPB, OPB_HALF = C::OPB_HALF;
  constexpr int NPB = C::NPB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint8_t* qv = tiles + NTILE * TILE_BYTES;  // Q variants, indexed by class
  uint8_t* pt = qv + 3 * OPB;                // P^T, NPB buffers
  SmemCtl<NR>* ctl = reinterpret_cast<SmemCtl<NR>*>(pt + NPB * OPB);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: row group fastest (CTAs reading the same K'/V slice run
  // together and share it in L2), then slice, then KV head
  const int b = static_cast<int>(blockIdx.x);
  const int rg = b % p.n_rg;
  const int sp = (b / p.n_rg) % p.n_splits;
  const int g = b / (p.n_rg * p.n_splits);
  const int cta = (g * p.n_rg + rg) * p.n_splits + sp;
  const int it0 = static_cast<int>(static_cast<int64_t>(p.plan.n_items) * sp / p.n_splits);
  const int it1 = static_cast<int>(static_cast<int64_t>(p.plan.n_items) * (sp + 1) / p.n_splits);
  const int N = it1 - it0;
  const int64_t rows_left = p.Lq * p.G - static_cast<int64_t>(rg) * NR;
  const int n_rows = static_cast<int>(rows_left < NR ? rows_left : NR);

  if (threadIdx.x == 0) {
    for (int k = 0; k < NTILE; ++k) {
      mbar_init(&ctl->tile_full[k], 1);
      mbar_init(&ctl->tile_empty[k], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&ctl->s_full[k], 1);
      mbar_init(&ctl->s_free[k], SW);
      mbar_init(&ctl->p_full[k], SW);
      mbar_init(&ctl->pv_done[k], 1);
      mbar_init(&ctl->max_bar[k], SW);
    }
    mbar_init(&ctl->q_ready, SW);
    mbar_init(&ctl->o_final, 1);
    mbar_init(&ctl->epi_bar, SW);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == C::WARP_MMA) {
    tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::WARP_LOAD && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = ctl->tmem_base;
  volatile int* abort_flag = &ctl->abort;

  if (warp < SW) {
    // =========================================================== softmax
    const int quad = warp & 3;        // TMEM lane quarter: keys / dims 32*quad + lane
    const int rh = warp >> 2;         // rows 16*rh .. 16*rh + 15 of the group
    const int tau = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const float sc = p.scale_log2;

    // The rotated query operands (NR rows x 128 dims, K-major, 128-byte
    // swizzle) of the classes in the work list (the RoPE table holds the
    // positions s + r only when the cache extends past the first chunk, which
    // is when the list has successive-chunk items); task = (class, row,
    // 8-dim chunk of each half), 3 NR 8 tasks over 32 SW = 8 NR threads:
    // three per thread, their loads all issued before the first use.
    constexpr int QTASKS = 3;
    static_assert(3 * NR * 8 == QTASKS * 32 * SW, "three query tasks per softmax thread");
    uint4 xa[QTASKS], xb[QTASKS];
    float4 cs[QTASKS][4];
    bool live[QTASKS];
#pragma unroll
    for (int u = 0; u < QTASKS; ++u) {
      const int task = warp * 32 + lane + u * 32 * SW;
      const int cls = task / (NR * 8);
      const int rho = (task >> 3) % NR;
      const int c = task & 7;
      live[u] = rho < n_rows && p.plan.hi[cls] > p.plan.lo[cls];
      xa[u] = xb[u] = make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int e = 0; e < 4; ++e) cs[u][e] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (live[u]) {
        const int64_t rho_g = static_cast<int64_t>(rg) * NR + rho;
        const int64_t t = rho_g / p.G;
        const int h = g * p.G + static_cast<int>(rho_g % p.G);
        const __nv_bfloat16* qrow = p.q + (t * p.Hq + h) * static_cast<int64_t>(HD);
        const float4* t4 = reinterpret_cast<const float4*>(
            p.tab + query_table_row(p.q_start + t, cls, p.s, p.w, p.tab_c1) * (HD / 2) + 8 * c);
        xa[u] = *reinterpret_cast<const uint4*>(qrow + 8 * c);
        xb[u] = *reinterpret_cast<const uint4*>(qrow + 64 + 8 * c);
#pragma unroll
        for (int e = 0; e < 4; ++e) cs[u][e] = t4[e];
      }
    }
#pragma unroll
    for (int u = 0; u < QTASKS; ++u) {
      const int task = warp * 32 + lane + u * 32 * SW;
      const int cls = task / (NR * 8);
      const int rho = (task >> 3) % NR;
      const int c = task & 7;
      uint4 oa = make_uint4(0, 0, 0, 0), ob = oa;
      if (live[u]) {
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&xa[u]);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xb[u]);
        uint32_t* pa = reinterpret_cast<uint32_t*>(&oa);
        uint32_t* pb = reinterpret_cast<uint32_t*>(&ob);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 r = cs[u][e];
          const float2 x = __bfloat1622float2(a2[e]);
          const float2 y = __bfloat1622float2(b2[e]);
          pa[e] = pack_bf16(x.x * r.x - y.x * r.y, x.y * r.z - y.y * r.w);
          pb[e] = pack_bf16(x.x * r.y + y.x * r.x, x.y * r.w + y.y * r.z);
        }
      }
      uint8_t* dst = qv + cls * OPB + rho * 128 + ((c ^ (rho & 7)) << 4);
      *reinterpret_cast<uint4*>(dst) = oa;
      *reinterpret_cast<uint4*>(dst + OPB_HALF) = ob;
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->q_ready);

    // P^T store address of this thread's key (rows add 128 bytes and change
    // the swizzle phase)
    const int kh = tau >> 6, kin = tau & 63;

    float m_ref[16], l_part[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      m_ref[r] = -INFINITY;
      l_part[r] = 0.f;
    }
    bool ok = true;
    for (int n = 0; n < N && ok; ++n) {
      int kt, cls;
      plan_item(p.plan, it0 + n, kt, cls);
      const bool full = is_full(p.fullr, kt, cls);
      const int buf = n & 1;
      const uint32_t ph = static_cast<uint32_t>((n >> 1) & 1);

      ok = wait_poll(&ctl->s_full[buf], ph, abort_flag, p.status, p.timeout_ns, ST_SOFTMAX);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[16];
      tmem_ld16(tbase + lane_off + static_cast<uint32_t>(buf * NR + 16 * rh), sv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->s_free[buf]);

      if (!full) {
        const int64_t j = static_cast<int64_t>(kt) * BN + tau;
        const int64_t nj = j / p.s;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const int64_t i = row_pos<NR>(p, rg, 16 * rh + r);
          const bool valid =
              j <= i && pair_class(i / p.s - nj, i - j, p.w, p.reading) == cls;
          if (!valid) sv[r] = 0xff800000u;  // -inf
        }
      }

      // row maxima over the warp's 32 keys, then over the row half's four warps
      float mine = -INFINITY;
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int v = __reduce_max_sync(0xffffffffu, ordered(static_cast<int>(sv[r])));
        if (lane == r) mine = __int_as_float(ordered(v));
      }
      if (lane < 16) ctl->wmax[buf][warp][lane] = mine;
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->max_bar[buf]);
      ok = wait_poll(&ctl->max_bar[buf], ph, abort_flag, p.status, p.timeout_ns, ST_SOFTMAX);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      // reference update (identical in the four warps of a row half: same
      // maxima, same history); O^T holds items < n, so when a reference
      // moves its columns are rescaled once the last P.V landed
      {
        float alpha[16];
        bool any = false;
#pragma unroll
        for (int r4 = 0; r4 < 4; ++r4) {
          // tile maxima of rows 4 r4 .. 4 r4 + 3 over the row half's four warps
          float4 t = reinterpret_cast<const float4*>(ctl->wmax[buf][4 * rh])[r4];
#pragma unroll
          for (int wq = 1; wq < 4; ++wq) {
            const float4 o = reinterpret_cast<const float4*>(ctl->wmax[buf][4 * rh + wq])[r4];
            t.x = fmaxf(t.x, o.x);
            t.y = fmaxf(t.y, o.y);
            t.z = fmaxf(t.z, o.z);
            t.w = fmaxf(t.w, o.w);
          }
          const float tm[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int r = 4 * r4 + e;
            const float m_new = fmaxf(m_ref[r], tm[e]);
            const bool need = (m_new > m_ref[r]) &&
                              (m_ref[r] == -INFINITY || (m_new - m_ref[r]) * sc > RESCALE_LOG2);
            alpha[r] = 1.f;
            if (need) {
              alpha[r] = (m_ref[r] == -INFINITY) ? 0.f : ex2_approx((m_ref[r] - m_new) * sc);
              m_ref[r] = m_new;
              l_part[r] *= alpha[r];
              any = true;
            }
          }
        }
        if (any && n > 0) {
          const int m = n - 1;
          ok = wait_bounded(&ctl->pv_done[m & 1], static_cast<uint32_t>((m >> 1) & 1),
                            abort_flag, p.status, p.timeout_ns, ST_SOFTMAX);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          uint32_t o[16];
          const uint32_t t_o = tbase + lane_off + C::COL_O + static_cast<uint32_t>(16 * rh);
          tmem_ld16(t_o, o);
#pragma unroll
          for (int r = 0; r < 16; ++r) o[r] = __float_as_uint(__uint_as_float(o[r]) * alpha[r]);
          tmem_st16(t_o, o);
          tmem_st_wait();
        }
      }
      float pv[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const float mb = (m_ref[r] == -INFINITY) ? 0.f : m_ref[r] * sc;
        pv[r] = ex2_approx(fmaf(__uint_as_float(sv[r]), sc, -mb));
        l_part[r] += pv[r];
      }
      // the P^T buffer is free once the P.V of item n - NPB completed
      if (n >= NPB) {
        const int m = n - NPB;
        ok = wait_bounded(&ctl->pv_done[m & 1], static_cast<uint32_t>((m >> 1) & 1), abort_flag,
                          p.status, p.timeout_ns, ST_SOFTMAX);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      uint8_t* pb = pt + (n % NPB) * OPB + kh * OPB_HALF + ((kin & 7) << 1);
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int row = 16 * rh + r;
        const __nv_bfloat16 v = __float2bfloat16_rn(pv[r]);
        *reinterpret_cast<__nv_bfloat16*>(pb + row * 128 + (((kin >> 3) ^ (row & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[buf]);
    }

    // ---- epilogue: partial (m, l, O) of this slice
    if (ok && N > 0) {
      ok = wait_bounded(&ctl->o_final, 0u, abort_flag, p.status, p.timeout_ns, ST_SOFTMAX);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      uint32_t o[16];
      if (N > 0) {
        tc_fence_after();
        tmem_ld16(tbase + lane_off + C::COL_O + static_cast<uint32_t>(16 * rh), o);
      } else {
#pragma unroll
        for (int r = 0; r < 16; ++r) o[r] = 0u;
      }
      float mine = 0.f, mref_mine = -INFINITY;
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float v = l_part[r];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == r) {
          mine = v;
          mref_mine = m_ref[r];
        }
      }
      if (lane < 16) ctl->lsum[warp][lane] = mine;
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->epi_bar);
      ok = wait_bounded(&ctl->epi_bar, 0u, abort_flag, p.status, p.timeout_ns, ST_SOFTMAX);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        float* po = p.part + static_cast<size_t>(cta) * NR * HD;
        float* pm = p.part + static_cast<size_t>(p.n_cta) * NR * HD + static_cast<size_t>(cta) * NR;
        float* pl = pm + static_cast<size_t>(p.n_cta) * NR;
#pragma unroll
        for (int r = 0; r < 16; ++r)
          if (16 * rh + r < n_rows) po[(16 * rh + r) * HD + tau] = __uint_as_float(o[r]);
        if (quad == 0 && lane < 16 && 16 * rh + lane < n_rows) {
          pm[16 * rh + lane] = (mref_mine == -INFINITY) ? -INFINITY : mref_mine * sc;
          pl[16 * rh + lane] = ctl->lsum[warp][lane] + ctl->lsum[warp + 1][lane] +
                               ctl->lsum[warp + 2][lane] + ctl->lsum[warp + 3][lane];
        }
      }
    }
  } else if (warp == C::WARP_LOAD) {
    // =========================================================== TMA producer
    if (lane == 0) {
      int last_li[NTILE];
#pragma unroll
      for (int k = 0; k < NTILE; ++k) last_li[k] = -1;
      bool ok = true;
      for (int n = 0; n < N && ok; ++n) {
        int kt, cls;
        plan_item(p.plan, it0 + n, kt, cls);
        for (int which = 0; which < 2; ++which) {  // 0: keys, 1: values
          const int li = 2 * n + which;
          const int slot = li % NTILE;
          const int use = li / NTILE;
          if (use > 0) {
            ok = wait_bounded(&ctl->tile_empty[slot], static_cast<uint32_t>((use - 1) & 1),
                              abort_flag, p.status, p.timeout_ns, ST_LOAD);
            if (!ok) break;
          }
          if ((p.debug & 1) && li == 0) continue;  // test hook: withhold the first key tile
          uint8_t* dst = tiles + slot * TILE_BYTES;
          const CUtensorMap* tm = which ? &tm_v : &tm_k;
          mbar_arrive_expect_tx(&ctl->tile_full[slot], TILE_BYTES);
          tma_load_3d(dst, tm, &ctl->tile_full[slot], 0, g, kt * BN);
          tma_load_3d(dst + HALF_BYTES, tm, &ctl->tile_full[slot], 64, g, kt * BN);
          last_li[slot] = li;
        }
      }
      for (int k = 0; k < NTILE; ++k)
        if (last_li[k] >= 0)
          wait_drain(&ctl->tile_full[k], static_cast<uint32_t>((last_li[k] / NTILE) & 1),
                     p.status, p.timeout_ns, ST_DRAIN);
    }
    __syncwarp();
  } else if (warp == C::WARP_MMA) {
    // =========================================================== MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32_major(BN, NR, false, false);
      const uint32_t id_o = idesc_bf16_f32_major(HD, NR, true, false);
      // Descriptors built once; a k-step or buffer adds its byte offset / 16
      // to the start-address field (shared addresses stay below 256 KiB).
      const uint64_t dq0 = sdesc_sw128(smem_u32(qv), 16, 1024);
      const uint64_t dp0 = sdesc_sw128(smem_u32(pt), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(tiles), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(tiles), HALF_BYTES, 1024);
      auto tile_wait = [&](int li) {
        return wait_spin(&ctl->tile_full[li % NTILE], static_cast<uint32_t>((li / NTILE) & 1),
                         abort_flag, p.status, p.timeout_ns, ST_MMA);
      };
      bool ok = wait_bounded(&ctl->q_ready, 0u, abort_flag, p.status, p.timeout_ns, ST_MMA);
      for (int n = 0; n <= N && ok; ++n) {
        if (n < N) {
          int kt, cls;
          plan_item(p.plan, it0 + n, kt, cls);
          const int li = 2 * n;
          ok = tile_wait(li);
          if (!ok) break;
          if (n >= 2) {
            ok = wait_spin(&ctl->s_free[n & 1], static_cast<uint32_t>(((n - 2) >> 1) & 1),
                           abort_flag, p.status, p.timeout_ns, ST_MMA);
            if (!ok) break;
          }
          tc_fence_after();
          const uint64_t dk = dk0 + static_cast<uint64_t>(((li % NTILE) * TILE_BYTES) >> 4);
          const uint64_t dq = dq0 + static_cast<uint64_t>((cls * OPB) >> 4);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint64_t ka = static_cast<uint64_t>(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4);
            const uint64_t kb = static_cast<uint64_t>(((kk >> 2) * OPB_HALF + (kk & 3) * 32) >> 4);
            mma_ss(tbase + static_cast<uint32_t>((n & 1) * NR), dk + ka, dq + kb, id_s,
                   kk > 0 ? 1u : 0u);
          }
          mma_commit(&ctl->s_full[n & 1]);
          mma_commit(&ctl->tile_empty[li % NTILE]);
        }
        if (n >= 1) {
          const int m = n - 1;
          const int lv = 2 * m + 1;
          ok = tile_wait(lv);
          if (!ok) break;
          ok = wait_spin(&ctl->p_full[m & 1], static_cast<uint32_t>((m >> 1) & 1), abort_flag,
                         p.status, p.timeout_ns, ST_MMA);
          if (!ok) break;
          tc_fence_after();
          const uint64_t dv = dv0 + static_cast<uint64_t>(((lv % NTILE) * TILE_BYTES) >> 4);
          const uint64_t dp = dp0 + static_cast<uint64_t>(((m % NPB) * OPB) >> 4);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t kb = static_cast<uint64_t>(((kk >> 2) * OPB_HALF + (kk & 3) * 32) >> 4);
            mma_ss(tbase + C::COL_O, dv + static_cast<uint64_t>((kk * 2048) >> 4), dp + kb, id_o,
                   (m > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&ctl->pv_done[m & 1]);
          mma_commit(&ctl->tile_empty[lv % NTILE]);
        }
      }
      if (ok && N > 0) mma_commit(&ctl->o_final);
      // no MMA may still be running when TMEM is released
      mma_commit(&ctl->drain);
      wait_drain(&ctl->drain, 0u, p.status, p.timeout_ns, ST_DRAIN);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// Merge the slices of each (token, head) row: with slice maxima m_k (log2
// units), sums l_k and unnormalised outputs O_k, out = sum_k 2^(m_k - M) O_k /
// sum_k 2^(m_k - M) l_k with M = max m_k; LSE (natural log) = (M + log2 of the
// denominator) ln 2.  One CTA per row, one thread per dim: it loads the
// first MERGE_BATCH slices' values of its dim, fetches the slices' (m, l)
// into shared memory while those loads are in flight, then accumulates.
constexpr int MERGE_MAX_SPLITS = DECODE_MAX_CTAS;
constexpr int MERGE_BATCH = 32;

__global__ void __launch_bounds__(HD)
    dca_decode_combine_kernel(const float* __restrict__ part, __nv_bfloat16* __restrict__ out,
                              float* __restrict__ lse, int Hq, int G, int nr, int n_rg,
                              int n_splits, int n_cta) {
  __shared__ float wk[MERGE_MAX_SPLITS];
  __shared__ float lk[MERGE_MAX_SPLITS];
  __shared__ float red[HD / 32];
  const int row = static_cast<int>(blockIdx.x);  // t * Hq + h
  const int t = row / Hq, h = row % Hq;
  const int g = h / G;
  const int rho_g = t * G + (h % G);
  const int rg = rho_g / nr, rho = rho_g % nr;
  const int c0 = (g * n_rg + rg) * n_splits;
  const float* pm = part + static_cast<size_t>(n_cta) * nr * HD;
  const float* pl = pm + static_cast<size_t>(n_cta) * nr;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* po = part + (static_cast<size_t>(c0) * nr + rho) * HD + tid;
  const size_t stride = static_cast<size_t>(nr) * HD;

  float ov[MERGE_BATCH];
#pragma unroll
  for (int u = 0; u < MERGE_BATCH; ++u) ov[u] = u < n_splits ? __ldcg(po + u * stride) : 0.f;

  float mx = -INFINITY;
  for (int k = tid; k < n_splits; k += HD) {
    const float m = __ldcg(pm + (c0 + k) * nr + rho);
    wk[k] = m;
    lk[k] = __ldcg(pl + (c0 + k) * nr + rho);
    mx = fmaxf(mx, m);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  const float M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  float lsum = 0.f;
  for (int k = tid; k < n_splits; k += HD) {
    const float w = (wk[k] == -INFINITY) ? 0.f : exp2f(wk[k] - M);
    wk[k] = w;
    lsum = fmaf(w, lk[k], lsum);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
  __syncthreads();  // wk complete; red reused below
  if (lane == 0) red[warp] = lsum;
  __syncthreads();
  const float L = red[0] + red[1] + red[2] + red[3];

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < n_splits; k0 += MERGE_BATCH) {
    if (k0 > 0) {
#pragma unroll
      for (int u = 0; u < MERGE_BATCH; ++u)
        ov[u] = k0 + u < n_splits ? __ldcg(po + (k0 + u) * stride) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < MERGE_BATCH; ++u)
      if (k0 + u < n_splits) acc[u & 3] = fmaf(wk[k0 + u], ov[u], acc[u & 3]);
  }
  const float o = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  out[static_cast<size_t>(row) * HD + tid] = __float2bfloat16_rn(o / L);
  if (lse != nullptr && tid == 0) lse[row] = (M + log2f(L)) * 0.6931471805599453f;
}

template <int NR>
cudaError_t launch(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const Params& p,
                   cudaStream_t st) {
  constexpr size_t smem = smem_bytes<NR>();
  cudaError_t e = cudaFuncSetAttribute(dca_decode_kernel<NR>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dca_decode_kernel<NR><<<static_cast<unsigned>(p.n_cta), Cfg<NR>::THREADS, smem, st>>>(tm_k,
                                                                                         tm_v, p);
  return cudaGetLastError();
}

}  // namespace dec

cudaError_t launch_decode_sm100(const AttnArgs& a, float* part, cudaStream_t st) {
  using namespace dec;
  if (a.Lq <= 0) return cudaSuccess;
  CUtensorMap tm_k, tm_v;
  if (!encode_kv_map(&tm_k, a.kr, a.Lk, a.Hkv) || !encode_kv_map(&tm_v, a.v, a.Lk, a.Hkv))
    return cudaErrorInvalidValue;
  Params p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.tab = a.tab;
  p.part = part;
  p.q_start = a.q_start;
  p.Lq = a.Lq;
  p.Lk = a.Lk;
  p.s = a.s;
  p.w = a.w;
  p.tab_c1 = a.tab_c1;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.reading = a.reading;
  p.scale_log2 = a.scale_log2;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  p.debug = a.debug;
  const int64_t i_last = a.q_start + a.Lq - 1;
  p.plan = make_plan(a.q_start, i_last, a.s, a.w, BN, a.reading);
  p.fullr = make_full_ranges(a.q_start, i_last, a.s, a.w, BN, a.reading);
  const int nr = decode_group_rows(a.Lq, p.G);
  p.n_rg = decode_row_groups(a.Lq, p.G);
  const int max_splits = decode_max_splits(a.Hkv, p.n_rg);
  p.n_splits = p.plan.n_items < max_splits ? p.plan.n_items : max_splits;
  if (p.n_splits < 1) p.n_splits = 1;
  const int64_t n_cta = static_cast<int64_t>(a.Hkv) * p.n_rg * p.n_splits;
  if (n_cta > 0x7fffffffLL || a.Lq * a.Hq > 0x7fffffffLL) return cudaErrorInvalidValue;
  p.n_cta = static_cast<int>(n_cta);
  cudaError_t e = nr == 16 ? launch<16>(tm_k, tm_v, p, st) : launch<32>(tm_k, tm_v, p, st);
  if (e != cudaSuccess) return e;
  dca_decode_combine_kernel<<<static_cast<unsigned>(a.Lq * a.Hq), HD, 0, st>>>(
      part, static_cast<__nv_bfloat16*>(a.out), a.lse, a.Hq, p.G, nr, p.n_rg, p.n_splits,
      p.n_cta);
  return cudaGetLastError();
}

}  // namespace dca
