// dca_fwd_sm100.cu -- fused Dual Chunk Attention forward for sm_100a.
//
// One CTA computes one 128-row query tile for two query heads of the same KV
// group (GQA: the K/V tiles it streams are shared by both heads; when the group
// size is odd the last head runs alone).  Warp roles:
//   warps 0-3  softmax of head A (one query row per thread, TMEM lanes 0-127)
//   warps 4-7  softmax of head B
//   warp  8    TMA producer: K'/V tiles (128 keys x 128 dims, bf16, 128-byte
//              swizzle) into a ring of shared-memory slots
//   warp  9    MMA issuer (one thread): S = Q K'^T and O += P V with
//              tcgen05.mma kind::f16 (bf16 in, fp32 accumulate in TMEM)
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512);
// P (bf16) overwrites the first 64 columns of its S and is the TMEM A operand
// of the P.V MMA.
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
// Online softmax: running max kept per row; O and the row sum are rescaled
// only when the max grows by more than 2^8 (P stays <= 256, exact in fp32 and
// in bf16's exponent range), the final O / l uses the same reference max.
//
// Every wait is bounded (globaltimer); on timeout the CTA raises a shared
// abort flag, ORs a code into the device status word, drains its own TMA
// copies and MMAs, frees TMEM and exits.
#include <cuda_bf16.h>
#include <math.h>

#include <mutex>

#include "dca_internal.h"
#include "dca_plan.cuh"
#include "sm100_ptx.cuh"

namespace dca {
namespace sm100 {

constexpr int BM = 128;            // query rows per tile
constexpr int BN = 128;            // keys per tile
constexpr int HD = 128;            // head dim
constexpr int NSLOT = 4;           // K/V ring slots
constexpr int TILE_BYTES = 32768;  // 128 x 128 bf16
constexpr int HALF_BYTES = 16384;  // 128 rows x 64 bf16 (one 128-byte swizzle column block)
constexpr int NUM_THREADS = 320;
constexpr int WARP_LOAD = 8;
constexpr int WARP_MMA = 9;
constexpr float RESCALE_LOG2 = 8.0f;

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
  float scale_log2;
  unsigned int* status;
  unsigned long long timeout_ns;
  int debug;
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Rotate one query row by the positions of table row `trow` and write it to
// the 128-byte-swizzled K-major operand tile (two 16 KiB column blocks: dims
// 0-63 and 64-127; RoPE pairs (k, k+64) sit at the same offset of each block).
__device__ __forceinline__ void write_q_row(uint8_t* qb, int r, const __nv_bfloat16* qrow,
                                            const float2* trow) {
  const uint32_t row_off = static_cast<uint32_t>(r) * 128u;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 oa = make_uint4(0, 0, 0, 0), ob = oa;
    if (qrow != nullptr) {
      const uint4 xa = *reinterpret_cast<const uint4*>(qrow + 8 * c);
      const uint4 xb = *reinterpret_cast<const uint4*>(qrow + 64 + 8 * c);
      const float4* t4 = reinterpret_cast<const float4*>(trow + 8 * c);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&xa);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xb);
      uint32_t* pa = reinterpret_cast<uint32_t*>(&oa);
      uint32_t* pb = reinterpret_cast<uint32_t*>(&ob);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 t = t4[e];
        const float2 x = __bfloat1622float2(a2[e]);
        const float2 y = __bfloat1622float2(b2[e]);
        pa[e] = pack_bf16(x.x * t.x - y.x * t.y, x.y * t.z - y.y * t.w);
        pb[e] = pack_bf16(x.x * t.y + y.x * t.x, x.y * t.w + y.y * t.z);
      }
    }
    const uint32_t phys = static_cast<uint32_t>((c ^ (r & 7)) * 16);
    *reinterpret_cast<uint4*>(qb + row_off + phys) = oa;
    *reinterpret_cast<uint4*>(qb + HALF_BYTES + row_off + phys) = ob;
  }
}

// Mask row i of a score tile (keys j0 .. j0+127) to the pairs that are causal
// and belong to class `cls`.
__device__ __forceinline__ void mask_row(uint32_t* sv, int64_t i, int64_t j0, int cls,
                                         int64_t s) {
  const int64_t ni = i / s;
  const int64_t nj0 = j0 / s;
  int64_t dn64 = ni - nj0;
  int dn = static_cast<int>(dn64 > (1 << 20) ? (1 << 20) : dn64);
  const int64_t b64 = (nj0 + 1) * s - j0;  // first column of the next chunk
  int bnd = static_cast<int>(b64 > (1 << 30) ? (1 << 30) : b64);
  const int s32 = static_cast<int>(s > (1 << 30) ? (1 << 30) : s);
  const int64_t lim64 = i - j0;  // last causal column
  const int lim = static_cast<int>(lim64 > 1024 ? 1024 : (lim64 < -1 ? -1 : lim64));
  const uint32_t NEG_INF = 0xff800000u;
#pragma unroll
  for (int e = 0; e < BN; ++e) {
    if (e >= bnd) {
      dn -= 1;
      bnd += s32;
    }
    const int ce = dn <= 0 ? CLS_INTRA : (dn == 1 ? CLS_SUCC : CLS_INTER);
    if (e > lim || ce != cls) sv[e] = NEG_INF;
  }
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

  // ---- work unit (longest causal rows first)
  const int units_per_qt = p.Hkv * p.n_pairs;
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x / units_per_qt);
  const int u = static_cast<int>(blockIdx.x % units_per_qt);
  const int g = u / p.n_pairs;
  const int pr = u % p.n_pairs;
  const int h0 = g * p.G + 2 * pr;
  const bool two = (2 * pr + 1) < p.G;
  const int64_t i0 = p.q_start + static_cast<int64_t>(qt) * BM;
  const int64_t q_end = p.q_start + p.Lq;
  const int64_t i_last = (i0 + BM - 1 < q_end - 1) ? i0 + BM - 1 : q_end - 1;
  const int64_t i_hi = i0 + BM - 1;
  const TilePlan plan = make_plan(i0, i_last, p.s, BN);
  const int N = plan.n_items;

  if (threadIdx.x == 0) {
    for (int k = 0; k < NSLOT; ++k) {
      mbar_init(&ctl->slot_full[k], 1);
      mbar_init(&ctl->slot_empty[k], 1);
    }
    for (int st = 0; st < 2; ++st) {
      mbar_init(&ctl->s_full[st], 1);
      mbar_init(&ctl->p_full[st], 128);
      mbar_init(&ctl->q_ready[st], 128);
      mbar_init(&ctl->o_final[st], 1);
    }
    mbar_init(&ctl->drain, 1);
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
    const int stage = warp >> 2;
    const int sub = warp & 3;
    const int r = sub * 32 + lane;
    const int64_t i = i0 + r;
    const bool real = i <= i_last;
    if (stage == 0 || two) {
      uint8_t* qb = stage ? q_buf1 : q_buf0;
      const int h = h0 + stage;
      const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
      const uint32_t tS = tbase + lane_off + static_cast<uint32_t>(stage * 128);
      const uint32_t tO = tbase + lane_off + 256u + static_cast<uint32_t>(stage * 128);
      const __nv_bfloat16* qrow =
          real ? p.q + ((i - p.q_start) * p.Hq + h) * static_cast<int64_t>(HD) : nullptr;
      const float sc = p.scale_log2;

      int kt, cls;
      plan_item(plan, 0, kt, cls);
      write_q_row(qb, r, qrow,
                  real ? p.tab + query_table_row(i, cls, p.s, p.w, p.tab_c1) * 64 : nullptr);
      fence_proxy_async_smem();
      mbar_arrive(&ctl->q_ready[stage]);

      float m_ref = -INFINITY;
      float l_sum = 0.f;
      bool ok = true;
      for (int n = 0; n < N; ++n) {
        plan_item(plan, n, kt, cls);
        ok = wait_bounded(&ctl->s_full[stage], static_cast<uint32_t>(n & 1), abort_flag,
                          p.status, p.timeout_ns, ST_SOFTMAX << stage);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();

        uint32_t sv[BN];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32u * c, sv + 32 * c);
        const int64_t j0 = static_cast<int64_t>(kt) * BN;
        if (!item_is_full(i0, i_hi, j0, j0 + BN - 1, p.s, cls)) mask_row(sv, i, j0, cls, p.s);

        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < BN; ++e) mx = fmaxf(mx, __uint_as_float(sv[e]));
        const float m_new = fmaxf(m_ref, mx);
        const bool need =
            (m_new > m_ref) && (m_ref == -INFINITY || (m_new - m_ref) * sc > RESCALE_LOG2);
        float alpha = 1.f;
        if (need) {
          alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx((m_ref - m_new) * sc);
          m_ref = m_new;
          l_sum *= alpha;
        }
        const float mb = (m_ref == -INFINITY) ? 0.f : m_ref * sc;
        float rs = 0.f;
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) {
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float a = ex2_approx(fmaf(__uint_as_float(sv[64 * hlf + 2 * e]), sc, -mb));
            const float b = ex2_approx(fmaf(__uint_as_float(sv[64 * hlf + 2 * e + 1]), sc, -mb));
            rs += a + b;
            pk[e] = pack_bf16(a, b);
          }
          tmem_st32(tS + 32u * hlf, pk);
        }
        l_sum += rs;
        // O still holds items < n (their MMAs completed before S(n) did); rescale
        // it before P(n) V(n) accumulates onto it.  Warp-uniform (TMEM access is
        // warp-collective); rows whose max did not move use alpha = 1.
        if (n > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + 32u * c, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + 32u * c, o);
          }
        }
        tmem_st_wait();
        if (n + 1 < N) {
          int kt2, cls2;
          plan_item(plan, n + 1, kt2, cls2);
          if (cls2 != cls) {  // phase switch: next items need another query rotation
            write_q_row(qb, r, qrow,
                        real ? p.tab + query_table_row(i, cls2, p.s, p.w, p.tab_c1) * 64
                             : nullptr);
            fence_proxy_async_smem();
          }
        }
        tc_fence_before();
        mbar_arrive(&ctl->p_full[stage]);
      }
      if (ok) {
        ok = wait_bounded(&ctl->o_final[stage], 0u, abort_flag, p.status, p.timeout_ns,
                          ST_SOFTMAX << stage);
        ok = __all_sync(0xffffffffu, ok);
      }
      if (ok) {
        tc_fence_after();
        const float inv = 1.f / l_sum;
        __nv_bfloat16* orow =
            real ? p.out + ((i - p.q_start) * p.Hq + h) * static_cast<int64_t>(HD) : nullptr;
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
  } else {
    // =========================================================== MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(BM, BN, false);
      const uint32_t id_o = idesc_bf16_f32(BM, HD, true);
      const uint32_t q_addr[2] = {smem_u32(q_buf0), smem_u32(q_buf1)};
      const uint32_t slot_addr0 = smem_u32(slots);
      auto issue_s = [&](int st, int li) {
        const uint32_t kb = slot_addr0 + static_cast<uint32_t>((li % NSLOT) * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = static_cast<uint32_t>((kk >> 2) * HALF_BYTES + (kk & 3) * 32);
          mma_ss(tbase + static_cast<uint32_t>(st * 128), sdesc_sw128(q_addr[st] + off, 16, 1024),
                 sdesc_sw128(kb + off, 16, 1024), id_s, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int st, int li, bool acc) {
        const uint32_t vb = slot_addr0 + static_cast<uint32_t>((li % NSLOT) * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          mma_ts(tbase + 256u + static_cast<uint32_t>(st * 128),
                 tbase + static_cast<uint32_t>(st * 128 + kk * 8),
                 sdesc_sw128(vb + static_cast<uint32_t>(kk * 2048), HALF_BYTES, 1024), id_o,
                 (acc || kk > 0) ? 1u : 0u);
        }
      };
      auto full_wait = [&](int li) {
        return wait_bounded(&ctl->slot_full[li % NSLOT], static_cast<uint32_t>((li / NSLOT) & 1),
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
        ok = wait_bounded(&ctl->p_full[0], static_cast<uint32_t>(n & 1), abort_flag, p.status,
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
          ok = wait_bounded(&ctl->p_full[1], static_cast<uint32_t>(n & 1), abort_flag, p.status,
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
static bool encode_kv_map(CUtensorMap* m, const void* base, int64_t n_rows, int Hkv) {
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

}  // namespace sm100

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
