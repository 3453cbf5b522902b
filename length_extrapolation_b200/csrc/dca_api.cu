// dca_api.cu -- the library's C ABI (declared in include/dca.h): argument
// validation on the host, workspace layout, and the launches of the
// preparation and attention kernels on the caller's stream.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/dca.h"
#include "dca_internal.h"
#include "dca_plan.cuh"
#include "dca_select_rows.cuh"
#include "dca_sparse_plan.cuh"

namespace {

constexpr size_t HDR_BYTES = 1024;  // status word + padding
constexpr int VERSION = 100;        // 0.1.0

std::atomic<long long> g_timeout_ns{10LL * 1000 * 1000 * 1000};
std::atomic<int> g_debug_flags{0};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Layout {
  int64_t cap = 0;       // key capacity
  int64_t T = 0;         // RoPE table rows
  int64_t n_direct = 0;  // table rows indexed by position
  size_t tab_off = 0, kr_off = 0, total = 0;
};

bool basic_params_ok(int Hq, int Hkv, int d, int64_t s, int64_t w, int64_t c, int dtype) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return false;
  if (d <= 0 || d % 2 != 0) return false;
  if (s < 1 || w < 0 || w > s || c < 1) return false;
  if (dtype != DCA_BF16 && dtype != DCA_F32) return false;
  return true;
}

Layout make_layout(int64_t cap, int Hkv, int d, int64_t s, int64_t w, int dtype) {
  Layout L;
  L.cap = cap;
  L.T = dca::table_rows(cap, s, w);
  L.n_direct = L.T - 1;
  const size_t esize = dtype == DCA_BF16 ? 2 : 4;
  L.tab_off = HDR_BYTES;
  L.kr_off = align_up(L.tab_off + static_cast<size_t>(L.T) * (d / 2) * sizeof(float2), 1024);
  L.total = L.kr_off + align_up(static_cast<size_t>(cap) * Hkv * d * esize, 1024);
  return L;
}

// Largest key capacity whose layout fits in ws_bytes (layout size grows with cap).
int64_t capacity_for(size_t ws_bytes, int Hkv, int d, int64_t s, int64_t w, int dtype) {
  int64_t lo = 0, hi = (1LL << 31) - 1;
  if (make_layout(0, Hkv, d, s, w, dtype).total > ws_bytes) return -1;
  while (lo < hi) {
    const int64_t mid = lo + (hi - lo + 1) / 2;
    if (make_layout(mid, Hkv, d, s, w, dtype).total <= ws_bytes)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Checks shared by every compute entry point; returns a dca_status.
int check_common(int64_t q_start, int64_t Lq, int64_t Lk, int Hq, int Hkv, int d, int64_t s,
                 int64_t w, int64_t c, double yarn_scale, int dtype, const void* ws,
                 size_t ws_bytes, Layout* layout) {
  if (!basic_params_ok(Hq, Hkv, d, s, w, c, dtype)) return DCA_ERR_ARG;
  if (q_start < 0 || Lq < 0 || Lk < 0 || q_start + Lq > Lk) return DCA_ERR_ARG;
  if (Lk > (1LL << 31) - 1) return DCA_ERR_ARG;
  if (Lk > s && s + w > c) return DCA_ERR_ARG;
  if (!(yarn_scale > 0.0) || !isfinite(yarn_scale)) return DCA_ERR_ARG;
  if (d != 128) return DCA_ERR_UNSUPPORTED;
  if (ws == nullptr || !aligned(ws, 256)) return DCA_ERR_WORKSPACE;
  const int64_t cap = capacity_for(ws_bytes, Hkv, d, s, w, dtype);
  if (cap < Lk) return DCA_ERR_WORKSPACE;
  *layout = make_layout(cap, Hkv, d, s, w, dtype);
  return DCA_OK;
}

float logit_scale_log2(double yarn_scale, int d) {
  const double m = yarn_scale <= 1.0 ? 1.0 : 0.1 * log(yarn_scale) + 1.0;
  return static_cast<float>(m * m / sqrt(static_cast<double>(d)) * 1.4426950408889634);
}

int prepare_impl(const void* k_cache, int64_t Lk, int64_t k_rows_valid, int Hkv, int d,
                 int64_t s, int64_t w, int64_t c, double rope_base, int dtype, void* ws,
                 const Layout& L, cudaStream_t st) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  float2* tab = reinterpret_cast<float2*>(base + L.tab_off);
  cudaError_t e = cudaSuccess;
  if (k_rows_valid == 0) e = dca::launch_rope_table(tab, L.T, L.n_direct, c, rope_base, d, st);
  if (e == cudaSuccess)
    e = dca::launch_rotate_keys(k_cache, base + L.kr_off, tab, k_rows_valid, Lk, Hkv, s, dtype,
                                st);
  return e == cudaSuccess ? DCA_OK : DCA_ERR_CUDA;
}

int attend_impl(const void* q, const void* v, void* out, int64_t q_start, int64_t Lq, int64_t Lk,
                int Hq, int Hkv, int d, int64_t s, int64_t w, double yarn_scale, int dtype,
                void* ws, const Layout& L, cudaStream_t st, int reading = 0) {
  if (Lq == 0) return DCA_OK;
  uint8_t* base = static_cast<uint8_t*>(ws);
  dca::AttnArgs a;
  a.q = q;
  a.kr = base + L.kr_off;
  a.v = v;
  a.out = out;
  a.tab = reinterpret_cast<const float2*>(base + L.tab_off);
  a.q_start = q_start;
  a.Lq = Lq;
  a.Lk = Lk;
  a.s = s;
  a.w = w;
  a.tab_c1 = L.T - 1;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.reading = reading;
  a.scale_log2 = logit_scale_log2(yarn_scale, d);
  a.status = reinterpret_cast<unsigned int*>(base);
  a.timeout_ns = static_cast<unsigned long long>(g_timeout_ns.load());
  a.debug = g_debug_flags.exchange(0);
  cudaError_t e = dtype == DCA_BF16 ? dca::launch_attention_sm100(a, st)
                                    : dca::launch_attention_f32(a, st);
  return e == cudaSuccess ? DCA_OK : DCA_ERR_CUDA;
}

bool ptrs_ok(const void* p) { return p != nullptr && aligned(p, 16); }

// One non-blocking copy stream per device for the host-buffer entry point,
// created on first use with that device current and kept until exit.
std::mutex g_copy_mu;
cudaStream_t g_copy_stream[64] = {};

int copy_stream_on_current_device(cudaStream_t* out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DCA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_copy_mu);
  if (g_copy_stream[dev] == nullptr &&
      cudaStreamCreateWithFlags(&g_copy_stream[dev], cudaStreamNonBlocking) != cudaSuccess) {
    g_copy_stream[dev] = nullptr;
    return DCA_ERR_CUDA;
  }
  *out = g_copy_stream[dev];
  return DCA_OK;
}

// Host-side checks of a one-shot or chunked prefill call (no device work).
int prefill_checks(const void* q, const void* k, const void* v, const void* out, int64_t q_start,
                   int64_t Lq, int64_t Lk, int Hq, int Hkv, int d, int64_t s, int64_t w,
                   int64_t c, double rope_base, double yarn_scale, int dtype, const void* ws,
                   size_t ws_bytes, Layout* L) {
  int rc = check_common(q_start, Lq, Lk, Hq, Hkv, d, s, w, c, yarn_scale, dtype, ws, ws_bytes, L);
  if (rc != DCA_OK) return rc;
  if (!(rope_base > 0.0) || !isfinite(rope_base)) return DCA_ERR_ARG;
  if (Lq == 0) return DCA_OK;
  if (!ptrs_ok(q) || !ptrs_ok(k) || !ptrs_ok(v) || !ptrs_ok(out)) return DCA_ERR_ARG;
  return DCA_OK;
}

// Scratch bytes of a decode call (0 for invalid sizes).
size_t decode_scratch_bytes(int64_t Lq, int Hq, int Hkv) {
  if (Lq < 1 || Lq > DCA_DECODE_MAX_TOKENS || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return 0;
  const int G = Hq / Hkv;
  const int n_rg = dca::decode_row_groups(Lq, G);
  const int n_cta = Hkv * n_rg * dca::decode_max_splits(Hkv, n_rg);
  return align_up(dca::decode_part_floats(n_cta, dca::decode_group_rows(Lq, G)) * sizeof(float),
                  256);
}

// Window reading from the options (NULL = defaults); -1 when invalid.
int reading_of(const dca_options* opts) {
  if (opts == nullptr) return DCA_WINDOW_QUERY_OFFSET;
  if (opts->window_reading != DCA_WINDOW_QUERY_OFFSET &&
      opts->window_reading != DCA_WINDOW_TRUE_DISTANCE)
    return -1;
  for (int k = 0; k < 7; ++k)
    if (opts->reserved[k] != 0) return -1;
  return opts->window_reading;
}

// Sparse workspace: the host-copied prefix (counts, runs, lists), the
// bitmaps, then the gathered vertical rows (1 KiB aligned for TMA).
struct SparseLayout {
  int64_t cap = 0, nv_cap = 0, s_cap = 0, wpr = 0;
  size_t nv_off = 0, ns_off = 0, nruns_off = 0, runs_off = 0, vidx_off = 0, soff_off = 0;
  size_t host_bytes = 0, vbit_off = 0, sbit_off = 0, gk_off = 0, gv_off = 0, total = 0;
};

bool sparse_cfg_ok(const dca_sparse_config* cfg) {
  return cfg != nullptr && cfg->kv_capacity >= 1 && cfg->kv_capacity <= (1LL << 31) - 1 &&
         cfg->max_vertical >= 0 && cfg->max_vertical <= (1LL << 31) - 1 && cfg->max_slash >= 0 &&
         cfg->max_slash <= (1LL << 31) - 1;
}

SparseLayout make_sparse_layout(const dca_sparse_config* cfg, int Hq) {
  SparseLayout S;
  S.cap = cfg->kv_capacity;
  S.nv_cap = (cfg->max_vertical + 127) / 128 * 128;
  if (S.nv_cap < 128) S.nv_cap = 128;
  S.s_cap = cfg->max_slash > 0 ? cfg->max_slash : 1;
  S.wpr = S.cap / 32 + 8;  // bits 0 .. cap + 127 are readable (row padding)
  size_t o = 0;
  S.nv_off = o;
  o = align_up(o + sizeof(int32_t) * Hq, 256);
  S.ns_off = o;
  o = align_up(o + sizeof(int32_t) * Hq, 256);
  S.nruns_off = o;
  o = align_up(o + sizeof(int32_t) * Hq, 256);
  S.runs_off = o;
  o = align_up(o + sizeof(int2) * static_cast<size_t>(Hq) * dca::SPARSE_MAX_RUNS, 256);
  S.vidx_off = o;
  o = align_up(o + sizeof(int32_t) * static_cast<size_t>(Hq) * S.nv_cap, 256);
  S.soff_off = o;
  o = align_up(o + sizeof(int32_t) * static_cast<size_t>(Hq) * S.s_cap, 256);
  S.host_bytes = o;
  S.vbit_off = o;
  o = align_up(o + sizeof(uint32_t) * static_cast<size_t>(Hq) * S.wpr, 256);
  S.sbit_off = o;
  o = align_up(o + sizeof(uint32_t) * static_cast<size_t>(Hq) * S.wpr, 1024);
  S.gk_off = o;
  o = align_up(o + static_cast<size_t>(S.nv_cap) * Hq * 128 * 2, 1024);
  S.gv_off = o;
  o = align_up(o + static_cast<size_t>(S.nv_cap) * Hq * 128 * 2, 1024);
  S.total = o;
  return S;
}

dca::SparseArgs sparse_args(const SparseLayout& S, const void* sws) {
  const uint8_t* b = static_cast<const uint8_t*>(sws);
  dca::SparseArgs a;
  a.vidx = reinterpret_cast<const int32_t*>(b + S.vidx_off);
  a.nv = reinterpret_cast<const int32_t*>(b + S.nv_off);
  a.runs = reinterpret_cast<const int2*>(b + S.runs_off);
  a.nruns = reinterpret_cast<const int32_t*>(b + S.nruns_off);
  a.vbit = reinterpret_cast<const uint32_t*>(b + S.vbit_off);
  a.sbit = reinterpret_cast<const uint32_t*>(b + S.sbit_off);
  a.gk = b + S.gk_off;
  a.gv = b + S.gv_off;
  a.wpr = S.wpr;
  a.nv_cap = S.nv_cap;
  return a;
}

// Checks one head's list: sorted, no repeats, inside [0, Lk); returns its
// number of runs of consecutive values, or -1.
int64_t list_runs(const int32_t* a, int64_t n, int64_t Lk) {
  int64_t runs = 0;
  for (int64_t e = 0; e < n; ++e) {
    if (a[e] < 0 || a[e] >= Lk) return -1;
    if (e > 0 && a[e] <= a[e - 1]) return -1;
    if (e == 0 || a[e] != a[e - 1] + 1) ++runs;
  }
  return runs;
}

}  // namespace

namespace dca {
int check_prefill_args(const void* q, const void* k, const void* v, const void* out, int64_t L,
                       int Hq, int Hkv, int d, int64_t s, int64_t w, int64_t c, double rope_base,
                       double yarn_scale, int dtype, const void* ws, size_t ws_bytes) {
  Layout lay;
  return prefill_checks(q, k, v, out, 0, L, L, Hq, Hkv, d, s, w, c, rope_base, yarn_scale, dtype,
                        ws, ws_bytes, &lay);
}
}  // namespace dca

extern "C" {

int dca_version(void) { return VERSION; }

const char* dca_status_string(int status) {
  switch (status) {
    case DCA_OK: return "DCA_OK";
    case DCA_ERR_ARG: return "DCA_ERR_ARG: invalid size, pointer, alignment or parameter";
    case DCA_ERR_UNSUPPORTED: return "DCA_ERR_UNSUPPORTED: head dim must be 128";
    case DCA_ERR_CUDA: return "DCA_ERR_CUDA: a CUDA call failed";
    case DCA_ERR_WORKSPACE: return "DCA_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case DCA_ERR_TIMEOUT: return "DCA_ERR_TIMEOUT: a kernel gave up on a bounded wait";
    default: return "unknown dca status";
  }
}

size_t dca_workspace_size(int64_t kv_capacity, int Hq, int Hkv, int d, int64_t chunk_size,
                          int64_t local_window, int64_t pretrain_window, int dtype) {
  if (!basic_params_ok(Hq, Hkv, d, chunk_size, local_window, pretrain_window, dtype)) return 0;
  if (kv_capacity < 0 || kv_capacity > (1LL << 31) - 1) return 0;
  return make_layout(kv_capacity, Hkv, d, chunk_size, local_window, dtype).total;
}

int dca_workspace_init(void* workspace, size_t ws_bytes, void* cuda_stream) {
  if (workspace == nullptr || ws_bytes < HDR_BYTES || !aligned(workspace, 256))
    return DCA_ERR_WORKSPACE;
  return cudaMemsetAsync(workspace, 0, HDR_BYTES, static_cast<cudaStream_t>(cuda_stream)) ==
                 cudaSuccess
             ? DCA_OK
             : DCA_ERR_CUDA;
}

int dca_prepare(const void* k_cache, int64_t Lk, int64_t k_rows_valid, int Hkv, int d,
                int64_t chunk_size, int64_t local_window, int64_t pretrain_window,
                double rope_base, int dtype, void* workspace, size_t ws_bytes,
                void* cuda_stream) {
  Layout L;
  int rc = check_common(0, 0, Lk, Hkv, Hkv, d, chunk_size, local_window, pretrain_window, 1.0,
                        dtype, workspace, ws_bytes, &L);
  if (rc != DCA_OK) return rc;
  if (!(rope_base > 0.0) || !isfinite(rope_base)) return DCA_ERR_ARG;
  if (k_rows_valid < 0 || k_rows_valid > Lk) return DCA_ERR_ARG;
  if (Lk > k_rows_valid && !ptrs_ok(k_cache)) return DCA_ERR_ARG;
  return prepare_impl(k_cache, Lk, k_rows_valid, Hkv, d, chunk_size, local_window,
                      pretrain_window, rope_base, dtype, workspace, L,
                      static_cast<cudaStream_t>(cuda_stream));
}

int dca_attend(const void* q_block, const void* v_cache, void* out_block, int64_t q_start,
               int64_t Lq, int64_t Lk, int Hq, int Hkv, int d, int64_t chunk_size,
               int64_t local_window, int64_t pretrain_window, double yarn_scale, int dtype,
               void* workspace, size_t ws_bytes, void* cuda_stream) {
  return dca_attend_ex(q_block, v_cache, out_block, q_start, Lq, Lk, Hq, Hkv, d, chunk_size,
                       local_window, pretrain_window, yarn_scale, dtype, nullptr, workspace,
                       ws_bytes, cuda_stream);
}

int dca_attend_ex(const void* q_block, const void* v_cache, void* out_block, int64_t q_start,
                  int64_t Lq, int64_t Lk, int Hq, int Hkv, int d, int64_t chunk_size,
                  int64_t local_window, int64_t pretrain_window, double yarn_scale, int dtype,
                  const dca_options* opts, void* workspace, size_t ws_bytes, void* cuda_stream) {
  const int reading = reading_of(opts);
  if (reading < 0) return DCA_ERR_ARG;
  Layout L;
  int rc = check_common(q_start, Lq, Lk, Hq, Hkv, d, chunk_size, local_window, pretrain_window,
                        yarn_scale, dtype, workspace, ws_bytes, &L);
  if (rc != DCA_OK) return rc;
  if (Lq > 0 && (!ptrs_ok(q_block) || !ptrs_ok(v_cache) || !ptrs_ok(out_block)))
    return DCA_ERR_ARG;
  return attend_impl(q_block, v_cache, out_block, q_start, Lq, Lk, Hq, Hkv, d, chunk_size,
                     local_window, yarn_scale, dtype, workspace, L,
                     static_cast<cudaStream_t>(cuda_stream), reading);
}

size_t dca_decode_scratch_size(int64_t Lq, int Hq, int Hkv) {
  return decode_scratch_bytes(Lq, Hq, Hkv);
}

int dca_decode(const void* q_block, const void* v_cache, void* out_block, float* lse,
               int64_t q_start, int64_t Lq, int64_t Lk, int Hq, int Hkv, int d,
               int64_t chunk_size, int64_t local_window, int64_t pretrain_window,
               double yarn_scale, int dtype, const dca_options* opts, void* workspace,
               size_t ws_bytes, void* scratch, size_t scratch_bytes, void* cuda_stream) {
  const int reading = reading_of(opts);
  if (reading < 0) return DCA_ERR_ARG;
  Layout L;
  int rc = check_common(q_start, Lq, Lk, Hq, Hkv, d, chunk_size, local_window, pretrain_window,
                        yarn_scale, dtype, workspace, ws_bytes, &L);
  if (rc != DCA_OK) return rc;
  if (Lq == 0) return DCA_OK;
  if (Lq > DCA_DECODE_MAX_TOKENS) return DCA_ERR_ARG;
  if (!ptrs_ok(q_block) || !ptrs_ok(v_cache) || !ptrs_ok(out_block)) return DCA_ERR_ARG;
  if (lse != nullptr && !aligned(lse, 4)) return DCA_ERR_ARG;
  if (!ptrs_ok(scratch) || scratch_bytes < decode_scratch_bytes(Lq, Hq, Hkv)) return DCA_ERR_ARG;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  dca::AttnArgs a;
  a.q = q_block;
  a.kr = base + L.kr_off;
  a.v = v_cache;
  a.out = out_block;
  a.tab = reinterpret_cast<const float2*>(base + L.tab_off);
  a.q_start = q_start;
  a.Lq = Lq;
  a.Lk = Lk;
  a.s = chunk_size;
  a.w = local_window;
  a.tab_c1 = L.T - 1;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.reading = reading;
  a.scale_log2 = logit_scale_log2(yarn_scale, d);
  a.status = reinterpret_cast<unsigned int*>(base);
  a.timeout_ns = static_cast<unsigned long long>(g_timeout_ns.load());
  a.debug = g_debug_flags.exchange(0);
  a.lse = lse;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e = dtype == DCA_BF16 ? dca::launch_decode_sm100(a, static_cast<float*>(scratch), st)
                                    : dca::launch_attention_f32(a, st);
  return e == cudaSuccess ? DCA_OK : DCA_ERR_CUDA;
}

int dca_prefill_chunked(const void* q_block, const void* k_cache, const void* v_cache,
                        void* out_block, int64_t q_start, int64_t Lq, int64_t Lk, int Hq,
                        int Hkv, int d, int64_t chunk_size, int64_t local_window,
                        int64_t pretrain_window, double rope_base, double yarn_scale,
                        int dtype, void* workspace, size_t ws_bytes, void* cuda_stream) {
  return dca_prefill_chunked_ex(q_block, k_cache, v_cache, out_block, q_start, Lq, Lk, Hq, Hkv,
                                d, chunk_size, local_window, pretrain_window, rope_base,
                                yarn_scale, dtype, nullptr, workspace, ws_bytes, cuda_stream);
}

int dca_prefill_chunked_ex(const void* q_block, const void* k_cache, const void* v_cache,
                           void* out_block, int64_t q_start, int64_t Lq, int64_t Lk, int Hq,
                           int Hkv, int d, int64_t chunk_size, int64_t local_window,
                           int64_t pretrain_window, double rope_base, double yarn_scale,
                           int dtype, const dca_options* opts, void* workspace, size_t ws_bytes,
                           void* cuda_stream) {
  const int reading = reading_of(opts);
  if (reading < 0) return DCA_ERR_ARG;
  Layout L;
  int rc = prefill_checks(q_block, k_cache, v_cache, out_block, q_start, Lq, Lk, Hq, Hkv, d,
                          chunk_size, local_window, pretrain_window, rope_base, yarn_scale, dtype,
                          workspace, ws_bytes, &L);
  if (rc != DCA_OK || Lq == 0) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  rc = prepare_impl(k_cache, Lk, 0, Hkv, d, chunk_size, local_window, pretrain_window, rope_base,
                    dtype, workspace, L, st);
  if (rc != DCA_OK) return rc;
  return attend_impl(q_block, v_cache, out_block, q_start, Lq, Lk, Hq, Hkv, d, chunk_size,
                     local_window, yarn_scale, dtype, workspace, L, st, reading);
}

int dca_prefill(const void* q, const void* k, const void* v, void* out, int64_t L, int Hq,
                int Hkv, int d, int64_t chunk_size, int64_t local_window,
                int64_t pretrain_window, double rope_base, double yarn_scale, int dtype,
                void* workspace, size_t ws_bytes, void* cuda_stream) {
  return dca_prefill_chunked(q, k, v, out, 0, L, L, Hq, Hkv, d, chunk_size, local_window,
                             pretrain_window, rope_base, yarn_scale, dtype, workspace, ws_bytes,
                             cuda_stream);
}

int dca_device_status(void* workspace, void* cuda_stream) {
  if (workspace == nullptr) return DCA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DCA_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpy(&word, workspace, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess)
    return DCA_ERR_CUDA;
  if (word != 0) {
    if (cudaMemset(workspace, 0, sizeof word) != cudaSuccess) return DCA_ERR_CUDA;
    return DCA_ERR_TIMEOUT;
  }
  return DCA_OK;
}

size_t dca_host_arena_size(int64_t L, int64_t block, int Hq, int Hkv, int d, int64_t chunk_size,
                           int64_t local_window, int64_t pretrain_window, int dtype) {
  const size_t ws = dca_workspace_size(L, Hq, Hkv, d, chunk_size, local_window, pretrain_window,
                                       dtype);
  if (ws == 0 || L < 0) return 0;
  const int64_t blk = (block <= 0 || block > L) ? L : block;
  const size_t esize = dtype == DCA_BF16 ? 2 : 4;
  const size_t kv = align_up(static_cast<size_t>(L) * Hkv * d * esize, 1024);
  const size_t qo = align_up(static_cast<size_t>(blk) * Hq * d * esize, 1024);
  return align_up(ws, 1024) + 2 * kv + 4 * qo;  // two query and two output block buffers
}

int dca_prefill_host(const void* q_h, const void* k_h, const void* v_h, void* out_h, int64_t L,
                     int64_t block, int Hq, int Hkv, int d, int64_t chunk_size,
                     int64_t local_window, int64_t pretrain_window, double rope_base,
                     double yarn_scale, int dtype, void* arena, size_t arena_bytes,
                     void* cuda_stream) {
  if (q_h == nullptr || k_h == nullptr || v_h == nullptr || out_h == nullptr) return DCA_ERR_ARG;
  const size_t need = dca_host_arena_size(L, block, Hq, Hkv, d, chunk_size, local_window,
                                          pretrain_window, dtype);
  if (need == 0) return DCA_ERR_ARG;
  if (arena == nullptr || !aligned(arena, 256) || arena_bytes < need) return DCA_ERR_WORKSPACE;
  if (L == 0) return DCA_OK;
  const int64_t blk = (block <= 0 || block > L) ? L : block;
  const size_t esize = dtype == DCA_BF16 ? 2 : 4;
  const size_t ws_bytes =
      dca_workspace_size(L, Hq, Hkv, d, chunk_size, local_window, pretrain_window, dtype);
  const size_t kv = align_up(static_cast<size_t>(L) * Hkv * d * esize, 1024);
  const size_t qo = align_up(static_cast<size_t>(blk) * Hq * d * esize, 1024);
  uint8_t* base = static_cast<uint8_t*>(arena);
  uint8_t* ws = base;
  uint8_t* kc = base + align_up(ws_bytes, 1024);
  uint8_t* vc = kc + kv;
  uint8_t* qb[2] = {vc + kv, vc + kv + qo};
  uint8_t* ob[2] = {vc + kv + 2 * qo, vc + kv + 3 * qo};
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaStream_t cs = nullptr;
  if (copy_stream_on_current_device(&cs) != DCA_OK) return DCA_ERR_CUDA;
  // events: start (caller's stream), inputs of a block landed (copy stream),
  // a block's attention done (caller's stream), last copy done (copy stream)
  cudaEvent_t ev_start = nullptr, ev_done = nullptr, ev_in[2] = {}, ev_out[2] = {};
  auto destroy_events = [&]() {
    for (cudaEvent_t e : {ev_start, ev_done, ev_in[0], ev_in[1], ev_out[0], ev_out[1]})
      if (e != nullptr) cudaEventDestroy(e);
  };
  for (cudaEvent_t* e : {&ev_start, &ev_done, &ev_in[0], &ev_in[1], &ev_out[0], &ev_out[1]})
    if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) {
      destroy_events();
      return DCA_ERR_CUDA;
    }
  const size_t krow = static_cast<size_t>(Hkv) * d * esize;
  const size_t qrow = static_cast<size_t>(Hq) * d * esize;
  const int64_t nb = (L + blk - 1) / blk;
  // host -> device copies of block b's key/value rows and query rows (copy stream)
  auto copy_in = [&](int64_t b) {
    const int64_t q0 = b * blk, lq = (L - q0 < blk) ? L - q0 : blk;
    return cudaMemcpyAsync(kc + q0 * krow, static_cast<const uint8_t*>(k_h) + q0 * krow,
                           lq * krow, cudaMemcpyHostToDevice, cs) == cudaSuccess &&
           cudaMemcpyAsync(vc + q0 * krow, static_cast<const uint8_t*>(v_h) + q0 * krow,
                           lq * krow, cudaMemcpyHostToDevice, cs) == cudaSuccess &&
           cudaMemcpyAsync(qb[b & 1], static_cast<const uint8_t*>(q_h) + q0 * qrow, lq * qrow,
                           cudaMemcpyHostToDevice, cs) == cudaSuccess &&
           cudaEventRecord(ev_in[b & 1], cs) == cudaSuccess;
  };
  int rc = dca_workspace_init(ws, ws_bytes, cuda_stream);
  bool ok = rc == DCA_OK && cudaEventRecord(ev_start, st) == cudaSuccess &&
            cudaStreamWaitEvent(cs, ev_start, 0) == cudaSuccess && copy_in(0);
  if (rc == DCA_OK && !ok) rc = DCA_ERR_CUDA;
  // Copy-stream order: in(0) | in(1), out(0) | in(2), out(1) | ...  The inputs
  // of block b + 1 land while block b is attended; in(b + 2) follows out(b),
  // which waits for block b's attention, so query buffer b & 1 is free again,
  // and block b + 2's attention waits for in(b + 2), so output buffer b & 1
  // has been copied out.  Key/value rows of later blocks are not read by
  // earlier blocks.
  for (int64_t b = 0; b < nb && rc == DCA_OK; ++b) {
    const int64_t q0 = b * blk, lq = (L - q0 < blk) ? L - q0 : blk, lk = q0 + lq;
    if (cudaStreamWaitEvent(st, ev_in[b & 1], 0) != cudaSuccess) {
      rc = DCA_ERR_CUDA;
      break;
    }
    // the rotated-key cache keeps rows [0, q0) from earlier blocks
    rc = dca_prepare(kc, lk, q0, Hkv, d, chunk_size, local_window, pretrain_window, rope_base,
                     dtype, ws, ws_bytes, cuda_stream);
    if (rc != DCA_OK) break;
    rc = dca_attend(qb[b & 1], vc, ob[b & 1], q0, lq, lk, Hq, Hkv, d, chunk_size, local_window,
                    pretrain_window, yarn_scale, dtype, ws, ws_bytes, cuda_stream);
    if (rc != DCA_OK) break;
    if (cudaEventRecord(ev_out[b & 1], st) != cudaSuccess || (b + 1 < nb && !copy_in(b + 1)) ||
        cudaStreamWaitEvent(cs, ev_out[b & 1], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint8_t*>(out_h) + q0 * qrow, ob[b & 1], lq * qrow,
                        cudaMemcpyDeviceToHost, cs) != cudaSuccess)
      rc = DCA_ERR_CUDA;
  }
  // the caller's stream covers every copy: synchronising it (or
  // dca_device_status) makes out_h readable
  if (cudaEventRecord(ev_done, cs) != cudaSuccess ||
      cudaStreamWaitEvent(st, ev_done, 0) != cudaSuccess)
    rc = DCA_ERR_CUDA;
  destroy_events();
  return rc;
}

int dca_plan_items(int64_t i0, int64_t i_last, int64_t tile_rows, int64_t chunk_size,
                   int64_t local_window, int window_reading, int bn, int32_t* items,
                   int max_items) {
  if (i0 < 0 || i_last < i0 || tile_rows < 1 || i_last >= i0 + tile_rows || chunk_size < 1 ||
      local_window < 0 || local_window > chunk_size || bn < 1 || max_items < 0 ||
      (max_items > 0 && items == nullptr) ||
      (window_reading != DCA_WINDOW_QUERY_OFFSET && window_reading != DCA_WINDOW_TRUE_DISTANCE))
    return DCA_ERR_ARG;
  const int64_t w = local_window;
  const int rd = window_reading;
  const dca::TilePlan P = dca::make_plan(i0, i_last, chunk_size, w, bn, rd);
  const dca::FullRanges F = dca::make_full_ranges(i0, i0 + tile_rows - 1, chunk_size, w, bn, rd);
  for (int n = 0; n < P.n_items && n < max_items; ++n) {
    int kt, cls;
    dca::plan_item(P, n, kt, cls);
    const int64_t j0 = static_cast<int64_t>(kt) * bn;
    const bool full =
        dca::item_is_full(i0, i0 + tile_rows - 1, j0, j0 + bn - 1, chunk_size, w, cls, rd);
    // the kernels use the precomputed ranges; they must agree with the predicate
    if (full != dca::is_full(F, kt, cls)) return DCA_ERR_ARG - 100;
    items[3 * n + 0] = kt;
    items[3 * n + 1] = cls;
    items[3 * n + 2] = full ? 1 : 0;
  }
  return P.n_items;
}

void dca_set_wait_timeout_ns(int64_t ns) {
  g_timeout_ns.store(ns > 0 ? ns : 10LL * 1000 * 1000 * 1000);
}

void dca_set_debug_flags(int flags) { g_debug_flags.store(flags); }

size_t dca_sparse_workspace_size(const dca_sparse_config* cfg, int Hq) {
  if (!sparse_cfg_ok(cfg) || Hq <= 0) return 0;
  return make_sparse_layout(cfg, Hq).total;
}

int dca_sparse_prepare(const dca_sparse_config* cfg, const int64_t* v_ptr, const int32_t* v_idx,
                       const int64_t* s_ptr, const int32_t* s_off, int64_t Lk, int Hq, int Hkv,
                       int d, int64_t chunk_size, int64_t local_window, int64_t pretrain_window,
                       int dtype, const void* v_cache, const void* workspace, size_t ws_bytes,
                       void* sparse_ws, size_t sparse_bytes, void* cuda_stream) {
  if (!sparse_cfg_ok(cfg) || v_ptr == nullptr || s_ptr == nullptr) return DCA_ERR_ARG;
  if (dtype == DCA_F32) return DCA_ERR_UNSUPPORTED;  // the sparse path is bf16
  // the dense workspace holds the rotated keys [0, Lk)
  Layout L;
  int rc = check_common(0, 0, Lk, Hq, Hkv, d, chunk_size, local_window, pretrain_window, 1.0,
                        dtype, workspace, ws_bytes, &L);
  if (rc != DCA_OK) return rc;
  if (dtype != DCA_BF16) return DCA_ERR_UNSUPPORTED;
  if (Lk < 1 || Lk > cfg->kv_capacity || !ptrs_ok(v_cache)) return DCA_ERR_ARG;
  if (sparse_ws == nullptr || !aligned(sparse_ws, 1024)) return DCA_ERR_WORKSPACE;
  const SparseLayout S = make_sparse_layout(cfg, Hq);
  if (sparse_bytes < S.total) return DCA_ERR_WORKSPACE;
  // host-side pattern checks and the copied prefix
  std::vector<uint8_t> blob(S.host_bytes, 0);
  int32_t* nv = reinterpret_cast<int32_t*>(blob.data() + S.nv_off);
  int32_t* ns = reinterpret_cast<int32_t*>(blob.data() + S.ns_off);
  int32_t* nr = reinterpret_cast<int32_t*>(blob.data() + S.nruns_off);
  int2* runs = reinterpret_cast<int2*>(blob.data() + S.runs_off);
  int32_t* vi = reinterpret_cast<int32_t*>(blob.data() + S.vidx_off);
  int32_t* so = reinterpret_cast<int32_t*>(blob.data() + S.soff_off);
  if (v_ptr[0] != 0 || s_ptr[0] != 0) return DCA_ERR_ARG;
  for (int h = 0; h < Hq; ++h) {
    const int64_t n_v = v_ptr[h + 1] - v_ptr[h], n_s = s_ptr[h + 1] - s_ptr[h];
    if (n_v < 0 || n_v > cfg->max_vertical || n_s < 0 || n_s > cfg->max_slash) return DCA_ERR_ARG;
    if ((n_v > 0 && v_idx == nullptr) || (n_s > 0 && s_off == nullptr)) return DCA_ERR_ARG;
    if (n_v > 0 && list_runs(v_idx + v_ptr[h], n_v, Lk) < 0) return DCA_ERR_ARG;
    const int64_t r = n_s > 0 ? list_runs(s_off + s_ptr[h], n_s, Lk) : 0;
    if (r < 0 || r > dca::SPARSE_MAX_RUNS) return DCA_ERR_ARG;
    nv[h] = static_cast<int32_t>(n_v);
    ns[h] = static_cast<int32_t>(n_s);
    nr[h] = static_cast<int32_t>(r);
    for (int64_t e = 0; e < n_v; ++e) vi[h * S.nv_cap + e] = v_idx[v_ptr[h] + e];
    int k = -1;
    for (int64_t e = 0; e < n_s; ++e) {
      const int32_t o = s_off[s_ptr[h] + e];
      so[h * S.s_cap + e] = o;
      if (e == 0 || o != s_off[s_ptr[h] + e - 1] + 1)
        runs[h * dca::SPARSE_MAX_RUNS + (++k)] = make_int2(o, o + 1);
      else
        runs[h * dca::SPARSE_MAX_RUNS + k].y = o + 1;
    }
  }
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  uint8_t* sb = static_cast<uint8_t*>(sparse_ws);
  if (cudaMemcpyAsync(sb, blob.data(), S.host_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return DCA_ERR_CUDA;
  if (cudaMemsetAsync(sb + S.vbit_off, 0, S.gk_off - S.vbit_off, st) != cudaSuccess)
    return DCA_ERR_CUDA;
  const dca::SparseArgs a = sparse_args(S, sparse_ws);
  cudaError_t e = dca::launch_sparse_bits(a.vidx, a.nv, S.nv_cap,
                                          reinterpret_cast<const int32_t*>(sb + S.soff_off),
                                          reinterpret_cast<const int32_t*>(sb + S.ns_off), S.s_cap,
                                          reinterpret_cast<uint32_t*>(sb + S.vbit_off),
                                          reinterpret_cast<uint32_t*>(sb + S.sbit_off), S.wpr, Hq,
                                          st);
  if (e == cudaSuccess) {
    const uint8_t* wb = static_cast<const uint8_t*>(workspace);
    e = dca::launch_sparse_gather(a.vidx, a.nv, S.nv_cap, wb + L.kr_off, v_cache, sb + S.gk_off,
                                  sb + S.gv_off, Hq, Hkv, st);
  }
  return e == cudaSuccess ? DCA_OK : DCA_ERR_CUDA;
}

int dca_sparse_attend(const dca_sparse_config* cfg, const void* q_block, const void* v_cache,
                      void* out_block, int64_t q_start, int64_t Lq, int64_t Lk, int Hq, int Hkv,
                      int d, int64_t chunk_size, int64_t local_window, int64_t pretrain_window,
                      double yarn_scale, int dtype, const dca_options* opts, void* workspace,
                      size_t ws_bytes, const void* sparse_ws, size_t sparse_bytes,
                      void* cuda_stream) {
  const int reading = reading_of(opts);
  if (reading < 0 || !sparse_cfg_ok(cfg)) return DCA_ERR_ARG;
  if (dtype == DCA_F32) return DCA_ERR_UNSUPPORTED;  // the sparse path is bf16
  Layout L;
  int rc = check_common(q_start, Lq, Lk, Hq, Hkv, d, chunk_size, local_window, pretrain_window,
                        yarn_scale, dtype, workspace, ws_bytes, &L);
  if (rc != DCA_OK) return rc;
  if (dtype != DCA_BF16) return DCA_ERR_UNSUPPORTED;
  if (Lk > cfg->kv_capacity) return DCA_ERR_ARG;
  if (sparse_ws == nullptr || !aligned(sparse_ws, 1024)) return DCA_ERR_WORKSPACE;
  const SparseLayout S = make_sparse_layout(cfg, Hq);
  if (sparse_bytes < S.total) return DCA_ERR_WORKSPACE;
  if (Lq == 0) return DCA_OK;
  if (!ptrs_ok(q_block) || !ptrs_ok(v_cache) || !ptrs_ok(out_block)) return DCA_ERR_ARG;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  dca::AttnArgs a;
  a.q = q_block;
  a.kr = base + L.kr_off;
  a.v = v_cache;
  a.out = out_block;
  a.tab = reinterpret_cast<const float2*>(base + L.tab_off);
  a.q_start = q_start;
  a.Lq = Lq;
  a.Lk = Lk;
  a.s = chunk_size;
  a.w = local_window;
  a.tab_c1 = L.T - 1;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.reading = reading;
  a.scale_log2 = logit_scale_log2(yarn_scale, d);
  a.status = reinterpret_cast<unsigned int*>(base);
  a.timeout_ns = static_cast<unsigned long long>(g_timeout_ns.load());
  a.debug = g_debug_flags.exchange(0);
  const cudaError_t e = dca::launch_sparse_sm100(a, sparse_args(S, sparse_ws),
                                                 static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? DCA_OK : DCA_ERR_CUDA;
}

int dca_class_rows(int64_t j, int64_t i_first, int n_rows, int64_t kv_len, int64_t chunk_size,
                   int64_t local_window, int window_reading, int cls, int64_t chunk,
                   int32_t* range) {
  if (j < 0 || j > (1LL << 31) - 1 || i_first < 0 || n_rows < 1 || n_rows > 64 ||
      chunk_size < 1 || local_window < 0 || local_window > chunk_size || cls < -1 || cls > 2 ||
      range == nullptr ||
      (window_reading != DCA_WINDOW_QUERY_OFFSET && window_reading != DCA_WINDOW_TRUE_DISTANCE))
    return DCA_ERR_ARG;
  int ra, rb;
  dca::class_row_range(j, i_first, n_rows, kv_len, chunk_size, local_window, window_reading, cls,
                       chunk, &ra, &rb);
  range[0] = ra;
  range[1] = rb;
  return DCA_OK;
}

int dca_row_keys(int64_t i, int cls, int64_t chunk_size, int64_t local_window, int window_reading,
                 int64_t* range) {
  if (i < 0 || i > (1LL << 31) - 2 || cls < 0 || cls > 2 || chunk_size < 1 || local_window < 0 ||
      local_window > chunk_size || range == nullptr ||
      (window_reading != DCA_WINDOW_QUERY_OFFSET && window_reading != DCA_WINDOW_TRUE_DISTANCE))
    return DCA_ERR_ARG;
  // the kernel's 32-bit form: chunk size and window clamped to 2^31 - 1
  const int s32 = chunk_size < 0x7fffffff ? static_cast<int>(chunk_size) : 0x7fffffff;
  const int w32 = local_window < 0x7fffffff ? static_cast<int>(local_window) : 0x7fffffff;
  int lo, hi;
  dca::row_key_range<int>(static_cast<int>(i), cls, s32, w32, window_reading, lo, hi);
  range[0] = lo;
  range[1] = hi;
  return DCA_OK;
}

int dca_sparse_plan_items(const int32_t* v_idx, int64_t n_v, const int32_t* s_off, int64_t n_s,
                          int64_t i0, int64_t i_last, int64_t chunk_size, int64_t local_window,
                          int window_reading, int32_t* items, int max_items) {
  if (chunk_size < 1 || local_window < 0 || local_window > chunk_size) return DCA_ERR_ARG;
  if (window_reading != DCA_WINDOW_QUERY_OFFSET && window_reading != DCA_WINDOW_TRUE_DISTANCE)
    return DCA_ERR_ARG;
  if (i0 < 0 || i_last < i0 || i_last - i0 >= 128 || (i0 % 128) != 0) return DCA_ERR_ARG;
  if (n_v < 0 || n_s < 0 || (n_v > 0 && !v_idx) || (n_s > 0 && !s_off) || max_items < 0 ||
      (max_items > 0 && !items))
    return DCA_ERR_ARG;
  const int64_t lim = (1LL << 31) - 1;
  if ((n_v > 0 && list_runs(v_idx, n_v, lim) < 0)) return DCA_ERR_ARG;
  const int64_t nr = n_s > 0 ? list_runs(s_off, n_s, lim) : 0;
  if (nr < 0 || nr > dca::SPARSE_MAX_RUNS) return DCA_ERR_ARG;
  std::vector<int2> runs;
  for (int64_t e = 0; e < n_s; ++e) {
    if (e == 0 || s_off[e] != s_off[e - 1] + 1)
      runs.push_back(make_int2(s_off[e], s_off[e] + 1));
    else
      runs.back().y = s_off[e] + 1;
  }
  std::vector<dca::SparsePlan> P(1);
  dca::sparse_plan_build(P[0], v_idx, static_cast<int>(n_v), runs.data(), static_cast<int>(nr), i0,
                         i_last, chunk_size, local_window, window_reading, 128);
  dca::SparseIter it;
  dca::sparse_iter_init(it);
  int n = 0, src, start, cls;
  while (dca::sparse_iter_next(it, P[0], src, start, cls)) {
    if (n < max_items) {
      items[3 * n] = src;
      items[3 * n + 1] = start;
      items[3 * n + 2] = cls;
    }
    ++n;
  }
  // the kernels size their loops by the plan's count: it must match the list
  if (n != P[0].n_items) return DCA_ERR_UNSUPPORTED;
  return n;
}

size_t dca_sparse_select_scratch_size(int64_t Lk, int Hq, int64_t chunk_size) {
  if (Lk < 1 || Lk > (1LL << 31) - 1 || Hq <= 0 || chunk_size < 1) return 0;
  return dca::select_scratch_bytes(Lk, Hq, (Lk + chunk_size - 1) / chunk_size);
}

int dca_sparse_select(const dca_sparse_config* cfg, const void* q_block, const void* v_cache,
                      int64_t q_start, int64_t Lq, int64_t Lk, int Hq, int Hkv, int d,
                      int64_t chunk_size, int64_t local_window, int64_t pretrain_window,
                      double rope_base, double yarn_scale, int dtype, const dca_options* opts,
                      int n_last, int continuous_positions, int64_t n_vertical, int64_t n_slash,
                      void* workspace, size_t ws_bytes, void* sparse_ws, size_t sparse_bytes,
                      void* scratch, size_t scratch_bytes, void* cuda_stream) {
  const int reading = reading_of(opts);
  if (reading < 0 || !sparse_cfg_ok(cfg)) return DCA_ERR_ARG;
  if (dtype == DCA_F32) return DCA_ERR_UNSUPPORTED;  // the sparse path is bf16
  Layout L;
  int rc = check_common(q_start, Lq, Lk, Hq, Hkv, d, chunk_size, local_window, pretrain_window,
                        yarn_scale, dtype, workspace, ws_bytes, &L);
  if (rc != DCA_OK) return rc;
  if (dtype != DCA_BF16) return DCA_ERR_UNSUPPORTED;
  if (!(rope_base > 0.0) || !isfinite(rope_base)) return DCA_ERR_ARG;
  if (Lq < 1 || n_last < 1 || n_last > 64 || n_last > Lq || Lk > cfg->kv_capacity)
    return DCA_ERR_ARG;
  if (continuous_positions != 0 && continuous_positions != 1) return DCA_ERR_ARG;
  if (n_vertical < 0 || n_vertical > cfg->max_vertical || n_slash < 0 ||
      n_slash > cfg->max_slash || n_slash > dca::SPARSE_MAX_RUNS)
    return DCA_ERR_ARG;
  if (!ptrs_ok(q_block) || !ptrs_ok(v_cache)) return DCA_ERR_ARG;
  if (sparse_ws == nullptr || !aligned(sparse_ws, 1024)) return DCA_ERR_WORKSPACE;
  const SparseLayout S = make_sparse_layout(cfg, Hq);
  if (sparse_bytes < S.total) return DCA_ERR_WORKSPACE;
  const int64_t n_chunks = (Lk + chunk_size - 1) / chunk_size;
  if (scratch == nullptr || !aligned(scratch, 256) ||
      scratch_bytes < dca::select_scratch_bytes(Lk, Hq, n_chunks))
    return DCA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  uint8_t* sb = static_cast<uint8_t*>(sparse_ws);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  // the head's lists are rewritten; bitmaps start empty
  if (cudaMemsetAsync(sb + S.vbit_off, 0, S.gk_off - S.vbit_off, st) != cudaSuccess)
    return DCA_ERR_CUDA;
  dca::SelectArgs a;
  a.q = q_block;
  a.kr = base + L.kr_off;
  a.tab = reinterpret_cast<const float2*>(base + L.tab_off);
  a.scratch = scratch;
  a.q_start = q_start;
  a.Lq = Lq;
  a.Lk = Lk;
  a.s = chunk_size;
  a.w = local_window;
  a.tab_c1 = L.T - 1;
  a.n_chunks = n_chunks;
  a.n_v = n_vertical;
  a.n_s = n_slash;
  a.n_last = n_last;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.reading = reading;
  a.continuous = continuous_positions;
  a.rope_base = rope_base;
  a.scale_log2 = logit_scale_log2(yarn_scale, d);
  a.nv = reinterpret_cast<int32_t*>(sb + S.nv_off);
  a.ns = reinterpret_cast<int32_t*>(sb + S.ns_off);
  a.vidx = reinterpret_cast<int32_t*>(sb + S.vidx_off);
  a.soff = reinterpret_cast<int32_t*>(sb + S.soff_off);
  a.nruns = reinterpret_cast<int32_t*>(sb + S.nruns_off);
  a.runs = reinterpret_cast<int2*>(sb + S.runs_off);
  a.vbit = reinterpret_cast<uint32_t*>(sb + S.vbit_off);
  a.sbit = reinterpret_cast<uint32_t*>(sb + S.sbit_off);
  a.nv_cap = S.nv_cap;
  a.s_cap = S.s_cap;
  a.wpr = S.wpr;
  a.status = reinterpret_cast<unsigned int*>(base);
  a.timeout_ns = static_cast<unsigned long long>(g_timeout_ns.load());
  cudaError_t e = dca::launch_select(a, st);
  if (e == cudaSuccess) {
    const dca::SparseArgs sa = sparse_args(S, sparse_ws);
    e = dca::launch_sparse_gather(sa.vidx, sa.nv, S.nv_cap, base + L.kr_off, v_cache,
                                  sb + S.gk_off, sb + S.gv_off, Hq, Hkv, st);
  }
  return e == cudaSuccess ? DCA_OK : DCA_ERR_CUDA;
}

int dca_sparse_pattern_get(const dca_sparse_config* cfg, int Hq, const void* sparse_ws,
                           size_t sparse_bytes, int32_t* v_counts, int32_t* v_idx,
                           int32_t* s_counts, int32_t* s_off, void* cuda_stream) {
  if (!sparse_cfg_ok(cfg) || Hq <= 0 || !v_counts || !s_counts) return DCA_ERR_ARG;
  if ((cfg->max_vertical > 0 && !v_idx) || (cfg->max_slash > 0 && !s_off)) return DCA_ERR_ARG;
  if (sparse_ws == nullptr || !aligned(sparse_ws, 1024)) return DCA_ERR_WORKSPACE;
  const SparseLayout S = make_sparse_layout(cfg, Hq);
  if (sparse_bytes < S.total) return DCA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DCA_ERR_CUDA;
  std::vector<uint8_t> blob(S.host_bytes);
  if (cudaMemcpy(blob.data(), sparse_ws, S.host_bytes, cudaMemcpyDeviceToHost) != cudaSuccess)
    return DCA_ERR_CUDA;
  const int32_t* nv = reinterpret_cast<const int32_t*>(blob.data() + S.nv_off);
  const int32_t* ns = reinterpret_cast<const int32_t*>(blob.data() + S.ns_off);
  const int32_t* vi = reinterpret_cast<const int32_t*>(blob.data() + S.vidx_off);
  const int32_t* so = reinterpret_cast<const int32_t*>(blob.data() + S.soff_off);
  for (int h = 0; h < Hq; ++h) {
    v_counts[h] = nv[h];
    s_counts[h] = ns[h];
    for (int64_t e = 0; e < nv[h] && e < cfg->max_vertical; ++e)
      v_idx[h * cfg->max_vertical + e] = vi[h * S.nv_cap + e];
    for (int64_t e = 0; e < ns[h] && e < cfg->max_slash; ++e)
      s_off[h * cfg->max_slash + e] = so[h * S.s_cap + e];
  }
  return DCA_OK;
}

}  // extern "C"
