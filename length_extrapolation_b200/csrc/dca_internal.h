// dca_internal.h -- declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dca {

// Arguments of one attention launch (both kernels).
struct AttnArgs {
  const void* q;        // [Lq][Hq][128] query block
  const void* kr;       // rotated keys R(j mod s) k_j, [cap][Hkv][128] (workspace)
  const void* v;        // [Lk][Hkv][128]
  void* out;            // [Lq][Hq][128]
  const float2* tab;    // RoPE table [T][64] (cos, sin)
  int64_t q_start, Lq, Lk;
  int64_t s, w, tab_c1; // chunk size, local window, table row of position c-1
  int Hq, Hkv;
  int reading;          // window reading: 0 (r_i < w) or 1 (i - j < w)
  float scale_log2;     // m^2 / sqrt(d) * log2(e)
  unsigned int* status; // device status word (workspace header)
  unsigned long long timeout_ns;
  int debug;
  float* lse = nullptr;  // optional [Lq][Hq] natural-log LSE (fp32 kernel and decode only)
};

// Split-KV decode: a few query rows against a long cache.  CTAs per
// (KV head, row group, slice) and the partial-result scratch they write.
// A row group is 16 (token, head) rows when the query block has at most 16
// rows per KV head, otherwise 32 (the MMA N of the decode kernel).
constexpr int DECODE_MAX_CTAS = 148; // one CTA per SM of a B200
inline int decode_group_rows(int64_t Lq, int G) { return Lq * G <= 16 ? 16 : 32; }
inline int decode_row_groups(int64_t Lq, int G) {
  const int nr = decode_group_rows(Lq, G);
  return static_cast<int>((Lq * G + nr - 1) / nr);
}
inline int decode_max_splits(int Hkv, int n_rg) {
  const int per = DECODE_MAX_CTAS / (Hkv * n_rg);
  return per > 1 ? per : 1;
}
// fp32 words of partial results: O [cta][nr][128], then m, l [cta][nr].
inline size_t decode_part_floats(int n_cta, int nr) {
  return static_cast<size_t>(n_cta) * nr * (128 + 2);
}

cudaError_t launch_rope_table(float2* tab, int64_t T, int64_t n_direct, int64_t c, double base,
                              int d, cudaStream_t st);
cudaError_t launch_rotate_keys(const void* k, void* kr, const float2* tab, int64_t j_begin,
                               int64_t j_end, int Hkv, int64_t s, int dtype, cudaStream_t st);

// Tensor map of a [rows][Hkv][128] bf16 tensor for boxes of 64 dims x 1 head x
// 128 rows, 128-byte swizzle, rows >= n_rows read as zeros; false if the
// driver's encoder is unavailable or rejects the map.
bool encode_kv_map(CUtensorMap* m, const void* base, int64_t n_rows, int Hkv);

// Vertical-slash sparse attention: the index structures built by
// dca_sparse_prepare in the sparse workspace.
constexpr int SPARSE_MAX_RUNS = 1023;  // runs of consecutive slash offsets per head
struct SparseArgs {
  const int32_t* vidx;   // [Hq][nv_cap] sorted vertical keys
  const int32_t* nv;     // [Hq]
  const int2* runs;      // [Hq][SPARSE_MAX_RUNS] slash offset runs [x, y)
  const int32_t* nruns;  // [Hq]
  const uint32_t* vbit;  // [Hq][wpr]
  const uint32_t* sbit;  // [Hq][wpr]
  const void* gk;        // [nv_cap][Hq][128] gathered rotated keys
  const void* gv;        // [nv_cap][Hq][128] gathered values
  int64_t wpr, nv_cap;
};

// Key selection (scores of the last rows, top-k into the sparse workspace).
struct SelectArgs {
  const void* q;          // query block [Lq][Hq][128] bf16
  const void* kr;         // rotated keys [cap][Hkv][128] bf16
  const float2* tab;      // RoPE table
  void* scratch;          // select_scratch_bytes(Lk, Hq, n_chunks)
  int64_t q_start, Lq, Lk, s, w, tab_c1, n_chunks, n_v, n_s;
  int n_last, Hq, Hkv, reading, continuous;
  double rope_base;
  float scale_log2;
  // outputs in the sparse workspace (bitmaps zeroed before)
  int32_t *nv, *ns, *vidx, *soff, *nruns;
  int2* runs;
  uint32_t *vbit, *sbit;
  int64_t nv_cap, s_cap, wpr;
  unsigned int* status;   // device status word (timeouts of the score passes)
  unsigned long long timeout_ns;
};
size_t select_scratch_bytes(int64_t Lk, int Hq, int64_t n_chunks);
// Score passes of the selection (tcgen05).  Pass 1 writes per-slice row
// statistics `part` [Hq][select_stat_slices(Lk)][64] (max, sum); pass 2 reads
// the merged `stats` [Hq][64] and writes vert (stored, [Hq][Lk]) and slash
// (accumulated, [Hq][Lk]), in slices of select_slices(Lk).
cudaError_t launch_select_row_stats(const void* kr, const float* qv, const float2* crot,
                                    float2* part, int64_t i_first, int64_t Lk, int64_t s, int64_t w,
                                    int n_last, int Hq, int Hkv, int reading, int continuous,
                                    unsigned int* status, unsigned long long timeout_ns,
                                    cudaStream_t st);
int select_stat_slices(int64_t Lk);
cudaError_t launch_select_sums(const void* kr, const float* qv, const float2* crot,
                               const float2* stats, float* vert, float* slash, int64_t i_first,
                               int64_t Lk, int64_t s, int64_t w, int n_last, int Hq, int Hkv,
                               int reading, int continuous, unsigned int* status,
                               unsigned long long timeout_ns, cudaStream_t st);
int select_slices(int64_t Lk);
cudaError_t launch_select(const SelectArgs& sa, cudaStream_t st);

// Host-side argument checks of dca_prefill (no device work): the dca_status
// that dca_prefill would return before launching anything, or DCA_OK.
int check_prefill_args(const void* q, const void* k, const void* v, const void* out, int64_t L,
                       int Hq, int Hkv, int d, int64_t s, int64_t w, int64_t c, double rope_base,
                       double yarn_scale, int dtype, const void* ws, size_t ws_bytes);

// bf16 tcgen05/TMA kernel; returns a CUDA error or cudaSuccess, or
// cudaErrorInvalidValue when a tensor map cannot be encoded.
cudaError_t launch_attention_sm100(const AttnArgs& a, cudaStream_t st);
// fp32 CUDA-core kernel (writes a.lse when set).
cudaError_t launch_attention_f32(const AttnArgs& a, cudaStream_t st);
// bf16 split-KV decode (tcgen05) and the combine of its partial results into
// out (and a.lse when set); `part` holds decode_part_floats(...) words.
cudaError_t launch_decode_sm100(const AttnArgs& a, float* part, cudaStream_t st);
// Sparse attention kernel over the structures of `sa` (bf16).
cudaError_t launch_sparse_sm100(const AttnArgs& a, const SparseArgs& sa, cudaStream_t st);
// Preparation: membership bitmaps from the per-head lists (zeroed before),
// and the gathered vertical rows of the rotated keys and values.
cudaError_t launch_sparse_bits(const int32_t* vidx, const int32_t* nv, int64_t nv_cap,
                               const int32_t* soff, const int32_t* ns, int64_t s_cap,
                               uint32_t* vbit, uint32_t* sbit, int64_t wpr, int Hq,
                               cudaStream_t st);
cudaError_t launch_sparse_gather(const int32_t* vidx, const int32_t* nv, int64_t nv_cap,
                                 const void* kr, const void* v, void* gk, void* gv, int Hq,
                                 int Hkv, cudaStream_t st);

}  // namespace dca
