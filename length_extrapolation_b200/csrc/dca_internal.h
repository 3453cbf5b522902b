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
};

cudaError_t launch_rope_table(float2* tab, int64_t T, int64_t n_direct, int64_t c, double base,
                              int d, cudaStream_t st);
cudaError_t launch_rotate_keys(const void* k, void* kr, const float2* tab, int64_t j_begin,
                               int64_t j_end, int Hkv, int64_t s, int dtype, cudaStream_t st);

// bf16 tcgen05/TMA kernel; returns a CUDA error or cudaSuccess, or
// cudaErrorInvalidValue when a tensor map cannot be encoded.
cudaError_t launch_attention_sm100(const AttnArgs& a, cudaStream_t st);
// fp32 CUDA-core kernel.
cudaError_t launch_attention_f32(const AttnArgs& a, cudaStream_t st);

}  // namespace dca
