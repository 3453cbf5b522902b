// dca_sparse_prep.cu -- preparation of the vertical-slash sparse attention's
// index structures on the device (after the per-head lists were copied in):
//   - membership bitmaps: bit j of head h's vertical row when key j is a
//     vertical key, bit o of its slash row when offset o is a slash offset;
//   - the gathered vertical rows: the rotated keys R(j mod s) k_j and values
//     v_j of each head's vertical keys, in list order, in a compact
//     [nv_cap][Hq][128] array (rows past a head's count up to the next
//     128-row tile are zero, so masked scores meet finite values).
// Both are HBM-light: a few bytes per list entry and 512 bytes per vertical
// key and head.
#include <cuda_bf16.h>

#include "dca_internal.h"

namespace dca {
namespace {

// one thread per (head, list entry); bitmaps zeroed before
__global__ void sparse_bits_kernel(const int32_t* __restrict__ vidx, const int32_t* __restrict__ nv,
                                   int64_t nv_cap, const int32_t* __restrict__ soff,
                                   const int32_t* __restrict__ ns, int64_t s_cap,
                                   uint32_t* __restrict__ vbit, uint32_t* __restrict__ sbit,
                                   int64_t wpr, int Hq) {
  const int64_t per = nv_cap > s_cap ? nv_cap : s_cap;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= per * Hq) return;
  const int h = static_cast<int>(t / per);
  const int64_t e = t % per;
  if (e < nv[h]) {
    const int32_t j = vidx[h * nv_cap + e];
    atomicOr(&vbit[h * wpr + (j >> 5)], 1u << (j & 31));
  }
  if (e < ns[h]) {
    const int32_t o = soff[h * s_cap + e];
    atomicOr(&sbit[h * wpr + (o >> 5)], 1u << (o & 31));
  }
}

// one 16-thread group per (head, gathered row): 16 x 16 bytes of key and value
__global__ void sparse_gather_kernel(const int32_t* __restrict__ vidx,
                                     const int32_t* __restrict__ nv, int64_t nv_cap,
                                     const uint4* __restrict__ kr, const uint4* __restrict__ v,
                                     uint4* __restrict__ gk, uint4* __restrict__ gv, int Hq,
                                     int G, int Hkv) {
  const int64_t grp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  const int part = threadIdx.x & 15;
  if (grp >= nv_cap * Hq) return;
  const int h = static_cast<int>(grp % Hq);
  const int64_t e = grp / Hq;  // row of the gathered array (layout [nv_cap][Hq][128])
  const int n = nv[h];
  const int64_t pad_end = (static_cast<int64_t>(n) + 127) / 128 * 128;
  if (e >= pad_end) return;
  uint4 kk = make_uint4(0, 0, 0, 0), vv = kk;
  if (e < n) {
    const int64_t j = vidx[h * nv_cap + e];
    const int64_t src = (j * Hkv + h / G) * 16 + part;  // 16 uint4 per 128 bf16
    kk = kr[src];
    vv = v[src];
  }
  gk[grp * 16 + part] = kk;
  gv[grp * 16 + part] = vv;
}

}  // namespace

cudaError_t launch_sparse_bits(const int32_t* vidx, const int32_t* nv, int64_t nv_cap,
                               const int32_t* soff, const int32_t* ns, int64_t s_cap,
                               uint32_t* vbit, uint32_t* sbit, int64_t wpr, int Hq,
                               cudaStream_t st) {
  const int64_t per = nv_cap > s_cap ? nv_cap : s_cap;
  const int64_t n = per * Hq;
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = (n + 255) / 256;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  sparse_bits_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(vidx, nv, nv_cap, soff, ns,
                                                                     s_cap, vbit, sbit, wpr, Hq);
  return cudaGetLastError();
}

cudaError_t launch_sparse_gather(const int32_t* vidx, const int32_t* nv, int64_t nv_cap,
                                 const void* kr, const void* v, void* gk, void* gv, int Hq,
                                 int Hkv, cudaStream_t st) {
  const int64_t threads = nv_cap * Hq * 16;
  if (threads <= 0) return cudaSuccess;
  const int64_t blocks = (threads + 255) / 256;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  sparse_gather_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      vidx, nv, nv_cap, static_cast<const uint4*>(kr), static_cast<const uint4*>(v),
      static_cast<uint4*>(gk), static_cast<uint4*>(gv), Hq, Hq / Hkv, Hkv);
  return cudaGetLastError();
}

}  // namespace dca
