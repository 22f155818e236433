// qk_rmsnorm.cu -- per-head RMS normalisation of bf16 query/key vectors, in place.
//
// One warp per head vector: lanes load 16-byte chunks (8 bf16), the sum of squares is
// reduced with shuffles in fp32, and every element is scaled by rsqrt(mean + eps) (and an
// optional per-column gain) before rounding back to bf16.  HBM bound: 2 bytes read and 2
// written per element.

#include <cuda_bf16.h>

#include "pf_internal.h"

namespace pf {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(256) rmsnorm_kernel(uint4* __restrict__ x, long long n_vec,
                                                      int chunks, const uint4* __restrict__ gain,
                                                      float inv_d, float eps) {
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  uint4 g = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);  // bf16 1.0 pairs
  if (gain != nullptr && lane < chunks) g = gain[lane];
  for (long long v = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       v < n_vec; v += warps) {
    uint4 a = make_uint4(0, 0, 0, 0);
    if (lane < chunks) a = x[v * chunks + lane];
    float f[8] = {bf16_lo(a.x), bf16_hi(a.x), bf16_lo(a.y), bf16_hi(a.y),
                  bf16_lo(a.z), bf16_hi(a.z), bf16_lo(a.w), bf16_hi(a.w)};
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) ss = fmaf(f[k], f[k], ss);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float r = rsqrtf(fmaf(ss, inv_d, eps));
    if (lane < chunks) {
      const float gg[8] = {bf16_lo(g.x), bf16_hi(g.x), bf16_lo(g.y), bf16_hi(g.y),
                           bf16_lo(g.z), bf16_hi(g.z), bf16_lo(g.w), bf16_hi(g.w)};
      uint4 o;
      o.x = pack_bf16(f[0] * r * gg[0], f[1] * r * gg[1]);
      o.y = pack_bf16(f[2] * r * gg[2], f[3] * r * gg[3]);
      o.z = pack_bf16(f[4] * r * gg[4], f[5] * r * gg[5]);
      o.w = pack_bf16(f[6] * r * gg[6], f[7] * r * gg[7]);
      x[v * chunks + lane] = o;
    }
  }
}

}  // namespace

cudaError_t launch_qk_rmsnorm(void* x, long long n_vectors, int head_dim, const void* gain,
                              float eps, cudaStream_t stream) {
  if (n_vectors == 0) return cudaSuccess;
  const int chunks = head_dim / 8;
  long long blocks = (n_vectors + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  rmsnorm_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      reinterpret_cast<uint4*>(x), n_vectors, chunks, reinterpret_cast<const uint4*>(gain),
      1.0f / static_cast<float>(head_dim), eps);
  return cudaGetLastError();
}

}  // namespace pf
