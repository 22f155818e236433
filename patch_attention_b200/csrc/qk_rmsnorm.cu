// qk_rmsnorm.cu -- per-head RMS normalisation of bf16 query/key vectors, in place.
//
// A head vector of d bf16 elements is d/8 16-byte chunks.  A warp is cut into segments of
// SEG lanes (SEG = d/8 rounded up to a power of two) and normalises 32/SEG vectors at once,
// one chunk per lane: d = 128 packs 2 vectors per warp, d = 64 packs 4, so no lane idles for
// the power-of-two sizes.  The sum of squares is reduced in fp32 by xor shuffles inside each
// segment, and every element is scaled by rsqrt(mean + eps) (and an optional per-column gain)
// before rounding back to bf16.  Each lane keeps two vectors' chunks in flight.  HBM bound:
// 2 bytes read and 2 written per element.

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

__device__ __forceinline__ float sumsq8(const uint4& a) {
  const float f[8] = {bf16_lo(a.x), bf16_hi(a.x), bf16_lo(a.y), bf16_hi(a.y),
                      bf16_lo(a.z), bf16_hi(a.z), bf16_lo(a.w), bf16_hi(a.w)};
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) ss = fmaf(f[k], f[k], ss);
  return ss;
}

__device__ __forceinline__ uint4 scale8(const uint4& a, float r, const uint4& g) {
  uint4 o;
  o.x = pack_bf16(bf16_lo(a.x) * r * bf16_lo(g.x), bf16_hi(a.x) * r * bf16_hi(g.x));
  o.y = pack_bf16(bf16_lo(a.y) * r * bf16_lo(g.y), bf16_hi(a.y) * r * bf16_hi(g.y));
  o.z = pack_bf16(bf16_lo(a.z) * r * bf16_lo(g.z), bf16_hi(a.z) * r * bf16_hi(g.z));
  o.w = pack_bf16(bf16_lo(a.w) * r * bf16_lo(g.w), bf16_hi(a.w) * r * bf16_hi(g.w));
  return o;
}

template <int SEG>
__global__ void __launch_bounds__(256) rmsnorm_kernel(uint4* __restrict__ x, long long n_vec,
                                                      int chunks, const uint4* __restrict__ gain,
                                                      float inv_d, float eps) {
  constexpr int kPerWarp = 32 / SEG;  // vectors a warp normalises at once
  const int lane = threadIdx.x & 31;
  const int sub = lane / SEG;         // which vector of the warp's group
  const int c = lane % SEG;           // which chunk of that vector
  const bool active = c < chunks;
  uint4 g = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);  // bf16 1.0 pairs
  if (gain != nullptr && active) g = gain[c];
  const long long groups = (n_vec + kPerWarp - 1) / kPerWarp;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long w0 = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  // two groups per iteration: both loads are issued before either reduction
  for (long long gi = w0; gi < groups; gi += 2 * warps) {
    const long long v0 = gi * kPerWarp + sub;
    const long long v1 = (gi + warps) * kPerWarp + sub;
    const bool in0 = active && v0 < n_vec;
    const bool in1 = active && gi + warps < groups && v1 < n_vec;
    uint4 a0 = make_uint4(0, 0, 0, 0), a1 = make_uint4(0, 0, 0, 0);
    if (in0) a0 = x[v0 * chunks + c];
    if (in1) a1 = x[v1 * chunks + c];
    float s0 = sumsq8(a0), s1 = sumsq8(a1);
#pragma unroll
    for (int off = SEG / 2; off > 0; off >>= 1) {
      s0 += __shfl_xor_sync(0xffffffffu, s0, off);
      s1 += __shfl_xor_sync(0xffffffffu, s1, off);
    }
    if (in0) x[v0 * chunks + c] = scale8(a0, rsqrtf(fmaf(s0, inv_d, eps)), g);
    if (in1) x[v1 * chunks + c] = scale8(a1, rsqrtf(fmaf(s1, inv_d, eps)), g);
  }
}

template <int SEG>
cudaError_t launch_seg(void* x, long long n_vectors, int chunks, const void* gain, float inv_d,
                       float eps, cudaStream_t stream) {
  constexpr int kPerBlock = 8 * (32 / SEG);  // vectors per block-iteration (8 warps)
  long long blocks = (n_vectors + 2 * kPerBlock - 1) / (2 * kPerBlock);
  if (blocks > 148 * 8) blocks = 148 * 8;
  rmsnorm_kernel<SEG><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      reinterpret_cast<uint4*>(x), n_vectors, chunks, reinterpret_cast<const uint4*>(gain), inv_d, eps);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qk_rmsnorm(void* x, long long n_vectors, int head_dim, const void* gain,
                              float eps, cudaStream_t stream) {
  if (n_vectors == 0) return cudaSuccess;
  const int chunks = head_dim / 8;  // 1 .. 32 (head_dim a multiple of 8, at most 256)
  const float inv_d = 1.0f / static_cast<float>(head_dim);
  if (chunks <= 1) return launch_seg<1>(x, n_vectors, chunks, gain, inv_d, eps, stream);
  if (chunks <= 2) return launch_seg<2>(x, n_vectors, chunks, gain, inv_d, eps, stream);
  if (chunks <= 4) return launch_seg<4>(x, n_vectors, chunks, gain, inv_d, eps, stream);
  if (chunks <= 8) return launch_seg<8>(x, n_vectors, chunks, gain, inv_d, eps, stream);
  if (chunks <= 16) return launch_seg<16>(x, n_vectors, chunks, gain, inv_d, eps, stream);
  return launch_seg<32>(x, n_vectors, chunks, gain, inv_d, eps, stream);
}

}  // namespace pf
