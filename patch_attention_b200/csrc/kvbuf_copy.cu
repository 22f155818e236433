// kvbuf_copy.cu -- start-up fill of a layer's K/V buffer with the first step's full-spatial
// K and V ("기술 요약: PipeFusion", 핵심 메커니즘 2: stale activations exist only after the
// initial pass).  A bit copy with 16-byte vectors, both tensors in one grid-stride launch.

#include "pf_internal.h"

namespace pf {
namespace {

__global__ void __launch_bounds__(256) kvbuf_copy_kernel(const uint4* __restrict__ ks,
                                                         const uint4* __restrict__ vs,
                                                         uint4* __restrict__ kd,
                                                         uint4* __restrict__ vd, int64_t n16) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16; i += stride) {
    const uint4 k = __ldcs(ks + i);
    const uint4 v = __ldcs(vs + i);
    kd[i] = k;
    vd[i] = v;
  }
}

}  // namespace

cudaError_t launch_kvbuf_copy(const void* k_src, const void* v_src, void* k_dst, void* v_dst,
                              size_t n_elems, cudaStream_t stream) {
  const int64_t n16 = static_cast<int64_t>(n_elems / 8);  // bf16 elements -> 16-byte vectors
  if (n16 == 0) return cudaSuccess;
  int64_t blocks = (n16 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  kvbuf_copy_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(k_src), reinterpret_cast<const uint4*>(v_src),
      reinterpret_cast<uint4*>(k_dst), reinterpret_cast<uint4*>(v_dst), n16);
  return cudaGetLastError();
}

}  // namespace pf
