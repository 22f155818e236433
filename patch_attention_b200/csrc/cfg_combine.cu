// cfg_combine.cu -- guidance combine fused with the rel-MAE_t reduction (HBM-bound).
//
// out = eps_u + w (eps_c - eps_u) and, per sample, ||eps_c - eps_u||_1 / ||eps_u||_1
// ("조건부 가이드 스케줄링 기반 하이브리드 데이터-파이프라인 병렬 처리를 통한 디퓨전 모델 가속화",
// second block 단락 1-3: the two noise predictions of the guidance paths and the rel-MAE_t
// signal that drives the parallelism switch).
//
// One pass over the inputs: 16-byte streaming loads of eps_c and eps_u, fp32 out as
// 16-byte stores and/or bf16 out as 8-byte stores, while each thread accumulates
// |c - u| and |u| in fp32.  Warp shuffles and a block tree reduce them; each block writes
// one fp64 partial pair.  A second one-warp-per-sample kernel adds the partials in a
// fixed order in fp64, so the result is deterministic (no float atomics).

#include <cuda_bf16.h>

#include <mutex>

#include "pf_internal.h"

namespace pf {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;          // float4 loads in flight per thread per input
constexpr int kTargetBlocks = 148 * 8;

int blocks_per_sample(int batch, int64_t n) {
  const int64_t n4 = n / 4;
  const int64_t per_block = static_cast<int64_t>(kThreads) * kUnroll;
  int64_t g = (n4 + per_block - 1) / per_block;
  int64_t cap = kTargetBlocks / batch;
  if (cap < 1) cap = 1;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

__device__ __forceinline__ float4 ld_stream(const float4* p) { return __ldcs(p); }

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(kThreads) cfg_partial_kernel(
    const float4* __restrict__ c, const float4* __restrict__ u, int64_t n4, float w,
    float4* __restrict__ out_f32, uint2* __restrict__ out_bf16, double2* __restrict__ partials) {
  // let the finalize kernel be scheduled now; it waits for this grid's completion itself
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // launched as a programmatic dependent of the previous work on the stream (often the last
  // attention launch of a step): wait until that grid has finished and its writes are
  // visible before touching memory
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.y;
  const int g = blockIdx.x;
  const int G = gridDim.x;
  const float4* cb = c + static_cast<int64_t>(b) * n4;
  const float4* ub = u + static_cast<int64_t>(b) * n4;
  float num = 0.f, den = 0.f;
  const int64_t stride = static_cast<int64_t>(G) * kThreads;
  int64_t i = static_cast<int64_t>(g) * kThreads + threadIdx.x;
  // main loop: kUnroll independent float4 pairs in flight
  for (; i + (kUnroll - 1) * stride < n4; i += kUnroll * stride) {
    float4 cv[kUnroll], uv[kUnroll];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      cv[k] = ld_stream(cb + i + k * stride);
      uv[k] = ld_stream(ub + i + k * stride);
    }
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int64_t e = static_cast<int64_t>(b) * n4 + i + k * stride;
      float4 d = make_float4(cv[k].x - uv[k].x, cv[k].y - uv[k].y, cv[k].z - uv[k].z, cv[k].w - uv[k].w);
      float4 o = make_float4(fmaf(w, d.x, uv[k].x), fmaf(w, d.y, uv[k].y), fmaf(w, d.z, uv[k].z),
                             fmaf(w, d.w, uv[k].w));
      num += (fabsf(d.x) + fabsf(d.y)) + (fabsf(d.z) + fabsf(d.w));
      den += (fabsf(uv[k].x) + fabsf(uv[k].y)) + (fabsf(uv[k].z) + fabsf(uv[k].w));
      if (out_f32) __stcs(out_f32 + e, o);
      if (out_bf16) __stcs(out_bf16 + e, make_uint2(bf16x2(o.x, o.y), bf16x2(o.z, o.w)));
    }
  }
  for (; i < n4; i += stride) {
    const float4 cv = ld_stream(cb + i);
    const float4 uv = ld_stream(ub + i);
    const int64_t e = static_cast<int64_t>(b) * n4 + i;
    float4 d = make_float4(cv.x - uv.x, cv.y - uv.y, cv.z - uv.z, cv.w - uv.w);
    float4 o = make_float4(fmaf(w, d.x, uv.x), fmaf(w, d.y, uv.y), fmaf(w, d.z, uv.z), fmaf(w, d.w, uv.w));
    num += (fabsf(d.x) + fabsf(d.y)) + (fabsf(d.z) + fabsf(d.w));
    den += (fabsf(uv.x) + fabsf(uv.y)) + (fabsf(uv.z) + fabsf(uv.w));
    if (out_f32) __stcs(out_f32 + e, o);
    if (out_bf16) __stcs(out_bf16 + e, make_uint2(bf16x2(o.x, o.y), bf16x2(o.z, o.w)));
  }
  // warp tree, then block tree over the 8 warp sums
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    num += __shfl_xor_sync(0xffffffffu, num, off);
    den += __shfl_xor_sync(0xffffffffu, den, off);
  }
  __shared__ float s_num[kThreads / 32], s_den[kThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    s_num[warp] = num;
    s_den[warp] = den;
  }
  __syncthreads();
  if (warp == 0) {
    num = lane < kThreads / 32 ? s_num[lane] : 0.f;
    den = lane < kThreads / 32 ? s_den[lane] : 0.f;
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) {
      num += __shfl_xor_sync(0xffffffffu, num, off);
      den += __shfl_xor_sync(0xffffffffu, den, off);
    }
    if (lane == 0) partials[static_cast<int64_t>(b) * G + g] = make_double2(num, den);
  }
}

__global__ void cfg_finalize_kernel(const double2* __restrict__ partials, int G,
                                    float* __restrict__ relmae) {
  // launched as a programmatic dependent of cfg_partial_kernel: wait until that grid has
  // finished and its partials are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.x;
  const int lane = threadIdx.x;
  double num = 0.0, den = 0.0;
  for (int g = lane; g < G; g += 32) {
    const double2 v = partials[static_cast<int64_t>(b) * G + g];
    num += v.x;
    den += v.y;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    num += __shfl_xor_sync(0xffffffffu, num, off);
    den += __shfl_xor_sync(0xffffffffu, den, off);
  }
  if (lane == 0) {
    float r;
    if (den == 0.0)
      r = num == 0.0 ? 0.f : __int_as_float(0x7f800000);
    else
      r = static_cast<float>(num / den);
    relmae[b] = r;
  }
}

}  // namespace

// ----------------------------------------------------------------------------------------
// Variant with no caller workspace: the fp64 partial sums go to a fixed array that lives in
// this library's device image, so the call needs no device allocation at all.

// 4096 partial-sum pairs (64 KiB).  One pair per (sample, block) of the partial kernel; the
// grid gives a batch of B samples at most max(B, 1184) pairs, so any batch up to 4096 fits.
constexpr int kStaticPartials = 4096;
static __device__ __align__(256) double2 g_cfg_static_partials[kStaticPartials];

namespace {
// Device address of g_cfg_static_partials per device ordinal.  In host code the array's name
// only stands in for the symbol; the address must be asked of the runtime with the device
// current, once per device.
constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_addr[kMaxDevices] = {};
}  // namespace

int cfg_static_capacity_samples() { return kStaticPartials; }

cudaError_t launch_cfg_combine_relmae_static(const float* c, const float* u, int batch, int64_t n,
                                             float w, float* out_f32, uint16_t* out_bf16,
                                             float* relmae, cudaStream_t stream) {
  const int G = blocks_per_sample(batch, n);
  if (static_cast<int64_t>(batch) * G > kStaticPartials) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (g_static_addr[dev] == nullptr) {
      e = cudaGetSymbolAddress(&g_static_addr[dev], g_cfg_static_partials);
      if (e != cudaSuccess) {
        g_static_addr[dev] = nullptr;
        return e;
      }
    }
    scratch = g_static_addr[dev];
  }
  // Every slot the finalize reads is written by the partial kernel of the same call, so the
  // array needs no clearing between calls.
  return launch_cfg_combine_relmae(c, u, batch, n, w, out_f32, out_bf16, relmae, scratch, stream);
}

size_t cfg_workspace_bytes(int batch, int64_t n_per_sample) {
  if (batch < 1 || n_per_sample < 4) return 0;
  return static_cast<size_t>(batch) * blocks_per_sample(batch, n_per_sample) * sizeof(double2);
}

cudaError_t launch_cfg_combine_relmae(const float* c, const float* u, int batch, int64_t n,
                                      float w, float* out_f32, uint16_t* out_bf16, float* relmae,
                                      void* workspace, cudaStream_t stream) {
  const int G = blocks_per_sample(batch, n);
  dim3 grid(G, batch);
  // both kernels are programmatic dependents: the partial kernel's launch overlaps the end of
  // the previous grid (it waits for it with griddepcontrol.wait before touching memory), and
  // the finalize is scheduled while the partial kernel runs (hiding its launch latency) and
  // synchronises on it the same way
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t pcfg = {};
  pcfg.gridDim = grid;
  pcfg.blockDim = dim3(kThreads);
  pcfg.dynamicSmemBytes = 0;
  pcfg.stream = stream;
  pcfg.attrs = attr;
  pcfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&pcfg, cfg_partial_kernel, reinterpret_cast<const float4*>(c),
                                     reinterpret_cast<const float4*>(u), n / 4, w,
                                     reinterpret_cast<float4*>(out_f32), reinterpret_cast<uint2*>(out_bf16),
                                     reinterpret_cast<double2*>(workspace));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(batch);
  cfg.blockDim = dim3(32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, cfg_finalize_kernel, reinterpret_cast<const double2*>(workspace), G,
                            relmae);
}

}  // namespace pf
