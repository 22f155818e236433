// pf_internal.h -- declarations shared by the host API (pf_api.cpp) and the CUDA
// translation units.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace pf {

// Kernel parameters of one patch-attention micro-step.  Tensor maps describe 4-D
// [batch, rows, heads, head_dim] bf16 tensors (innermost first: head_dim, heads, rows,
// batch) with a 64-element x 128-row box and 128-byte swizzle.
struct AttnParams {
  CUtensorMap tm_q;   // Q_p   [B, P, H, d]
  CUtensorMap tm_kf;  // K_p   [B, P, H, d]   fresh rows of the patch
  CUtensorMap tm_vf;  // V_p
  CUtensorMap tm_kb;  // K buffer being read [B, N, H, d]
  CUtensorMap tm_vb;  // V buffer being read
  CUtensorMap tm_kt;  // K_txt [B, T, H, d]  (unused when T == 0)
  CUtensorMap tm_vt;  // V_txt
  const uint16_t* k_p;  // scatter source (fresh rows)
  const uint16_t* v_p;
  uint16_t* k_dst;      // scatter destination: buffer rows of the patch (K region base)
  uint16_t* v_dst;      // (V region base); both null => no scatter
  uint16_t* o;          // O_p [B, P, H, d]
  int batch, heads, plen, n_img, n_txt, patch, head_dim;
  float scale_log2;     // softmax scale * log2(e)
};

// Launch the fused scatter + attention kernel.  Returns the launch error.
cudaError_t launch_patch_attn(const AttnParams& p, cudaStream_t stream);

// Start-up copy of full-spatial K/V into a layer buffer (16-byte vectors).
cudaError_t launch_kvbuf_copy(const void* k_src, const void* v_src, void* k_dst, void* v_dst,
                              size_t n_elems, cudaStream_t stream);

// Guidance combine + rel-MAE.
size_t cfg_workspace_bytes(int batch, int64_t n_per_sample);
cudaError_t launch_cfg_combine_relmae(const float* c, const float* u, int batch, int64_t n,
                                      float w, float* out_f32, uint16_t* out_bf16, float* relmae,
                                      void* workspace, cudaStream_t stream);

// Device word written by kernels whose bounded waits expired (0 = none).
cudaError_t read_and_clear_watchdog(unsigned* value);

// Host check that a device of compute capability 10.x is current.
bool device_is_sm100();

}  // namespace pf
