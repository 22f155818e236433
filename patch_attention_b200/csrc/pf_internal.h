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
  CUtensorMap tm_kl;  // the same buffers bounded at lo_len rows [B, lo_len, H, d]: the rows
  CUtensorMap tm_vl;  //   past the lo segment are zero-filled, never read (unused if lo_len == 0)
  CUtensorMap tm_kt;  // K_txt [B, T, H, d]  (unused when T == 0)
  CUtensorMap tm_vt;  // V_txt
  const uint16_t* k_p;  // scatter source (fresh rows)
  const uint16_t* v_p;
  uint16_t* k_dst;      // scatter destination: buffer rows of the patch (K region base)
  uint16_t* v_dst;      // (V region base); both null => no scatter
  uint16_t* o;          // O [B, q_rows, H, d]
  int batch, heads, plen, n_img, n_txt, patch, head_dim;
  float scale_log2;     // softmax scale * log2(e)
  // Queries and context: q_rows query rows (tm_q); the context is the fresh rows
  // [0, fresh_rows) of tm_kf/tm_vf, buffer rows [0, lo_len) and [hi_row0, hi_row0 + hi_len),
  // then the n_txt text rows.  A patch micro-step has q_rows = fresh_rows = plen and the
  // buffer minus the patch's own rows; a text-query call has q_rows = n_txt, no fresh rows
  // and the whole buffer.
  int q_rows, fresh_rows, lo_len, hi_row0, hi_len;
  // Work decomposition: a "pair" is one (batch, head, group of NQ query tiles); its key
  // range is split into n_split contiguous parts, one CTA per (pair, part).
  int n_groups;         // query-tile groups per (batch, head)
  int n_pairs;          // batch * heads * n_groups
  int n_split;          // parts per pair (1 => no partials)
  float* ws_part;       // partial (O, m, l) slots, [pair][tile][part][d + 2][128] fp32
  unsigned* ws_cnt;     // per [pair][tile]: parts arrived, partials written; zero between launches
  int discard;          // drop the merged partials from L2 (1) rather than let them be written back
  // Order against the other calls on the same layer buffer without waiting for the whole
  // previous grid.  dep_scat counts CTAs of the layer's calls that finished their scatter
  // share, dep_read CTAs that finished reading the buffer; both are counted in call order (a
  // CTA counts once every CTA of the earlier calls has), so a count reaching the total of a
  // prefix of the calls means exactly that prefix is done.  Waits (all >=):
  //   hi rows:  *dep_scat >= dep_hi_target   (the scatters that wrote them)
  //   lo rows:  *dep_scat >= dep_lo_target
  //   scatter:  *dep_scat >= dep_scat_target (every earlier scatter) and
  //             *dep_read >= dep_war_target  (every earlier call that read the rows it writes)
  //   counting this CTA's reads: *dep_read >= dep_read_target (every earlier call) first.
  // Null dep_scat: wait for the previous grid instead (griddepcontrol.wait).
  unsigned long long* dep_scat;
  unsigned long long* dep_read;
  unsigned long long dep_hi_target;
  unsigned long long dep_lo_target;
  unsigned long long dep_scat_target;
  unsigned long long dep_war_target;
  unsigned long long dep_read_target;
};

// Query tiles per CTA chosen for a patch length (1 or 2).
int attn_tiles_per_cta(int plen);
// Number of 128-row context tiles of a call with the given segment lengths.
int attn_context_tiles(int fresh_rows, int lo_len, int hi_len, int n_txt);
// Key-range parts per (batch, head, query-tile group) for a call, given the number of SMs
// and the number of parts the workspace can hold.
int attn_choose_split(int n_pairs, int n_tiles, int n_sms, int max_split);
// Workspace bytes for n_pairs pairs split into n_split parts.
size_t attn_workspace_bytes(int n_pairs, int head_dim, int n_split);
// Zero the counters of a workspace.
cudaError_t launch_zero_u32(unsigned* p, size_t n, cudaStream_t stream);

// Launch the fused scatter + attention kernel.  Returns the launch error.
cudaError_t launch_patch_attn(const AttnParams& p, cudaStream_t stream);

// In-place per-head RMS normalisation of bf16 vectors (head_dim multiple of 8, <= 256).
cudaError_t launch_qk_rmsnorm(void* x, long long n_vectors, int head_dim, const void* gain,
                              float eps, cudaStream_t stream);

// Start-up copy of full-spatial K/V into a layer buffer (16-byte vectors).
cudaError_t launch_kvbuf_copy(const void* k_src, const void* v_src, void* k_dst, void* v_dst,
                              size_t n_elems, cudaStream_t stream);

// Guidance combine + rel-MAE.
size_t cfg_workspace_bytes(int batch, int64_t n_per_sample);
cudaError_t launch_cfg_combine_relmae(const float* c, const float* u, int batch, int64_t n,
                                      float w, float* out_f32, uint16_t* out_bf16, float* relmae,
                                      void* workspace, cudaStream_t stream);

// Guidance combine + rel-MAE with its partial sums in a static device array of the library
// (no caller workspace).  Returns cudaErrorInvalidValue if the batch exceeds the array.
cudaError_t launch_cfg_combine_relmae_static(const float* c, const float* u, int batch, int64_t n,
                                             float w, float* out_f32, uint16_t* out_bf16,
                                             float* relmae, cudaStream_t stream);
int cfg_static_capacity_samples();

// Device word written by kernels whose bounded waits expired (0 = none).
cudaError_t read_and_clear_watchdog(unsigned* value);

// A one-thread kernel whose bounded wait can never be satisfied: it gives up after limit_ns
// and sets its bit in the device word above.
cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t stream);

// Whether the current CUDA device is of compute capability 10.0 (what sm_100a code needs).  Returns cudaSuccess and
// sets *ok, or the error of the device query (no device, no driver).
cudaError_t device_is_sm100(bool* ok);

}  // namespace pf
