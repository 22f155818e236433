// pf_api.cpp -- host side of the C ABI declared in include/patchattn.h.
//
// Validates every argument before anything is enqueued, keeps the per-layer schedule
// state (which patch comes next, which buffer half is read), encodes the TMA tensor maps
// of each micro-step and launches the kernels.  Holds no device memory.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "patchattn.h"
#include "pf_internal.h"

struct pf_ctx {
  pf_config cfg;
  float scale;
  size_t tensor_elems;           // B * N * H * d: one K or V region of a buffer
  std::vector<uint8_t*> base;    // per layer, caller-owned
  std::vector<int> next_patch;   // PipeFusion: the patch the layer expects next
  std::vector<int> initialised;
  std::vector<int> read_half;    // two halves: which half holds the previous step's rows
  std::vector<std::vector<uint8_t>> seen;  // DistriFusion: patches done in the current step
  std::vector<int> seen_count;
  uint8_t* ws = nullptr;         // optional attention workspace (caller-owned)
  size_t ws_bytes = 0;
  int n_sms = 0;                 // queried on first use
  // Per layer, for the workspace's ordering counters (reset with the workspace): the CTAs of
  // the calls launched so far that will count a finished scatter, and those that will count
  // finished reads; both as they stood when the current step began; and, per patch, the read
  // count just before that patch's call of the previous step (two buffer halves).
  std::vector<unsigned long long> scat_target;
  std::vector<unsigned long long> read_target;
  std::vector<unsigned long long> scat_step_start;
  std::vector<unsigned long long> read_step_start;
  std::vector<std::vector<unsigned long long>> read_before_patch;
};

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once per process (thread-safe: the first
// caller does the lookup, concurrent callers wait for it).
EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pf_status check_config(const pf_config* c) {
  if (!c) return PF_ERR_INVALID_ARG;
  if (c->batch < 1 || c->heads < 1 || c->n_img < 1 || c->n_patches < 1 || c->n_txt < 0 ||
      c->n_layers < 1)
    return PF_ERR_SHAPE;
  if (c->n_img % c->n_patches != 0) return PF_ERR_SHAPE;
  if (c->head_dim != 64 && c->head_dim != 72 && c->head_dim != 128) return PF_ERR_UNSUPPORTED;
  if (c->schedule != PF_SCHED_PIPEFUSION && c->schedule != PF_SCHED_DISTRIFUSION &&
      c->schedule != PF_SCHED_PIPEFUSION_2H)
    return PF_ERR_UNSUPPORTED;
  if (!(c->softmax_scale >= 0.f) || std::isinf(c->softmax_scale)) return PF_ERR_INVALID_ARG;
  // TMA coordinates and per-row offsets are 32-bit
  const double rows = static_cast<double>(c->batch) * c->n_img;
  if (rows > 2e9 || static_cast<double>(c->n_txt) * c->batch > 2e9) return PF_ERR_SHAPE;
  return PF_OK;
}

size_t region_elems(const pf_config* c) {
  return static_cast<size_t>(c->batch) * c->n_img * c->heads * c->head_dim;
}

// [batch, rows, heads, d] bf16 -> 4-D tensor map, box = 64 columns x 1 head x 128 rows.
// The map covers the first `rows` rows of each batch element, whose rows are `batch_rows`
// apart (batch_rows >= rows; 0 means rows): loads past `rows` read zeros.
bool make_map(CUtensorMap* m, const void* base, int batch, int rows, int heads, int d,
              int batch_rows = 0) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if (batch_rows == 0) batch_rows = rows;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(batch)};
  const cuuint64_t row_bytes = static_cast<cuuint64_t>(heads) * d * 2;
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, row_bytes,
                                 row_bytes * static_cast<cuuint64_t>(batch_rows)};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

pf_status from_cuda(cudaError_t e) { return e == cudaSuccess ? PF_OK : PF_ERR_CUDA; }

// Attention launches: cudaErrorNotSupported is the library's own refusal (a kernel image
// whose compiled register count does not fit its warpgroup register split).
pf_status from_attn_launch(cudaError_t e) {
  if (e == cudaSuccess) return PF_OK;
  return e == cudaErrorNotSupported ? PF_ERR_UNSUPPORTED : PF_ERR_CUDA;
}

// (batch, head, query-tile group) pairs of a call with q_rows query rows
int pairs_for(const pf_config& c, int q_rows) {
  const int nq = pf::attn_tiles_per_cta(q_rows);
  const int groups = (q_rows + nq * 128 - 1) / (nq * 128);
  return c.batch * c.heads * groups;
}

int pairs_of(const pf_config& c) {
  const int a = pairs_for(c, c.n_img / c.n_patches);
  const int b = c.n_txt > 0 ? pairs_for(c, c.n_txt) : 0;
  return a > b ? a : b;
}

constexpr int kAssumedSms = 148;

// Counters first (fixed place, sized for the larger of patch and text-query calls), then the
// partial slots.
// Two counters (parts arrived, partials written) per query tile of every pair, then two
// 64-bit ordering counters per layer (CTAs that finished their scatter, CTAs that finished
// reading the buffer).
size_t pair_counter_bytes(int pairs) { return static_cast<size_t>(pairs) * 2 * 2 * 4; }
size_t counter_bytes(const pf_config& c) {
  const size_t b = pair_counter_bytes(pairs_of(c)) + static_cast<size_t>(c.n_layers) * 2 * 8;
  return ((b + 255) / 256) * 256;
}

// A layer with two buffer halves: the step being written goes to the half that the step does
// not read (DistriFusion, and PipeFusion over two halves).
bool two_halves(const pf_config& c) { return c.schedule != PF_SCHED_PIPEFUSION; }


size_t workspace_for(const pf_config& c, int n_sms) {
  const int plen = c.n_img / c.n_patches;
  const size_t cb = counter_bytes(c);
  size_t best = cb;  // the counters, split or not
  auto consider = [&](int q_rows, int tiles) {
    const int pairs = pairs_for(c, q_rows);
    const int k = pf::attn_choose_split(pairs, tiles, n_sms, 1 << 30);
    const size_t b = k > 1 ? cb + pf::attn_workspace_bytes(pairs, c.head_dim, k) : 0;
    if (b > best) best = b;
  };
  for (int p = 0; p < c.n_patches; ++p) {
    consider(plen, pf::attn_context_tiles(plen, p * plen, c.n_img - (p + 1) * plen, c.n_txt));
    if (plen % 128 == 0) break;  // every patch has the same tile count
  }
  if (c.n_txt > 0) consider(c.n_txt, pf::attn_context_tiles(0, c.n_img, 0, c.n_txt));
  return best;
}

bool layer_ok(const pf_ctx* ctx, int layer) { return layer >= 0 && layer < ctx->cfg.n_layers; }

// A step of a layer starts (two buffer halves): record the counts its calls' waits refer to.
// After pf_kvbuf_init or pf_set_state every earlier call has finished (the start-up copy
// waits for the stream's earlier work), so the previous step's per-patch counts are dropped.
void begin_step(pf_ctx* ctx, int layer, bool restart) {
  if (ctx->ws == nullptr) return;
  ctx->scat_step_start[layer] = ctx->scat_target[layer];
  ctx->read_step_start[layer] = ctx->read_target[layer];
  if (restart)
    std::fill(ctx->read_before_patch[layer].begin(), ctx->read_before_patch[layer].end(),
              ctx->read_target[layer]);
}

// What a call on a layer waits for, as counts of the layer's ordering counters.
struct Waits {
  unsigned long long hi, lo, war;  // scatters before hi rows / lo rows; reads before the scatter
};

// Fill the fields common to every attention call (sizes, scale, work decomposition and
// key-range split) and launch.  p carries the tensor maps, pointers and segments; w what the
// call waits for (with a workspace).
cudaError_t launch_attention(pf_ctx* ctx, pf::AttnParams& p, int layer, const Waits& w, void* stream) {
  const pf_config& c = ctx->cfg;
  p.batch = c.batch;
  p.heads = c.heads;
  p.n_img = c.n_img;
  p.n_txt = c.n_txt;
  p.head_dim = c.head_dim;
  p.scale_log2 = ctx->scale * 1.4426950408889634f;
  const int nq = pf::attn_tiles_per_cta(p.q_rows);
  p.n_groups = (p.q_rows + nq * 128 - 1) / (nq * 128);
  p.n_pairs = c.batch * c.heads * p.n_groups;
  p.n_split = 1;
  if (ctx->ws != nullptr) {
    if (ctx->n_sms == 0) {
      int dev = 0, n = 0;
      if (cudaGetDevice(&dev) == cudaSuccess &&
          cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
        ctx->n_sms = n;
      else
        ctx->n_sms = kAssumedSms;
    }
    const int tiles = pf::attn_context_tiles(p.fresh_rows, p.lo_len, p.hi_len, c.n_txt);
    const size_t cb = counter_bytes(c);
    int cap = 1;  // most parts the workspace can hold
    while (cap < 16 && cb + pf::attn_workspace_bytes(p.n_pairs, c.head_dim, cap + 1) <= ctx->ws_bytes)
      ++cap;
    p.n_split = pf::attn_choose_split(p.n_pairs, tiles, ctx->n_sms, cap);
    if (p.n_split > 1) {
      p.ws_cnt = reinterpret_cast<unsigned*>(ctx->ws);
      p.ws_part = reinterpret_cast<float*>(ctx->ws + cb);
      // a launch of several waves keeps writing partials while earlier ones are merged: drop
      // the merged ones from L2 instead of letting them go back to DRAM; a single wave's few
      // partials cost less to write back than the discard costs at the end of the launch
      p.discard = static_cast<long long>(p.n_pairs) * p.n_split > ctx->n_sms ? 1 : 0;
    }
  }
  if (ctx->ws != nullptr) {
    // order against the other calls on this layer through the workspace's counters, so that
    // the launch need not wait for the previous grid (often another layer's) before it reads
    unsigned long long* dep = reinterpret_cast<unsigned long long*>(
        ctx->ws + pair_counter_bytes(pairs_of(c))) + static_cast<size_t>(layer) * 2;
    p.dep_scat = dep;
    p.dep_read = dep + 1;
    p.dep_hi_target = w.hi;
    p.dep_lo_target = w.lo;
    p.dep_scat_target = ctx->scat_target[layer];
    p.dep_war_target = w.war;
    p.dep_read_target = ctx->read_target[layer];
  }
  const cudaError_t e = pf::launch_patch_attn(p, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess && ctx->ws != nullptr) {
    // every CTA of this launch counts itself once on each counter it takes part in
    const unsigned long long ctas = static_cast<unsigned long long>(p.n_pairs) * p.n_split;
    ctx->read_target[layer] += ctas;
    if (p.k_dst != nullptr) ctx->scat_target[layer] += ctas;
  }
  return e;
}

// K/V regions of a layer's buffer: half 0 is [K | V]; two-half schedules add half 1 [K | V].
uint8_t* region(const pf_ctx* ctx, int layer, int half, int kv) {
  const size_t bytes = ctx->tensor_elems * 2;
  return ctx->base[layer] + (static_cast<size_t>(half) * 2 + kv) * bytes;
}

}  // namespace

namespace pf {
cudaError_t device_is_sm100(bool* ok) {
  int dev = 0, major = 0, minor = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (e != cudaSuccess) {
    cudaGetLastError();  // clear the failed query from the thread's last-error slot
    return e;
  }
  // sm_100a code (tcgen05, TMA) runs on compute capability 10.0 only
  *ok = major == 10 && minor == 0;
  return cudaSuccess;
}
}  // namespace pf

extern "C" {

size_t pf_kvbuf_bytes(const pf_config* cfg) {
  if (check_config(cfg) != PF_OK) return 0;
  const size_t halves = two_halves(*cfg) ? 2 : 1;
  return halves * 2 * region_elems(cfg) * 2;
}

pf_status pf_create(const pf_config* cfg, void* const* kvbuf_per_layer, pf_ctx** out) {
  if (!out) return PF_ERR_INVALID_ARG;
  *out = nullptr;
  pf_status st = check_config(cfg);
  if (st != PF_OK) return st;
  if (!kvbuf_per_layer) return PF_ERR_INVALID_ARG;
  for (int l = 0; l < cfg->n_layers; ++l) {
    if (!kvbuf_per_layer[l]) return PF_ERR_INVALID_ARG;
    if (!aligned16(kvbuf_per_layer[l])) return PF_ERR_ALIGN;
  }
  // A device that is current must be a B200-class part (compute capability 10.0): the
  // kernels are built for sm_100a only.  Without any usable device the context is still
  // created (it is host state only); its launches then fail with PF_ERR_CUDA.
  bool sm100 = false;
  if (pf::device_is_sm100(&sm100) == cudaSuccess && !sm100) return PF_ERR_UNSUPPORTED;
  pf_ctx* ctx = new (std::nothrow) pf_ctx();
  if (!ctx) return PF_ERR_INVALID_ARG;
  ctx->cfg = *cfg;
  ctx->scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale
                                        : 1.0f / std::sqrt(static_cast<float>(cfg->head_dim));
  ctx->tensor_elems = region_elems(cfg);
  ctx->base.resize(cfg->n_layers);
  for (int l = 0; l < cfg->n_layers; ++l) ctx->base[l] = static_cast<uint8_t*>(kvbuf_per_layer[l]);
  ctx->next_patch.assign(cfg->n_layers, 0);
  ctx->initialised.assign(cfg->n_layers, 0);
  ctx->read_half.assign(cfg->n_layers, 0);
  ctx->seen.assign(cfg->n_layers, std::vector<uint8_t>(cfg->n_patches, 0));
  ctx->seen_count.assign(cfg->n_layers, 0);
  *out = ctx;
  return PF_OK;
}

pf_status pf_destroy(pf_ctx* ctx) {
  delete ctx;
  return PF_OK;
}

pf_status pf_kvbuf_init(pf_ctx* ctx, int layer, const void* k_full, const void* v_full,
                        void* stream) {
  if (!ctx || !k_full || !v_full) return PF_ERR_INVALID_ARG;
  if (!layer_ok(ctx, layer)) return PF_ERR_INVALID_ARG;
  if (!aligned16(k_full) || !aligned16(v_full)) return PF_ERR_ALIGN;
  const int half = ctx->read_half[layer];
  cudaError_t e = pf::launch_kvbuf_copy(k_full, v_full, region(ctx, layer, half, 0),
                                        region(ctx, layer, half, 1), ctx->tensor_elems,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return PF_ERR_CUDA;
  ctx->initialised[layer] = 1;
  ctx->next_patch[layer] = 0;
  std::fill(ctx->seen[layer].begin(), ctx->seen[layer].end(), 0);
  ctx->seen_count[layer] = 0;
  begin_step(ctx, layer, true);
  return PF_OK;
}

pf_status pf_patch_attn_step(pf_ctx* ctx, int layer, int patch, const void* q_p,
                             const void* k_p, const void* v_p, const void* k_txt,
                             const void* v_txt, void* o_p, void* stream) {
  if (!ctx) return PF_ERR_INVALID_ARG;
  const pf_config& c = ctx->cfg;
  if (!layer_ok(ctx, layer) || patch < 0 || patch >= c.n_patches) return PF_ERR_INVALID_ARG;
  if (!q_p || !k_p || !v_p || !o_p) return PF_ERR_INVALID_ARG;
  if (c.n_txt > 0 && (!k_txt || !v_txt)) return PF_ERR_INVALID_ARG;
  if (c.n_txt == 0 && (k_txt || v_txt)) return PF_ERR_INVALID_ARG;
  if (!aligned16(q_p) || !aligned16(k_p) || !aligned16(v_p) || !aligned16(o_p) ||
      (k_txt && !aligned16(k_txt)) || (v_txt && !aligned16(v_txt)))
    return PF_ERR_ALIGN;
  if (!ctx->initialised[layer]) return PF_ERR_STATE;
  // PipeFusion (either buffer layout) takes the patches in order; DistriFusion in any order
  const bool in_order = c.schedule != PF_SCHED_DISTRIFUSION;
  if (in_order) {
    if (patch != ctx->next_patch[layer]) return PF_ERR_ORDER;
  } else {
    if (ctx->seen[layer][patch]) return PF_ERR_ORDER;
  }

  const int plen = c.n_img / c.n_patches;
  const int d = c.head_dim;
  pf::AttnParams p;
  std::memset(&p, 0, sizeof(p));
  const int read = ctx->read_half[layer];
  const int write = two_halves(c) ? 1 - read : read;
  // rows of patches < p: this step's (PipeFusion) are in the half being written; the previous
  // step's (DistriFusion) in the half being read
  const bool lo_current = c.schedule != PF_SCHED_DISTRIFUSION;
  const int lo_half = lo_current ? write : read;
  const int lo_len = patch * plen;
  if (!make_map(&p.tm_q, q_p, c.batch, plen, c.heads, d) ||
      !make_map(&p.tm_kf, k_p, c.batch, plen, c.heads, d) ||
      !make_map(&p.tm_vf, v_p, c.batch, plen, c.heads, d) ||
      !make_map(&p.tm_kb, region(ctx, layer, read, 0), c.batch, c.n_img, c.heads, d) ||
      !make_map(&p.tm_vb, region(ctx, layer, read, 1), c.batch, c.n_img, c.heads, d))
    return PF_ERR_CUDA;
  // the rows before the patch through maps that end at the patch: the last tile of that
  // segment reads zeros, not the patch's own rows, which this launch's scatter is writing
  if (lo_len > 0 &&
      (!make_map(&p.tm_kl, region(ctx, layer, lo_half, 0), c.batch, lo_len, c.heads, d, c.n_img) ||
       !make_map(&p.tm_vl, region(ctx, layer, lo_half, 1), c.batch, lo_len, c.heads, d, c.n_img)))
    return PF_ERR_CUDA;
  if (c.n_txt > 0 && (!make_map(&p.tm_kt, k_txt, c.batch, c.n_txt, c.heads, d) ||
                      !make_map(&p.tm_vt, v_txt, c.batch, c.n_txt, c.heads, d)))
    return PF_ERR_CUDA;
  p.k_p = static_cast<const uint16_t*>(k_p);
  p.v_p = static_cast<const uint16_t*>(v_p);
  p.k_dst = reinterpret_cast<uint16_t*>(region(ctx, layer, write, 0));
  p.v_dst = reinterpret_cast<uint16_t*>(region(ctx, layer, write, 1));
  p.o = static_cast<uint16_t*>(o_p);
  p.plen = plen;
  p.patch = patch;
  p.q_rows = plen;
  p.fresh_rows = plen;
  p.lo_len = lo_len;
  p.hi_row0 = (patch + 1) * plen;
  p.hi_len = c.n_img - (patch + 1) * plen;
  Waits w{};
  unsigned long long read_before = 0;
  if (ctx->ws != nullptr) {
    const unsigned long long all_scat = ctx->scat_target[layer], all_read = ctx->read_target[layer];
    read_before = all_read;
    if (c.schedule == PF_SCHED_PIPEFUSION) {
      // one half: every earlier call wrote rows this call reads or read rows it overwrites
      w = {all_scat, all_scat, all_read};
    } else if (c.schedule == PF_SCHED_PIPEFUSION_2H) {
      // hi rows: written in earlier steps; lo rows: by this step's earlier calls; the rows
      // of patch p in the half being written: read by the calls before patch p of the
      // previous step (as its stale rows) and by older ones
      w = {ctx->scat_step_start[layer], all_scat, ctx->read_before_patch[layer][patch]};
    } else {
      // DistriFusion: every row read was written in earlier steps; every call of the
      // previous step read the rows of the half being written
      w = {ctx->scat_step_start[layer], ctx->scat_step_start[layer], ctx->read_step_start[layer]};
    }
  }
  const pf_status ls = from_attn_launch(launch_attention(ctx, p, layer, w, stream));
  if (ls != PF_OK) return ls;
  if (ctx->ws != nullptr) ctx->read_before_patch[layer][patch] = read_before;

  bool step_done = false;
  if (in_order) {
    ctx->next_patch[layer] = (patch + 1) % c.n_patches;
    step_done = ctx->next_patch[layer] == 0;
  } else {
    ctx->seen[layer][patch] = 1;
    if (++ctx->seen_count[layer] == c.n_patches) {
      std::fill(ctx->seen[layer].begin(), ctx->seen[layer].end(), 0);
      ctx->seen_count[layer] = 0;
      step_done = true;
    }
    ctx->next_patch[layer] = ctx->seen_count[layer];
  }
  if (step_done && two_halves(c)) {
    // every patch of the step wrote its fresh rows into the other half: it becomes the
    // previous step's half of the next step
    ctx->read_half[layer] = 1 - ctx->read_half[layer];
    begin_step(ctx, layer, false);
  }
  return PF_OK;
}

pf_status pf_text_attn_step(pf_ctx* ctx, int layer, const void* q_txt, const void* k_txt,
                            const void* v_txt, void* o_txt, void* stream) {
  if (!ctx) return PF_ERR_INVALID_ARG;
  const pf_config& c = ctx->cfg;
  if (!layer_ok(ctx, layer)) return PF_ERR_INVALID_ARG;
  if (c.n_txt == 0) return PF_ERR_SHAPE;
  if (!q_txt || !k_txt || !v_txt || !o_txt) return PF_ERR_INVALID_ARG;
  if (!aligned16(q_txt) || !aligned16(k_txt) || !aligned16(v_txt) || !aligned16(o_txt))
    return PF_ERR_ALIGN;
  if (!ctx->initialised[layer]) return PF_ERR_STATE;
  const int d = c.head_dim;
  const int read = ctx->read_half[layer];
  const int plen = c.n_img / c.n_patches;
  // the buffer as it stands: with PipeFusion over two halves, the rows of the patches done in
  // this step are in the half being written and the rest in the other; otherwise all of it is
  // in the half being read
  const bool split_halves = c.schedule == PF_SCHED_PIPEFUSION_2H;
  const int lo_len = split_halves ? ctx->next_patch[layer] * plen : c.n_img;
  pf::AttnParams p;
  std::memset(&p, 0, sizeof(p));
  const int lo_half = split_halves ? 1 - read : read;
  if (!make_map(&p.tm_q, q_txt, c.batch, c.n_txt, c.heads, d) ||
      !make_map(&p.tm_kt, k_txt, c.batch, c.n_txt, c.heads, d) ||
      !make_map(&p.tm_vt, v_txt, c.batch, c.n_txt, c.heads, d))
    return PF_ERR_CUDA;
  if (lo_len > 0 &&
      (!make_map(&p.tm_kl, region(ctx, layer, lo_half, 0), c.batch, lo_len, c.heads, d, c.n_img) ||
       !make_map(&p.tm_vl, region(ctx, layer, lo_half, 1), c.batch, lo_len, c.heads, d, c.n_img)))
    return PF_ERR_CUDA;
  if (lo_len < c.n_img &&
      (!make_map(&p.tm_kb, region(ctx, layer, read, 0), c.batch, c.n_img, c.heads, d) ||
       !make_map(&p.tm_vb, region(ctx, layer, read, 1), c.batch, c.n_img, c.heads, d)))
    return PF_ERR_CUDA;
  p.o = static_cast<uint16_t*>(o_txt);
  p.plen = plen;
  p.q_rows = c.n_txt;   // text queries
  p.fresh_rows = 0;     // no fresh patch rows, no scatter (k_dst stays null)
  p.lo_len = lo_len;
  p.hi_row0 = lo_len;
  p.hi_len = c.n_img - lo_len;
  Waits w{};
  if (ctx->ws != nullptr) {
    // lo rows: the half being written (two-half PipeFusion) or the one half; hi rows and
    // DistriFusion's rows: written in earlier steps
    const unsigned long long start = two_halves(c) ? ctx->scat_step_start[layer] : ctx->scat_target[layer];
    w = {start, c.schedule == PF_SCHED_DISTRIFUSION ? start : ctx->scat_target[layer], 0ull};
  }
  const pf_status ls = from_attn_launch(launch_attention(ctx, p, layer, w, stream));
  if (ls != PF_OK) return ls;
  return PF_OK;
}

pf_status pf_qk_rmsnorm(void* x, int64_t n_vectors, int head_dim, const void* gain, float eps,
                        void* stream) {
  if (!x || n_vectors < 0) return PF_ERR_INVALID_ARG;
  if (head_dim < 8 || head_dim > 256 || head_dim % 8 != 0) return PF_ERR_SHAPE;
  if (!(eps > 0.f) || !std::isfinite(eps)) return PF_ERR_INVALID_ARG;
  if (!aligned16(x) || (gain && !aligned16(gain))) return PF_ERR_ALIGN;
  return from_cuda(pf::launch_qk_rmsnorm(x, n_vectors, head_dim, gain, eps,
                                         static_cast<cudaStream_t>(stream)));
}

pf_status pf_get_state(const pf_ctx* ctx, int layer, int* next_patch) {
  if (!ctx || !next_patch || !layer_ok(ctx, layer)) return PF_ERR_INVALID_ARG;
  if (!ctx->initialised[layer]) return PF_ERR_STATE;
  *next_patch = ctx->next_patch[layer];
  return PF_OK;
}

pf_status pf_get_read_half(const pf_ctx* ctx, int layer, int* half) {
  if (!ctx || !half || !layer_ok(ctx, layer)) return PF_ERR_INVALID_ARG;
  *half = ctx->read_half[layer];
  return PF_OK;
}

pf_status pf_set_state(pf_ctx* ctx, int layer, int next_patch) {
  if (!ctx || !layer_ok(ctx, layer)) return PF_ERR_INVALID_ARG;
  if (next_patch < 0 || next_patch >= ctx->cfg.n_patches) return PF_ERR_INVALID_ARG;
  if (ctx->cfg.schedule != PF_SCHED_PIPEFUSION && next_patch != 0) return PF_ERR_UNSUPPORTED;
  ctx->next_patch[layer] = next_patch;
  ctx->initialised[layer] = 1;
  if (two_halves(ctx->cfg)) {
    // a step starts
    std::fill(ctx->seen[layer].begin(), ctx->seen[layer].end(), 0);
    ctx->seen_count[layer] = 0;
  }
  begin_step(ctx, layer, true);
  return PF_OK;
}

size_t pf_workspace_bytes(const pf_config* cfg) {
  if (check_config(cfg) != PF_OK) return 0;
  return workspace_for(*cfg, kAssumedSms);
}

pf_status pf_set_workspace(pf_ctx* ctx, void* ws, size_t ws_bytes, void* stream) {
  if (!ctx) return PF_ERR_INVALID_ARG;
  if (ws == nullptr) {
    ctx->ws = nullptr;
    ctx->ws_bytes = 0;
    return PF_OK;
  }
  if (!aligned16(ws)) return PF_ERR_ALIGN;
  const size_t cb = counter_bytes(ctx->cfg);
  if (ws_bytes < cb) return PF_ERR_INVALID_ARG;
  cudaError_t e = pf::launch_zero_u32(static_cast<unsigned*>(ws), cb / 4, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return PF_ERR_CUDA;
  ctx->ws = static_cast<uint8_t*>(ws);
  ctx->ws_bytes = ws_bytes;
  const int L = ctx->cfg.n_layers;
  ctx->scat_target.assign(L, 0ull);
  ctx->read_target.assign(L, 0ull);
  ctx->scat_step_start.assign(L, 0ull);
  ctx->read_step_start.assign(L, 0ull);
  ctx->read_before_patch.assign(L, std::vector<unsigned long long>(ctx->cfg.n_patches, 0ull));
  return PF_OK;
}

size_t pf_cfg_workspace_bytes(int batch, int64_t n_per_sample) {
  if (batch < 1 || n_per_sample < 4 || n_per_sample % 4 != 0) return 0;
  return pf::cfg_workspace_bytes(batch, n_per_sample);
}

pf_status pf_cfg_combine_relmae(const float* eps_c, const float* eps_u, int batch,
                                int64_t n_per_sample, float w, float* out_f32,
                                uint16_t* out_bf16, float* relmae, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (!eps_c || !eps_u || !relmae || !workspace) return PF_ERR_INVALID_ARG;
  if (batch < 1 || n_per_sample < 4) return PF_ERR_SHAPE;
  if (n_per_sample % 4 != 0) return PF_ERR_SHAPE;
  if (static_cast<double>(batch) * static_cast<double>(n_per_sample) > 9.0e15) return PF_ERR_SHAPE;
  if (!std::isfinite(w)) return PF_ERR_INVALID_ARG;
  if (!aligned16(eps_c) || !aligned16(eps_u) || (out_f32 && !aligned16(out_f32)) ||
      (out_bf16 && (reinterpret_cast<uintptr_t>(out_bf16) & 7u)) ||
      (reinterpret_cast<uintptr_t>(relmae) & 3u) || !aligned16(workspace))
    return PF_ERR_ALIGN;
  if (workspace_bytes < pf::cfg_workspace_bytes(batch, n_per_sample)) return PF_ERR_INVALID_ARG;
  return from_cuda(pf::launch_cfg_combine_relmae(eps_c, eps_u, batch, n_per_sample, w, out_f32,
                                                 out_bf16, relmae, workspace,
                                                 static_cast<cudaStream_t>(stream)));
}

pf_status pf_cfg_combine_relmae_static(const float* eps_c, const float* eps_u, int batch,
                                       int64_t n_per_sample, float w, float* out_f32,
                                       uint16_t* out_bf16, float* relmae, void* stream) {
  if (!eps_c || !eps_u || !relmae) return PF_ERR_INVALID_ARG;
  if (batch < 1 || n_per_sample < 4) return PF_ERR_SHAPE;
  if (n_per_sample % 4 != 0) return PF_ERR_SHAPE;
  if (batch > pf::cfg_static_capacity_samples()) return PF_ERR_SHAPE;
  if (static_cast<double>(batch) * static_cast<double>(n_per_sample) > 9.0e15) return PF_ERR_SHAPE;
  if (!std::isfinite(w)) return PF_ERR_INVALID_ARG;
  if (!aligned16(eps_c) || !aligned16(eps_u) || (out_f32 && !aligned16(out_f32)) ||
      (out_bf16 && (reinterpret_cast<uintptr_t>(out_bf16) & 7u)) ||
      (reinterpret_cast<uintptr_t>(relmae) & 3u))
    return PF_ERR_ALIGN;
  return from_cuda(pf::launch_cfg_combine_relmae_static(eps_c, eps_u, batch, n_per_sample, w, out_f32,
                                                        out_bf16, relmae,
                                                        static_cast<cudaStream_t>(stream)));
}

pf_status pf_switch_init(pf_switch* s, float enter_below, int enter_patience, float exit_above,
                         int max_parallel_steps) {
  if (!s || !std::isfinite(enter_below) || enter_below < 0.f || std::isnan(exit_above) ||
      exit_above < 0.f || enter_patience < 1)
    return PF_ERR_INVALID_ARG;
  s->enter_below = enter_below;
  s->enter_patience = enter_patience;
  s->exit_above = exit_above;
  s->max_parallel_steps = max_parallel_steps;
  s->phase = PF_PHASE_WARMUP;
  s->step = 0;
  s->below_run = 0;
  s->parallel_steps = 0;
  s->tau1 = -1;
  s->tau2 = -1;
  return PF_OK;
}

pf_status pf_switch_update(pf_switch* s, float relmae, int* phase_out) {
  if (!s || std::isnan(relmae)) return PF_ERR_INVALID_ARG;
  const int t = s->step++;
  switch (s->phase) {
    case PF_PHASE_WARMUP:
      s->below_run = relmae <= s->enter_below ? s->below_run + 1 : 0;
      if (s->below_run >= s->enter_patience) {
        s->phase = PF_PHASE_PARALLEL;
        s->tau1 = t + 1;
      }
      break;
    case PF_PHASE_PARALLEL:
      ++s->parallel_steps;
      if (relmae >= s->exit_above ||
          (s->max_parallel_steps > 0 && s->parallel_steps >= s->max_parallel_steps)) {
        s->phase = PF_PHASE_FULL;
        s->tau2 = t + 1;
      }
      break;
    default:
      break;
  }
  if (phase_out) *phase_out = s->phase;
  return PF_OK;
}

pf_status pf_check_device_status(pf_ctx* ctx, void* stream) {
  if (!ctx) return PF_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PF_ERR_CUDA;
  unsigned v = 0;
  if (pf::read_and_clear_watchdog(&v) != cudaSuccess) return PF_ERR_CUDA;
  return v ? PF_ERR_TIMEOUT : PF_OK;
}

pf_status pf_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return PF_ERR_INVALID_ARG;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (pf::launch_selftest_wait(limit_ns, st) != cudaSuccess) return PF_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PF_ERR_CUDA;
  unsigned v = 0;
  if (pf::read_and_clear_watchdog(&v) != cudaSuccess) return PF_ERR_CUDA;
  return v ? PF_ERR_TIMEOUT : PF_OK;
}

const char* pf_status_string(pf_status s) {
  switch (s) {
    case PF_OK: return "ok";
    case PF_ERR_INVALID_ARG: return "invalid argument";
    case PF_ERR_SHAPE: return "invalid shape";
    case PF_ERR_ALIGN: return "pointer not 16-byte aligned";
    case PF_ERR_UNSUPPORTED: return "unsupported configuration";
    case PF_ERR_ORDER: return "patch out of order";
    case PF_ERR_STATE: return "layer buffer not initialised";
    case PF_ERR_CUDA: return "CUDA error";
    case PF_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

int pf_version(void) { return 100; }

}  // extern "C"
