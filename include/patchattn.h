/*
 * patchattn.h -- C ABI of the B200 (sm_100a) PipeFusion patch-attention library.
 *
 * The library runs, on one GPU, the data path of PipeFusion's patch-level attention
 * ("기술 요약: PipeFusion", 핵심 메커니즘 1-4; "PipeFusion: Patch-level Pipeline Parallelism
 * for Diffusion Transformers Inference", Résumé Technique / Mécanismes Principaux):
 *
 *   - the image tokens of a diffusion step are cut into M non-overlapping patches, here
 *     the contiguous row-major token ranges [p*P, (p+1)*P), P = n_img / M;
 *   - each layer keeps a full-spatial K/V buffer; when patch p of step s is computed,
 *     the buffer rows of patches < p already hold step s (written by the calls for those
 *     patches), the rows of patches > p still hold step s-1 ("stale" activations of the
 *     previous sampler step, 2. 시간적 중복성 활용), and patch p's own rows are
 *     overwritten with the fresh K/V passed to the call;
 *   - the patch's queries then attend to every buffer row plus the step's always-fresh
 *     text tokens (MM-DiT joint attention), softmax(scale * Q K^T) V.
 *
 * and the guidance combine that feeds hybrid-CFG switching ("조건부 가이드 스케줄링 기반
 * 하이브리드 데이터-파이프라인 병렬 처리를 통한 디퓨전 모델 가속화", second block 단락 1-3):
 *   out = eps_u + w * (eps_c - eps_u),  rel-MAE_t = ||eps_c - eps_u||_1 / ||eps_u||_1.
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Memory: the caller owns all device memory (inputs, outputs, K/V buffers, workspace);
 *    the library allocates no device memory.  A pf_ctx holds host state only.
 *  - Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Work is enqueued asynchronously; pointers must stay valid until the
 *    stream has executed it.
 *  - Layout: every attention tensor is contiguous row-major [batch, tokens, heads,
 *    head_dim] bf16 (the natural output of a QKV projection); strides are derived.
 *    All device pointers must be 16-byte aligned (else PF_ERR_ALIGN).
 *  - Errors: every call returns pf_status; nothing aborts and no exception crosses the
 *    ABI.  Argument, shape, order and state errors are detected on the host before any
 *    work is enqueued, and leave the context unchanged.  Launch failures return
 *    PF_ERR_CUDA.  Faults of enqueued work surface at the caller's next stream sync.
 *  - Thread safety: a pf_ctx must not be used from two host threads at once.
 */
#ifndef PATCHATTN_H_
#define PATCHATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PF_OK = 0,
  PF_ERR_INVALID_ARG = 1, /* NULL where a pointer is required, negative size, bad layer/patch */
  PF_ERR_SHAPE = 2,       /* n_img not a multiple of n_patches, zero-sized dimension */
  PF_ERR_ALIGN = 3,       /* a device pointer is not 16-byte aligned */
  PF_ERR_UNSUPPORTED = 4, /* head_dim not in {64, 72, 128}, unknown schedule, a current device
                             that is not compute capability 10.0 (pf_create), or a kernel image
                             whose compiled register count does not fit its register split */
  PF_ERR_ORDER = 5,       /* patch called out of order for the layer's schedule */
  PF_ERR_STATE = 6,       /* step before pf_kvbuf_init of that layer */
  PF_ERR_CUDA = 7,        /* a CUDA runtime/driver call or a kernel launch failed */
  PF_ERR_TIMEOUT = 8      /* a kernel's bounded wait expired (reported by pf_check_device_status) */
} pf_status;

/* Which rows of the other patches a patch sees.
 *  PF_SCHED_PIPEFUSION: this step's rows for patches < p (written by the earlier calls of
 *    the step), stale rows for patches > p.  Patches must be called 0, 1, ..., M-1 per
 *    step, then wrap to 0 for the next step.
 *  PF_SCHED_DISTRIFUSION: every other patch is seen at the previous step (the buffer is
 *    only written after the last patch of the step), the schedule of DistriFusion
 *    ("기술 요약: PipeFusion", 문제 정의: DistriFusion keeps full-spatial stale K/V).
 *    Patches may come in any order, each once per step; the step ends after M calls.
 *  PF_SCHED_PIPEFUSION_2H: the rows PF_SCHED_PIPEFUSION sees, bit for bit, kept in two
 *    buffer halves: the step being computed writes its patches into one half while the
 *    previous step's rows stay in the other, and the halves swap after patch M-1.  Twice
 *    the buffer memory; in exchange a call's scatter never overwrites rows that the
 *    step's earlier calls are still reading, so consecutive calls on one layer overlap on
 *    the GPU (with a workspace, see pf_workspace_bytes).  Patches in order, as PIPEFUSION. */
typedef enum {
  PF_SCHED_PIPEFUSION = 0,
  PF_SCHED_DISTRIFUSION = 1,
  PF_SCHED_PIPEFUSION_2H = 2
} pf_schedule;

typedef struct {
  int batch;           /* B >= 1 */
  int heads;           /* H >= 1 */
  int head_dim;        /* d in {64, 72, 128} */
  int n_img;           /* image tokens N >= 1, multiple of n_patches */
  int n_patches;       /* M >= 1 */
  int n_txt;           /* text tokens T >= 0 */
  int n_layers;        /* L >= 1: one K/V buffer per layer */
  float softmax_scale; /* 0 => 1/sqrt(head_dim) with the real head_dim */
  int schedule;        /* pf_schedule */
} pf_config;

typedef struct pf_ctx pf_ctx; /* opaque, host-only */

/* Bytes of ONE layer's K/V buffer: K region [B, N, H, d] bf16 followed by the V region of
 * the same size (2 * B * N * H * d * 2 bytes); under PF_SCHED_DISTRIFUSION and
 * PF_SCHED_PIPEFUSION_2H a second such [K | V] half follows (the step being written while
 * the other half holds the previous step), twice the bytes.  0 if cfg is NULL or invalid. */
size_t pf_kvbuf_bytes(const pf_config* cfg);

/* Create a context.  kvbuf_per_layer: host array of n_layers device pointers, each to a
 * caller-owned buffer of pf_kvbuf_bytes(cfg) bytes that must outlive the context.
 * On success *out receives the context; on failure *out is set to NULL.
 * If a CUDA device is current and it is not of compute capability 10.0 (the kernels are
 * built for sm_100a only), returns PF_ERR_UNSUPPORTED.  With no usable device at all the
 * context is still created (it is host state only) and its launches return PF_ERR_CUDA. */
pf_status pf_create(const pf_config* cfg, void* const* kvbuf_per_layer, pf_ctx** out);

/* Free the host state of ctx (not the caller's buffers).  NULL => PF_OK. */
pf_status pf_destroy(pf_ctx* ctx);

/* Start-up pass ("기술 요약: PipeFusion", 핵심 메커니즘 2: stale data exists only after the
 * initial start): copy the first step's full-spatial K and V, [B, N, H, d] bf16 each,
 * into layer `layer`'s buffer (with two halves: into the half pf_get_read_half names) and
 * reset that layer's patch counter to 0.  A bit copy. */
pf_status pf_kvbuf_init(pf_ctx* ctx, int layer, const void* k_full, const void* v_full,
                        void* stream);

/* One micro-step: layer `layer`, patch `patch` of the current step.
 *   q_p, k_p, v_p : fresh activations of the patch, [B, P, H, d] bf16
 *   k_txt, v_txt  : this step's text keys/values, [B, T, H, d] bf16 (both NULL iff T == 0)
 *   o_p           : output, [B, P, H, d] bf16, o_p = softmax(scale Q_p [K';K_txt]^T) [V';V_txt]
 *                   where K', V' is the buffer being read with patch p's rows replaced by
 *                   k_p, v_p.
 * The call also writes k_p, v_p into the buffer rows of patch p, fused into the attention
 * kernel: under PF_SCHED_PIPEFUSION into the buffer it reads (later patches of the step see
 * them), under PF_SCHED_DISTRIFUSION and PF_SCHED_PIPEFUSION_2H into the other half, which
 * becomes the half read once all M patches of the step have been called (PIPEFUSION_2H reads
 * the rows of patches < p from that other half).  o_p must not alias any input.
 * Overlap: the attention kernels are launched as programmatic dependents, so when the
 * previous work on the stream is another attention call of this library, this call's grid
 * may start before that one has finished.  It orders itself against it for the buffer, its
 * output and the workspace, but reads its own inputs (q_p, k_p, v_p, k_txt, v_txt) at once:
 * an input must not be the output of the attention call directly before it on the stream
 * (any other kernel in between, or a synchronisation, orders them as usual).
 * Errors: PF_ERR_STATE before pf_kvbuf_init(layer); PF_ERR_ORDER if `patch` is not the
 * layer's next patch (PipeFusion) or was already called this step (DistriFusion);
 * PF_ERR_INVALID_ARG / PF_ERR_ALIGN for bad pointers. */
pf_status pf_patch_attn_step(pf_ctx* ctx, int layer, int patch, const void* q_p,
                             const void* k_p, const void* v_p, const void* k_txt,
                             const void* v_txt, void* o_p, void* stream);

/* Joint attention for the text tokens (MM-DiT, named in "기술 요약: PipeFusion", 중요성 및
 * 주장): the step's text queries attend to the layer's K/V buffer as it stands plus the text
 * keys/values, softmax(scale Q_txt [K_buf;K_txt]^T) [V_buf;V_txt].  Called after the last
 * patch of a step, the buffer holds that step's K/V everywhere.  The buffer is only read
 * and the patch counter is not moved.  "As it stands": under PF_SCHED_PIPEFUSION_2H, the
 * rows of the step's patches called so far and the previous step's rows of the others;
 * under PF_SCHED_DISTRIFUSION, the half being read.
 *   q_txt, k_txt, v_txt, o_txt : [B, T, H, d] bf16 (o_txt must not alias an input; the
 *   inputs must not be the output of the attention call directly before it on the stream,
 *   as for pf_patch_attn_step)
 * Errors: PF_ERR_SHAPE if the configuration has no text tokens; PF_ERR_STATE before
 * pf_kvbuf_init(layer). */
pf_status pf_text_attn_step(pf_ctx* ctx, int layer, const void* q_txt, const void* k_txt,
                            const void* v_txt, void* o_txt, void* stream);

/* Per-head RMS normalisation of queries or keys, in place (the QK-norm of Flux-style DiTs):
 * each head_dim vector x becomes x / sqrt(mean(x^2) + eps) * gain, computed in fp32 and
 * rounded to bf16.
 *   x         : device bf16, n_vectors contiguous vectors of head_dim elements
 *               (e.g. [B, tokens, H, d] with n_vectors = B * tokens * H), 16-byte aligned
 *   gain      : device bf16 [head_dim], or NULL for a gain of 1
 *   eps       : > 0
 * head_dim must be a multiple of 8 and at most 256. */
pf_status pf_qk_rmsnorm(void* x, int64_t n_vectors, int head_dim, const void* gain, float eps,
                        void* stream);

/* Bytes of the optional attention workspace for this configuration (0 if cfg is invalid, or
 * if no call of the configuration would split).  With a workspace set, a call may split each
 * query tile's key range over several CTAs so that the grid fills the GPU's SMs in near-whole
 * waves; the parts are merged exactly in the log-sum-exp sense (rescaled by their row maxima)
 * by the last part to finish.  The workspace also holds per-layer ordering counters: a call
 * reads a layer's buffer rows once the earlier calls that wrote them have scattered, and
 * scatters once the earlier calls that read the rows it overwrites have finished reading
 * (with two buffer halves, the calls up to the previous step's call for the same patch), so
 * consecutive calls of one stream overlap on the GPU (without a workspace, each call waits
 * for the previous one before it touches the buffer). */
size_t pf_workspace_bytes(const pf_config* cfg);

/* Attach a caller-owned device workspace (16-byte aligned, >= pf_workspace_bytes(cfg))
 * to ctx and zero its counters on `stream`.  ws = NULL detaches it (no key-range split).
 * A workspace belongs to one context (its ordering counters are counted against that
 * context's host-side totals), and the calls of a context run on one stream.  After
 * PF_ERR_TIMEOUT, set the workspace again to re-zero the counters. */
pf_status pf_set_workspace(pf_ctx* ctx, void* ws, size_t ws_bytes, void* stream);

/* Next patch index the layer expects (0 at the start of a step).  Checkpoint helper: a
 * layer's whole state is its buffer contents plus this counter. */
pf_status pf_get_state(const pf_ctx* ctx, int layer, int* next_patch);

/* Restore a counter saved with pf_get_state (the caller restores the buffer contents).
 * Under the two-half schedules only the start of a step (next_patch 0) can be restored
 * (else PF_ERR_UNSUPPORTED); the caller restores the half pf_get_read_half names. */
pf_status pf_set_state(pf_ctx* ctx, int layer, int next_patch);

/* Which half of the layer's buffer holds the previous step's rows (the half read for the
 * patches not yet called in this step): 0 or 1 under PF_SCHED_DISTRIFUSION and
 * PF_SCHED_PIPEFUSION_2H, where the halves swap after each step's last patch; always 0
 * under PF_SCHED_PIPEFUSION.  Errors: PF_ERR_INVALID_ARG for a bad layer or pointer. */
pf_status pf_get_read_half(const pf_ctx* ctx, int layer, int* half);

/* Workspace bytes pf_cfg_combine_relmae needs for `batch` samples of `n_per_sample`
 * floats (0 on invalid sizes). */
size_t pf_cfg_workspace_bytes(int batch, int64_t n_per_sample);

/* Guidance combine + rel-MAE_t, fused in one pass over eps_c and eps_u.
 *   eps_c, eps_u : device fp32 [batch, n_per_sample] (any [B, C, H, W] flattened per sample)
 *   w            : guidance weight
 *   out_f32      : device fp32 [batch, n_per_sample] = eps_u + w (eps_c - eps_u), or NULL
 *   out_bf16     : device bf16 (uint16 bits) same shape, round-to-nearest-even of the fp32
 *                  result, or NULL
 *   relmae       : device fp32 [batch]: per-sample ||eps_c - eps_u||_1 / ||eps_u||_1
 *                  (0 if both norms are 0, +inf if only the denominator is 0)
 *   workspace    : device scratch of pf_cfg_workspace_bytes(batch, n_per_sample) bytes,
 *                  no initialisation needed; one workspace per concurrently running call
 * The reduction is deterministic (fixed order, no float atomics): equal inputs give
 * bitwise-equal outputs.  n_per_sample must be a multiple of 4 (16-byte rows). */
pf_status pf_cfg_combine_relmae(const float* eps_c, const float* eps_u, int batch,
                                int64_t n_per_sample, float w, float* out_f32,
                                uint16_t* out_bf16, float* relmae, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Same computation and outputs as pf_cfg_combine_relmae, for callers that cannot allocate
 * device memory: code that runs where another framework owns the device allocator and must
 * see every allocation, or loops that cannot afford the device synchronisation a cudaMalloc
 * may imply.  The pages have no counterpart of this entry point; it is a deployment
 * convenience.
 *
 * The partial sums go to a fixed 64 KiB array inside the library's device image (4096
 * partial-sum pairs) instead of a caller workspace, so the call allocates nothing and takes
 * no workspace argument.  Limit: batch <= 4096 samples; a larger batch returns PF_ERR_SHAPE.
 * Every GPU that loads the library holds the array until the process exits.
 *
 * Set-up: the first call on each device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream capture.
 * The array is shared by all calls and keeps the last call's contents; nothing in it needs
 * to start at zero (each call writes every slot it reads).  Calls whose work overlaps on the
 * GPU (different streams, or different host threads) race on the array: serialise them.
 * Errors as for pf_cfg_combine_relmae; PF_ERR_CUDA if the address lookup fails. */
pf_status pf_cfg_combine_relmae_static(const float* eps_c, const float* eps_u, int batch,
                                       int64_t n_per_sample, float w, float* out_f32,
                                       uint16_t* out_bf16, float* relmae, void* stream);

/* Hybrid-CFG adaptive switching ("조건부 가이드 스케줄링 기반 하이브리드 데이터-파이프라인 병렬 처리를
 * 통한 디퓨전 모델 가속화", second block 단락 2-3): the denoising steps are divided into
 * Warm-Up, Parallelism and Fully-Connecting; the switch points tau1 and tau2 follow rel-MAE_t,
 * and parallelism is active while rel-MAE_t has settled below a threshold.  The pages give
 * no threshold values, so they are parameters:
 *   - Warm-Up -> Parallelism (tau1) once rel-MAE_t <= enter_below for enter_patience
 *     consecutive steps;
 *   - Parallelism -> Fully-Connecting (tau2) once rel-MAE_t >= exit_above, or after
 *     max_parallel_steps parallel steps (<= 0: no limit).  Fully-Connecting is final.
 * Host-only state, no allocation; one pf_switch per image (rel-MAE_t is per sample). */
typedef enum { PF_PHASE_WARMUP = 0, PF_PHASE_PARALLEL = 1, PF_PHASE_FULL = 2 } pf_phase;

typedef struct {
  float enter_below;
  int enter_patience;
  float exit_above;
  int max_parallel_steps;
  int phase;          /* pf_phase that applies to the next step */
  int step;           /* steps observed so far */
  int below_run;      /* consecutive steps with rel-MAE_t <= enter_below */
  int parallel_steps; /* steps spent in Parallelism */
  int tau1, tau2;     /* step indices where the phase changed (-1 until then) */
} pf_switch;

/* Initialise a controller (phase Warm-Up).  PF_ERR_INVALID_ARG for NULL, a non-finite or
 * negative threshold, or enter_patience < 1. */
pf_status pf_switch_init(pf_switch* s, float enter_below, int enter_patience, float exit_above,
                         int max_parallel_steps);

/* Feed rel-MAE_t of the step just finished; *phase_out (may be NULL) receives the phase for
 * the next step.  NaN rel-MAE_t is rejected with PF_ERR_INVALID_ARG and leaves the state. */
pf_status pf_switch_update(pf_switch* s, float relmae, int* phase_out);

/* Synchronise `stream`, then read the device status word the kernels write when a bounded
 * wait expires: PF_ERR_TIMEOUT if any did (and clear it), PF_ERR_CUDA if the stream reported
 * an error, else PF_OK.  The status word is one per device and process, shared by every
 * context and stream of the process on that device (the context argument only guards
 * against NULL): a timeout in any of them is reported, and cleared, by whichever call reads
 * the word first. */
pf_status pf_check_device_status(pf_ctx* ctx, void* stream);

/* Self-test of failure detection (the pages have no counterpart): launches a one-thread
 * kernel whose mbarrier wait is never satisfied, so its bounded wait gives up after
 * limit_ns (1 ns .. 10 s), sets its bit in the device status word and returns -- the path
 * every role of the attention kernel takes when a wait expires, without faulting or hanging
 * the device.  Synchronises `stream`, then reads and clears the status word.  Returns
 * PF_ERR_TIMEOUT when the wait gave up as designed (PF_OK would mean it did not), PF_ERR_CUDA
 * on a CUDA error, PF_ERR_INVALID_ARG for a limit out of range.  Shares the status word with
 * the other kernels: do not run it while attention launches are in flight. */
pf_status pf_selftest_bounded_wait(uint64_t limit_ns, void* stream);

/* Static description of a status code (never NULL). */
const char* pf_status_string(pf_status s);

/* Library version: major * 10000 + minor * 100 + patch. */
int pf_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PATCHATTN_H_ */
