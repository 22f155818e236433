// attn_fwd.cu -- fused KV-buffer scatter + patch attention for sm_100a (B200).
//
// One launch runs one PipeFusion micro-step ("기술 요약: PipeFusion", 핵심 메커니즘 1-3):
// the queries of patch p attend to the layer's full-spatial K/V context, in which patch
// p's own rows are the fresh K_p/V_p of the call, the other image rows come from the
// layer buffer (this step's rows for earlier patches, the previous step's for later
// ones), and the step's text tokens are appended (joint attention).  The same launch
// writes K_p/V_p into the buffer rows of patch p for the calls that follow.
//
// Two kernels, one per head_dim class, share the rest of the design below:
//   patch_attn_sn_kernel (head_dim 72, 128): one softmax thread per query row; each
//     128-key tile is handled as two 64-key halves so that the tensor core runs PV and the
//     next QK of one half while the softmax exponentiates the other;
//   patch_attn_hr_kernel (head_dim 64): two softmax threads per query row (each half of the
//     key tile), four softmax warps per SM sub-partition, for the exponential-bound case.
// A CTA handles one head of one batch element and NQ (1 or 2) tiles of 128 query rows.
// Warp roles: softmax warps (one TMEM lane quarter each), one single-thread tcgen05.mma
// issuer per query tile, a TMA producer (Q once, then K/V tiles through a shared-memory
// ring), and a scatter warp that copies the CTA's share of K_p/V_p into the buffer.
// S = Q K^T lands in TMEM (fp32); P is written back to TMEM as packed bf16 and the PV MMA
// reads it from there (A operand in TMEM, V as an MN-major B operand in shared memory); O
// accumulates in TMEM.
// The context is walked as segments so that patch p's rows are read from the fresh
// tensors, never from buffer rows that other CTAs of this launch are writing:
//   [fresh rows 0..P) | text rows 0..T) | buffer rows (p+1)P..N) | buffer rows 0..pP)
// The call's own tensors come first and the rows that the step's earlier calls wrote
// come last, so a launch has the most work it can do before those calls' writes must be
// complete.  Softmax is permutation invariant over keys, so this order gives the same
// result as the natural token order.  Row maxima are kept lazily: O is rescaled only when a row's
// maximum grows by more than 2^8, which is exact because the final O / l uses the same
// reference maximum for numerator and denominator.
//
// Work decomposition: one CTA per (pair, part), where a pair is one (batch, head, group of
// NQ query tiles) and its context tiles may be split into n_split contiguous parts (the
// host picks n_split for launches that overlap their neighbours).  Every part of a split
// writes its unnormalised O row with its reference maximum m and sum l to a workspace slot;
// the last part of a query tile to arrive (an atomic counter decides) waits, bounded, for
// the others' slots -- they have all arrived, so they are running -- and merges all parts
// in part order, O = sum_i 2^(m_i - M) O_i / sum_i 2^(m_i - M) l_i, into the bf16 output.
//
// Ordering between launches: with a workspace, calls on one layer buffer are ordered by two
// per-layer counters in global memory instead of by the completion of the previous grid, so
// that launches overlap: CTAs that finished their scatter share and CTAs that finished
// reading the buffer, each counted in call order, so that a counter reaching the host's total
// for a prefix of the calls means that prefix is done.  Before its buffer rows a launch waits
// for the scatters of the calls that wrote them; a scatter waits for the reads of the calls
// that read the rows it overwrites.  With a single buffer half those are all earlier calls.
// With two halves (the step being written goes to the other half) the rows of patch p in the
// half being written were last read by the calls before patch p of the previous step, so
// consecutive calls of a step wait on each other only where a call reads rows that the
// step's earlier calls wrote (its lo rows, walked last).
//
// Every wait is bounded (2 s); on expiry the kernel records the role in a device word,
// raises a CTA-wide abort flag, drains its in-flight copies and MMAs, frees TMEM and
// returns.

#include <cuda_bf16.h>

#include <mutex>

#include "pf_internal.h"
#include "sm100_ptx.cuh"

namespace pf {

__device__ unsigned int g_watchdog = 0;

#ifdef PF_TRACE
// Profiling build only: SM-cycle timestamps of CTA 0, [event][query tile][context tile].
// Events: 0 softmax sees S, 1 softmax has published P, 2 MMA issuer sees P,
// 3 MMA issuer has committed S, 4 MMA issuer sees the K tile, 5 softmax has S in
// registers, 6 softmax has the row maximum, 7 softmax has P packed, 8 P stored to TMEM.
constexpr int kTraceTiles = 512;
// 9 MMA issuer sees the V tile of j-1, 10 producer issued the K (t=0) / V (t=1) tile j.
// The second index is the softmax chain: the query tile (full-row kernels) or 2 * query tile
// + key half (half-row kernel).
__device__ unsigned long long g_trace[16 * 4 * kTraceTiles];
// Per CTA of the latest launch: SM id, start and end (global timer, ns).
constexpr int kTraceCtas = 4096;
__device__ unsigned long long g_cta[3 * kTraceCtas];
#define PF_TRACE_CTA(slot)                                                                 \
  do {                                                                                     \
    if (threadIdx.x == 0 && blockIdx.x < kTraceCtas) {                                     \
      unsigned smid;                                                                       \
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));                                    \
      g_cta[3 * blockIdx.x] = smid;                                                        \
      g_cta[3 * blockIdx.x + (slot)] = globaltimer_ns();                                   \
    }                                                                                      \
  } while (0)
#define PF_TRACE_AT(ev, t, j)                                                              \
  do {                                                                                     \
    if (blockIdx.x == 0 && (j) < kTraceTiles) g_trace[((ev) * 4 + (t)) * kTraceTiles + (j)] = clock64(); \
  } while (0)
// Per CTA, seen by thread 0 (a softmax thread of query tile 0), global timer ns: 0 set-up
// done, 1 S of the first context tile seen, 2 O complete, 3 partial stored and fenced, 4
// the last part is known, 5 merge done.
__device__ unsigned long long g_cta_ev[8 * kTraceCtas];
#define PF_TRACE_EV(slot)                                                                  \
  do {                                                                                     \
    if (threadIdx.x == 0 && blockIdx.x < kTraceCtas) g_cta_ev[8 * blockIdx.x + (slot)] = globaltimer_ns(); \
  } while (0)
#else
#define PF_TRACE_EV(slot) \
  do {                    \
  } while (0)
#define PF_TRACE_AT(ev, t, j) \
  do {                        \
  } while (0)
#define PF_TRACE_CTA(slot) \
  do {                     \
  } while (0)
#endif

namespace {

using namespace ptx;

constexpr int kRows = 128;             // query rows per Q tile == key rows per K/V tile
constexpr int kChunkBytes = 128 * 128; // 128 rows x 64 bf16 columns (one 128-byte swizzle span)
constexpr int kThreads = 384;          // 3 warpgroups: softmax 0, softmax 1, MMA/TMA/scatter
// Register split of patch_attn_sn_kernel (setmaxnreg): __launch_bounds__(kThreads, 1) lets
// the compiler use up to kLaunchRegs = 168 per thread (384 x 168 = 64512 of the SM's 65536),
// the third warpgroup drops to 88 and the two softmax warpgroups rise to 208:
// 128 x 88 + 256 x 208 = 64512, exactly the registers the CTA is launched with.
// setmaxnreg.inc waits until the CTA's pool can give the registers, so a kernel compiled to
// fewer registers than the split assumes would wait forever: the host reads the compiled
// count before the first launch on each device and refuses to launch when the split does not
// fit (sn_configure_once, hr_configure_once).
constexpr int kLaunchRegs = (65536 / kThreads) / 8 * 8;
constexpr uint32_t kRegsSoftmax = 208;
constexpr uint32_t kRegsOther = 88;
static_assert(128 * kRegsOther + 256 * kRegsSoftmax <= kThreads * kLaunchRegs, "register split");
constexpr int kWarpMma = 8;     // TMEM allocation; MMA issuer of query tile 0
constexpr int kWarpMma2 = 11;   // MMA issuer of query tile 1
constexpr int kWarpLoad = 9;
constexpr int kWarpScatter = 10;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;        // split-tile kernel: O_t at column 256 + 128 t, S_t at 128 t
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kMaxSplit = 16;          // most key-range parts per query tile

enum : unsigned { kWdLoad = 1u, kWdMma = 2u, kWdSoftmax = 4u, kWdEpilogue = 8u, kWdSelftest = 16u,
                  kWdScatter = 32u };

template <int D>
struct Dims {
  static constexpr int kChunks = (D + 63) / 64;          // 64-column chunks per row
  static constexpr int kMmaN = (D + 15) / 16 * 16;       // head_dim padded to 16 (72 -> 80)
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = D <= 64 ? 8 : 4;
};

template <int D, int NQ>
constexpr int smem_bytes() {
  return 1024 + (NQ + Dims<D>::kStages) * Dims<D>::kTileBytes + 512;
}

// Which tensor and rows the j-th 128-row context tile comes from.
struct Segments {
  int n_fresh, n_lo, n_hi, n_txt;  // tiles per segment
  int plen, lo_len, hi_row0, hi_len, txt_len;

  __device__ void init(const AttnParams& p) {
    plen = p.fresh_rows;
    lo_len = p.lo_len;
    hi_row0 = p.hi_row0;
    hi_len = p.hi_len;
    txt_len = p.n_txt;
    n_fresh = (plen + kRows - 1) / kRows;
    n_lo = (lo_len + kRows - 1) / kRows;
    n_hi = (hi_len + kRows - 1) / kRows;
    n_txt = (txt_len + kRows - 1) / kRows;
  }
  __device__ int total() const { return n_fresh + n_lo + n_hi + n_txt; }
  // Segment k in walk order (fresh, text, hi, lo): its last tile index + 1 and its rows.
  __device__ void bounds(int k, int& end, int& len) const {
    const int n[4] = {n_fresh, n_txt, n_hi, n_lo};
    const int r[4] = {plen, txt_len, hi_len, lo_len};
    end = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (i <= k) end += n[i];
    len = r[k];
  }
  // src: 0 = fresh tensors, 2 = text, 3 = buffer rows from hi_row0 (bounded by the end of
  // the buffer), 1 = buffer rows [0, lo_len) through the maps bounded at lo_len (a ragged
  // last tile reads zeros past the segment, never the rows of patch p that the scatter of
  // this launch is writing)
  __device__ void tile(int j, int& src, int& row0, int& nvalid) const {
    if (j < n_fresh) {
      src = 0; row0 = j * kRows; nvalid = min(kRows, plen - row0); return;
    }
    j -= n_fresh;
    if (j < n_txt) {
      src = 2; row0 = j * kRows; nvalid = min(kRows, txt_len - row0); return;
    }
    j -= n_txt;
    if (j < n_hi) {
      src = 3; row0 = hi_row0 + j * kRows; nvalid = min(kRows, hi_len - j * kRows); return;
    }
    j -= n_hi;
    src = 1; row0 = j * kRows; nvalid = min(kRows, lo_len - row0);
  }
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo
  return *reinterpret_cast<uint32_t*>(&v);
}

// O row chunk of 16 fp32 columns (c0 .. c0+15) -> bf16, scaled by inv; columns >= D dropped.
template <int D>
__device__ __forceinline__ void store_row16(uint16_t* dst, int c0, const uint32_t (&o)[16], float inv,
                                            bool in_range) {
  uint4 w0, w1;
  w0.x = pack_bf16(__uint_as_float(o[0]) * inv, __uint_as_float(o[1]) * inv);
  w0.y = pack_bf16(__uint_as_float(o[2]) * inv, __uint_as_float(o[3]) * inv);
  w0.z = pack_bf16(__uint_as_float(o[4]) * inv, __uint_as_float(o[5]) * inv);
  w0.w = pack_bf16(__uint_as_float(o[6]) * inv, __uint_as_float(o[7]) * inv);
  w1.x = pack_bf16(__uint_as_float(o[8]) * inv, __uint_as_float(o[9]) * inv);
  w1.y = pack_bf16(__uint_as_float(o[10]) * inv, __uint_as_float(o[11]) * inv);
  w1.z = pack_bf16(__uint_as_float(o[12]) * inv, __uint_as_float(o[13]) * inv);
  w1.w = pack_bf16(__uint_as_float(o[14]) * inv, __uint_as_float(o[15]) * inv);
  if (in_range) {
    if (c0 + 8 <= D) *reinterpret_cast<uint4*>(dst + c0) = w0;
    if (c0 + 16 <= D) *reinterpret_cast<uint4*>(dst + c0 + 8) = w1;
  }
}

// Merging the key-range parts of one query row.  Part i's slot holds, column-major with
// kRows rows per column, the unnormalised O row (d columns) and then m_i and l_i; row0
// points at this row's entry of part 0's slot.  The merged row is
//   O = sum_i 2^(m_i - mref) O_i / sum_i 2^(m_i - mref) l_i,   mref = max_i m_i
// (log-sum-exp combination of softmax parts), summed in part order whichever part merges.
// The slots sit in L2, written by other CTAs, so the merge is bound by L2 round trips: loads
// are issued for four parts at a time (and for the O row, 16 columns of all four) before any
// of them is used.
constexpr int kMergeGroup = 4;

__device__ __forceinline__ void merge_stats(const float* row0, size_t slot_elems, int d, int n_split,
                                            float& mref, float& inv) {
  float mr = -INFINITY, ls = 0.f;
  for (int i0 = 0; i0 < n_split; i0 += kMergeGroup) {
    float mv[kMergeGroup], lv[kMergeGroup];
#pragma unroll
    for (int g = 0; g < kMergeGroup; ++g) {
      const bool on = i0 + g < n_split;
      const float* si = row0 + static_cast<size_t>(i0 + g) * slot_elems;
      mv[g] = on ? __ldcg(si + static_cast<size_t>(d) * kRows) : -INFINITY;
      lv[g] = on ? __ldcg(si + static_cast<size_t>(d + 1) * kRows) : 0.f;
    }
    float mn = mr;
#pragma unroll
    for (int g = 0; g < kMergeGroup; ++g) mn = fmaxf(mn, mv[g]);
    ls *= ex2(mr - mn);  // 0 on the first group (mr = -inf); every part's m is finite
#pragma unroll
    for (int g = 0; g < kMergeGroup; ++g) ls += ex2(mv[g] - mn) * lv[g];  // absent parts add 0
    mr = mn;
  }
  mref = mr;
  inv = 1.f / ls;
}

// Columns c_begin .. c_begin + NCOLS - 1 of the merged row to bf16 at dst (which points at
// column c_begin of the output row), CB at a time.  NCOLS and CB are multiples of 8.
template <int NCOLS, int CB = 16>
__device__ __forceinline__ void merge_columns(const float* row0, size_t slot_elems, int d, int n_split,
                                              int c_begin, float mref, float inv, uint16_t* dst,
                                              bool in_range) {
  static_assert(NCOLS % 8 == 0 && CB % 8 == 0, "whole 16-byte stores");
#pragma unroll
  for (int cb = 0; cb < NCOLS; cb += CB) {
    const int nc = NCOLS - cb < CB ? NCOLS - cb : CB;  // constant once unrolled
    float acc[CB];
#pragma unroll
    for (int k = 0; k < CB; ++k) acc[k] = 0.f;
    for (int i0 = 0; i0 < n_split; i0 += kMergeGroup) {
      float v[kMergeGroup][CB], mv[kMergeGroup];
#pragma unroll
      for (int g = 0; g < kMergeGroup; ++g) {
        const bool on = i0 + g < n_split;
        const float* si = row0 + static_cast<size_t>(i0 + g) * slot_elems;
        mv[g] = on ? __ldcg(si + static_cast<size_t>(d) * kRows) : -INFINITY;
#pragma unroll
        for (int k = 0; k < CB; ++k)
          if (k < nc) v[g][k] = on ? __ldcg(si + static_cast<size_t>(c_begin + cb + k) * kRows) : 0.f;
      }
#pragma unroll
      for (int g = 0; g < kMergeGroup; ++g) {
        const float w = ex2(mv[g] - mref) * inv;
#pragma unroll
        for (int k = 0; k < CB; ++k)
          if (k < nc) acc[k] = fmaf(w, v[g][k], acc[k]);
      }
    }
    if (in_range) {
#pragma unroll
      for (int k = 0; k < CB; k += 8) {
        if (k < nc) {
          uint4 w0;
          w0.x = pack_bf16(acc[k + 0], acc[k + 1]);
          w0.y = pack_bf16(acc[k + 2], acc[k + 3]);
          w0.z = pack_bf16(acc[k + 4], acc[k + 5]);
          w0.w = pack_bf16(acc[k + 6], acc[k + 7]);
          *reinterpret_cast<uint4*>(dst + cb + k) = w0;
        }
      }
    }
  }
}

// Barrier among the `count` threads of one softmax warpgroup (ids 1 and 2; 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Barrier among `count` threads that also ANDs a predicate over them: every participant
// gets the same answer, so a warpgroup agrees on whether to take a path with barriers.
__device__ __forceinline__ bool named_bar_and(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// 2^x on the FMA pipe: x = n + f with n = round(x) (1.5 * 2^23 shifter), 2^f from a
// degree-3 polynomial fitted on [-1/2, 1/2] for least maximum relative error (7.5e-5,
// Lawson's iteratively reweighted least squares), and n added to the exponent field.
// x is clamped to >= -125 so the result stays normal; callers never pass masked (-inf)
// logits here.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  const float2 sh = make_float2(12582912.f, 12582912.f);
  const float2 t = __fadd2_rn(x, sh);                                     // 1.5 * 2^23 + round(x)
  const float2 r = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));  // round(x), exact
  const float2 f = __ffma2_rn(r, make_float2(-1.f, -1.f), x);             // x - round(x), exact
  float2 p = __ffma2_rn(make_float2(0.05517132f, 0.05517132f), f, make_float2(0.24261054f, 0.24261054f));
  p = __ffma2_rn(p, f, make_float2(0.69326097f, 0.69326097f));
  p = __ffma2_rn(p, f, make_float2(0.99992812f, 0.99992812f));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// Of every 8 pairs of columns, the pairs whose exponentials run on the FMA pipe instead of
// the special-function unit.  The polynomial costs about 5 issue slots per element against
// 1 for the unit (16 results/clk/SM); measured over 0..4 of 8, 2 of 8 was fastest for both
// head_dim 64 and 128.
template <int D>
constexpr int kPolyPairs = 2;

__device__ __forceinline__ void raise_abort(volatile int* abort, unsigned code) {
  *abort = 1;
  atomicOr(&g_watchdog, code);
}

// The scatter warp's work: this CTA's contiguous 1/gridDim share of the flattened
// [B, P, H, d] fresh K and V, copied into the buffer rows of the patch (16-byte vectors,
// two in flight per lane).  Nothing when the call has no scatter (k_dst == nullptr).
template <int D>
__device__ __forceinline__ void scatter_share(const AttnParams& p, int lane) {
  if (p.k_dst == nullptr) return;
  // scatters go in call order, and earlier calls read these buffer rows: wait until every
  // earlier scatter is done and every CTA of those calls has finished reading (or, without
  // counters, for the previous grid)
  if (p.dep_scat != nullptr) {
    if (!wait_count_geq64(p.dep_scat, p.dep_scat_target, nullptr, kWaitNs) ||
        !wait_count_geq64(p.dep_read, p.dep_war_target, nullptr, kWaitNs)) {
      if (lane == 0) atomicOr(&g_watchdog, kWdScatter);
      return;
    }
  } else {
    grid_dep_wait();
  }
  const long long per_b = static_cast<long long>(p.plen) * p.heads * D / 8;  // 16-byte vectors
  const long long total = per_b * p.batch;
  const long long lo = total * blockIdx.x / gridDim.x;
  const long long hi = total * (blockIdx.x + 1) / gridDim.x;
  const long long img_b = static_cast<long long>(p.n_img) * p.heads * D / 8;
  const long long patch_off = static_cast<long long>(p.patch) * per_b;
  const uint4* ksrc = reinterpret_cast<const uint4*>(p.k_p);
  const uint4* vsrc = reinterpret_cast<const uint4*>(p.v_p);
  uint4* kdst = reinterpret_cast<uint4*>(p.k_dst);
  uint4* vdst = reinterpret_cast<uint4*>(p.v_dst);
  // walk the share one batch element at a time: within one, the destination is the source
  // index shifted by a constant
  for (long long bb = lo / per_b; bb * per_b < hi; ++bb) {
    const long long b_lo = bb * per_b > lo ? bb * per_b : lo;
    const long long b_hi = (bb + 1) * per_b < hi ? (bb + 1) * per_b : hi;
    const long long shift = bb * (img_b - per_b) + patch_off;
    for (long long base = b_lo + lane; base < b_hi; base += 32 * 2) {
      const long long i1 = base + 32;
      const uint4 k0 = __ldg(ksrc + base), v0 = __ldg(vsrc + base);
      uint4 k1, v1;
      if (i1 < b_hi) {
        k1 = __ldg(ksrc + i1);
        v1 = __ldg(vsrc + i1);
      }
      kdst[base + shift] = k0;
      vdst[base + shift] = v0;
      if (i1 < b_hi) {
        kdst[i1 + shift] = k1;
        vdst[i1 + shift] = v1;
      }
    }
  }
  if (p.dep_scat != nullptr) {
    // this CTA's share is in the buffer: count it for later calls on the layer
    __threadfence();
    __syncwarp();
    if (lane == 0) count_release(p.dep_scat);
  }
}

// The producer's wait before its first tile of buffer rows of one kind: hi rows (src 3) and
// lo rows (src 1) each have the scatter count the host gave for the calls that wrote them
// (with two buffer halves the hi rows were written in earlier steps, the lo rows by the
// step's earlier calls).  Without counters, one wait for the previous grid covers both.
// False when a bounded wait gave up.
__device__ __forceinline__ bool buffer_rows_ready(const AttnParams& p, int src, bool& hi_done,
                                                  bool& lo_done, const volatile int* abort) {
  if (p.dep_scat == nullptr) {
    if (!hi_done && !lo_done) grid_dep_wait();
    hi_done = lo_done = true;
    return true;
  }
  if (src == 3 && !hi_done) {
    if (!wait_count_geq64(p.dep_scat, p.dep_hi_target, abort, kWaitNs)) return false;
    hi_done = true;
  }
  if (src == 1 && !lo_done) {
    if (!wait_count_geq64(p.dep_scat, p.dep_lo_target, abort, kWaitNs)) return false;
    lo_done = true;
  }
  return true;
}

// Count this CTA's finished reads (after its copies have landed), once every CTA of the
// layer's earlier calls has counted its own: the counter then passes the total of a prefix of
// the calls only when exactly that prefix has finished reading.
__device__ __forceinline__ void count_reads_done(const AttnParams& p) {
  if (p.dep_read == nullptr) return;
  if (!wait_count_geq64(p.dep_read, p.dep_read_target, nullptr, kWaitNs)) {
    atomicOr(&g_watchdog, kWdLoad);
    return;
  }
  count_release(p.dep_read);
}

// After the merge, the partial slots of a query tile ([part][d + 2][128] fp32) are dead: the next launch writes every slot before it reads one.  Dropping their L2 lines
// keeps them from being written back to DRAM.  `tid` / `nthreads` split the lines among the
// merging threads.
// Which (pair, part) a CTA computes.  CTAs are numbered (batch x head, part, query-tile
// group): the query-tile groups of one head that read the same key range are neighbours, so
// they run in the same wave and read each context tile from DRAM about once while it sits in
// L2; where a wave ends inside a head, only the key range of one part is read twice (the
// waves of a launch rarely hold whole heads).  The parts of a pair are n_groups CTAs apart,
// within one wave for all but the CTAs at a wave's end, so the last part usually merges
// partials that are still in L2.
struct CtaWork {
  int pair, part, grp, hd, b;
};
__device__ __forceinline__ CtaWork cta_work(const AttnParams& p) {
  const int per_bh = p.n_groups * p.n_split;
  const int bh = static_cast<int>(blockIdx.x) / per_bh;
  const int rem = static_cast<int>(blockIdx.x) - bh * per_bh;
  CtaWork w;
  w.part = rem / p.n_groups;
  w.grp = rem - w.part * p.n_groups;
  w.pair = bh * p.n_groups + w.grp;
  w.hd = bh % p.heads;
  w.b = bh / p.heads;
  return w;
}

// After a merge: mark every part's slot of the query tile dead in L2, so the partials are
// dropped instead of written back to DRAM.
template <int D>
__device__ __forceinline__ void discard_partials(const float* slot0, int n_split, int tid, int nthreads) {
  static_assert((D + 2) * kRows * 4 % 128 == 0, "slots are whole 128-byte lines");
  const char* base = reinterpret_cast<const char*>(slot0);
  // the workspace only has to be 16-byte aligned: skip when the lines are not whole
  if ((reinterpret_cast<uintptr_t>(base) & 127u) != 0) return;
  const int lines = n_split * (D + 2) * kRows * 4 / 128;
  for (int i = tid; i < lines; i += nthreads) discard_l2_line(base + static_cast<size_t>(i) * 128);
}

// ------------------------------------------------------------------ head_dim 64: half rows
//
// With head_dim 64 a key tile costs the tensor core half of what it costs at 128 while the
// softmax still exponentiates 128 x 128 scores per query tile, so the exponentials, not the
// MMAs, bound the loop; with one thread per query row there are only two softmax warps per
// SM sub-partition to keep the special-function unit busy, and each runs a long dependent
// chain.  Here every query row is shared by two threads: half 0 of a query tile's softmax
// warps takes keys 0..63 of each key tile, half 1 keys 64..127, so four softmax warps run
// per sub-partition.  The two threads of a row keep one reference maximum m (they exchange
// their half-tile maxima through shared memory once per tile, behind a 64-thread barrier
// that also carries their agreement on aborting), one O accumulator in TMEM (each half
// rescales 32 of its 64 columns) and a row sum each, added once at the end.
//
// TMEM, per query tile t (256 columns at 256 t): S (128 fp32 columns) | O (64) | P_0 (32) |
// P_1 (32): P (packed bf16) has its own columns, so QK(j+1) is issued (one N = 128 MMA
// chain) as soon as every softmax warp of the tile has S(j) in registers and runs while
// they exponentiate.  P(j) may overwrite P(j-1) only after PV(j-1) has read it: QK(j+1) was
// issued by the same thread after PV(j-1), so S(j+1) being complete implies it (the last
// tile waits for the PV itself).
//
// Warps: 0-15 softmax (warp w: query tile w / 8, half (w / 4) % 2, TMEM lane quarter w % 4),
// 16 TMEM allocation + MMA issuer of query tile 0, 17 TMA producer, 18 scatter, 19 MMA
// issuer of query tile 1.  Named barriers: 1 + 4 t + quarter (the two warps of a row
// quarter, 64 threads), 9 + t (the 256 softmax threads of query tile t).
constexpr int kHrThreads = 640;
constexpr int kHrLaunchRegs = (65536 / kHrThreads) / 8 * 8;  // 96
constexpr uint32_t kHrRegsSoftmax = 104;
constexpr uint32_t kHrRegsOther = 56;
static_assert(128 * kHrRegsOther + 512 * kHrRegsSoftmax <= kHrThreads * kHrLaunchRegs, "register split");
constexpr int kHrWarpMma0 = 16;
constexpr int kHrWarpLoad = 17;
constexpr int kHrWarpScatter = 18;
constexpr int kHrWarpMma1 = 19;
constexpr int kHrStages = 8;
constexpr int kHrTile = kRows * 64 * 2;  // 16 KB: 128 rows x 64 bf16, one 128-byte swizzle span
constexpr int kHrPoly = 0;               // of every 8 column pairs, exponentiated on the FMA pipe
constexpr uint32_t kHrColO = 128;        // within a query tile's 256 columns
constexpr uint32_t kHrColP = 192;

template <int NQ>
constexpr int hr_smem_bytes() {
  return 1024 + (NQ + kHrStages) * kHrTile + 512;
}

// Maximum of 64 values: 8 independent chains of three-input maxima, then a tree.
__device__ __forceinline__ float row_max64(const uint32_t (&s)[64]) {
  float mv[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mv[k] = __uint_as_float(s[k]);
#pragma unroll
  for (int k = 8; k < 56; k += 2)
    mv[(k >> 1) & 7] = max3(mv[(k >> 1) & 7], __uint_as_float(s[k]), __uint_as_float(s[k + 1]));
  mv[0] = max3(mv[0], mv[4], __uint_as_float(s[56]));
  mv[1] = max3(mv[1], mv[5], __uint_as_float(s[57]));
  mv[2] = max3(mv[2], mv[6], __uint_as_float(s[58]));
  mv[3] = max3(mv[3], mv[7], __uint_as_float(s[59]));
  mv[0] = max3(mv[0], __uint_as_float(s[60]), __uint_as_float(s[61]));
  mv[1] = max3(mv[1], __uint_as_float(s[62]), __uint_as_float(s[63]));
  return max3(mv[0], mv[1], fmaxf(mv[2], mv[3]));
}

// p_k = 2^(s_k c - m) for 64 scores, packed to bf16 pairs, POLY of every 8 column pairs on
// the FMA pipe; the fp32 sum goes to lsum.  Masked keys (-inf) give 0 on the special-function
// unit and 2^-125 on the polynomial.
template <int POLY>
__device__ __forceinline__ void exps64(const uint32_t (&s)[64], float c, float m, uint32_t (&pk)[32],
                                       float& lsum) {
  const float2 cc = make_float2(c, c), nm = make_float2(-m, -m);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1])), cc, nm);
    const float2 pe = (k & 7) < POLY ? exp2_poly2(x) : make_float2(ex2(x.x), ex2(x.y));
    acc[k & 3] = __fadd2_rn(acc[k & 3], pe);
    pk[k] = pack_bf16(pe.x, pe.y);
  }
  const float2 a = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  lsum = a.x + a.y;
}

template <int NQ>
__global__ void __launch_bounds__(kHrThreads, 1) patch_attn_hr_kernel(const __grid_constant__ AttnParams p) {
  constexpr int D = 64;
  constexpr int S = kHrStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + NQ * kHrTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + S * kHrTile);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + S;
  uint64_t* s_full = kv_empty + S;  // [t]
  uint64_t* s_free = s_full + 2;    // [t]: every softmax warp of the tile has S in registers
  uint64_t* p_full = s_free + 2;    // [t]
  uint64_t* pv_done = p_full + 2;   // [t]
  uint64_t* o_full = pv_done + 2;   // [t]
  uint64_t* mma_done = o_full + 2;  // [issuer]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ float xch_m[2][2][2][kRows];  // [tile parity][t][half][row]: half-tile maxima
  __shared__ float xch_l[2][2][kRows];     // [t][half][row]: row sums at the end
  __shared__ int s_last[4];  // [t]: this CTA merges query tile t; [2 + t]: the partials are ready

  PF_TRACE_CTA(1);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const CtaWork wk = cta_work(p);
  const int pair = wk.pair, part = wk.part, hd = wk.hd, b = wk.b;
  const int q0 = wk.grp * NQ * kRows;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int st = 0; st < S; ++st) {
      mbar_init(smem_u32(kv_full + st), 1);
      mbar_init(smem_u32(kv_empty + st), NQ);  // one commit per MMA issuer (one per query tile)
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(s_full + t), 1);
      mbar_init(smem_u32(s_free + t), 8);  // one arrival per softmax warp of the tile
      mbar_init(smem_u32(p_full + t), 8);
      mbar_init(smem_u32(pv_done + t), 1);
      mbar_init(smem_u32(o_full + t), 1);
      mbar_init(smem_u32(mma_done + t), 1);
    }
    *abort = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kHrWarpLoad && lane == 0) {
    prefetch_tmap(&p.tm_q);
    if (p.fresh_rows > 0) {
      prefetch_tmap(&p.tm_kf);
      prefetch_tmap(&p.tm_vf);
    }
    if (p.lo_len > 0) {
      prefetch_tmap(&p.tm_kl);
      prefetch_tmap(&p.tm_vl);
    }
    if (p.hi_len > 0) {
      prefetch_tmap(&p.tm_kb);
      prefetch_tmap(&p.tm_vb);
    }
    if (p.n_txt > 0) {
      prefetch_tmap(&p.tm_kt);
      prefetch_tmap(&p.tm_vt);
    }
  }
  if (warp == kHrWarpMma0) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  PF_TRACE_EV(0);
  // the next micro-step may start its CTAs (set-up, Q and fresh K/V loads) on SMs this grid
  // leaves idle; everything that touches memory this grid writes waits (grid_dep_wait)
  grid_dep_launch();

  Segments seg;
  seg.init(p);
  const int n_all = seg.total();
  // part r takes context tiles [ceil(r n / k), ceil((r + 1) n / k)): the first parts take the
  // extra tiles; the walk starts with the call's own tensors (fresh rows, text), which need
  // nothing from earlier micro-steps
  const int j0 = static_cast<int>((static_cast<long long>(part) * n_all + p.n_split - 1) / p.n_split);
  const int j1 = static_cast<int>((static_cast<long long>(part + 1) * n_all + p.n_split - 1) / p.n_split);
  const int n_tiles = j1 - j0;  // this CTA's context tiles: j0 .. j1-1

  if (warp >= 16) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kHrRegsOther));
    if (warp == kHrWarpLoad) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        const uint32_t qbar = smem_u32(q_full);
        mbar_arrive_expect_tx(qbar, NQ * kHrTile);
        for (int t = 0; t < NQ; ++t)
          tma_load_4d(smem_u32(sQ + t * kHrTile), &p.tm_q, 0, hd, q0 + t * kRows, b, qbar);
        int issued = 0;
        bool ok = true;
        bool dep_hi = false, dep_lo = false;
        for (int j = 0; j < n_tiles && ok; ++j) {
          int src, row0, nv;
          seg.tile(j0 + j, src, row0, nv);
          if ((src == 1 || src == 3) && !buffer_rows_ready(p, src, dep_hi, dep_lo, abort)) {
            ok = false;
            break;
          }
          for (int kv = 0; kv < 2; ++kv) {
            const int i = 2 * j + kv;
            const int st = i % S;
            if (!mbar_wait(smem_u32(kv_empty + st), ((i / S) & 1) ^ 1, abort, kWaitNs)) {
              ok = false;
              break;
            }
            const CUtensorMap* m = src == 0 ? (kv ? &p.tm_vf : &p.tm_kf)
                                   : src == 1 ? (kv ? &p.tm_vl : &p.tm_kl)
                                   : src == 3 ? (kv ? &p.tm_vb : &p.tm_kb)
                                              : (kv ? &p.tm_vt : &p.tm_kt);
            const uint32_t fb = smem_u32(kv_full + st);
            mbar_arrive_expect_tx(fb, kHrTile);
            tma_load_4d(smem_u32(sKV + st * kHrTile), m, 0, hd, row0, b, fb);
            issued = i + 1;
          }
        }
        if (!ok) raise_abort(abort, kWdLoad);
        // drain: every issued copy must land before the CTA exits
        mbar_wait(qbar, 0, nullptr, kWaitNs);
        for (int i = issued > S ? issued - S : 0; i < issued; ++i)
          mbar_wait(smem_u32(kv_full + (i % S)), (i / S) & 1, nullptr, kWaitNs);
        // this CTA has read all it reads of the buffer: count it for later calls' scatters
        count_reads_done(p);
      }
    } else if (warp == kHrWarpMma0 || (NQ == 2 && warp == kHrWarpMma1)) {
      // ------------------------------------------------------------ MMA issuer of query tile t
      if (lane == 0) {
        const int t = warp == kHrWarpMma0 ? 0 : 1;
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0);  // N = 128 keys, K-major K
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 64, 1);   // N = 64 columns, MN-major V
        const uint32_t q_lo = ((smem_u32(sQ) + t * kHrTile) >> 4) | desc_lbo_bits(16);
        const uint32_t k_lo = (smem_u32(sKV) >> 4) | desc_lbo_bits(16);
        const uint32_t v_lo = (smem_u32(sKV) >> 4) | desc_lbo_bits(kChunkBytes);
        const uint32_t tbase = tmem + t * 256;
        auto issue_qk = [=](int st) {
          const uint32_t b0 = k_lo + static_cast<uint32_t>((st * kHrTile) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tbase, smem_desc_lo(q_lo + 2 * kk), smem_desc_lo(b0 + 2 * kk), idesc_qk, kk > 0);
        };
        // O += [P_0 | P_1] V: 16 keys per MMA, P from TMEM
        auto issue_pv = [=](int st, bool acc) {
          const uint32_t v0 = v_lo + static_cast<uint32_t>((st * kHrTile) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tbase + kHrColO, tbase + kHrColP + kk * 8,
                   smem_desc_lo(v0 + static_cast<uint32_t>((kk * 2048) >> 4)), idesc_pv, acc || kk > 0);
        };

        bool ok = mbar_wait(smem_u32(q_full), 0, abort, kWaitNs);
        if (ok && n_tiles > 0) {
          ok = mbar_wait(smem_u32(kv_full + 0), 0, abort, kWaitNs);  // K(0): load 0, stage 0
          tc_fence_after();
          if (ok) {
            issue_qk(0);
            mma_commit(smem_u32(s_full + t));
            mma_commit(smem_u32(kv_empty + 0));
          }
        }
        for (int j = 0; j < n_tiles && ok; ++j) {
          if (j + 1 < n_tiles) {
            // QK(j+1) as soon as every softmax warp of the tile has S(j) in registers
            const int iK = 2 * (j + 1), sK = iK % S;
            if (!(ok = mbar_wait(smem_u32(kv_full + sK), (iK / S) & 1, abort, kWaitNs))) break;
            if (!(ok = mbar_wait(smem_u32(s_free + t), j & 1, abort, kWaitNs))) break;
            tc_fence_after();
            PF_TRACE_AT(4, 2 * t, j);
            issue_qk(sK);
            mma_commit(smem_u32(s_full + t));
            mma_commit(smem_u32(kv_empty + sK));
            PF_TRACE_AT(3, 2 * t, j);
          }
          const int iV = 2 * j + 1, sV = iV % S;
          if (!(ok = mbar_wait(smem_u32(kv_full + sV), (iV / S) & 1, abort, kWaitNs))) break;
          if (!(ok = mbar_wait(smem_u32(p_full + t), j & 1, abort, kWaitNs))) break;
          tc_fence_after();
          PF_TRACE_AT(2, 2 * t, j);
          issue_pv(sV, j > 0);
          mma_commit(smem_u32(pv_done + t));
          mma_commit(smem_u32(kv_empty + sV));
          if (j + 1 == n_tiles) mma_commit(smem_u32(o_full + t));
          PF_TRACE_AT(3, 2 * t + 1, j);
        }
        if (!ok) raise_abort(abort, kWdMma);
        // drain every MMA issued by this thread before TMEM is released
        mma_commit(smem_u32(mma_done + t));
        mbar_wait(smem_u32(mma_done + t), 0, nullptr, kWaitNs);
      }
    } else if (warp == kHrWarpScatter) {
      // ------------------------------------------------------------ buffer scatter
      scatter_share<D>(p, lane);
    }
  } else if (warp < 8 * NQ) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHrRegsSoftmax));
    // ------------------------------------------------------------ softmax of one half + epilogue
    const int t = warp >> 3;
    const int hh = (warp >> 2) & 1;
    const int wq = warp & 3;
    const int pair_bar = 1 + 4 * t + wq;  // the two warps (halves) of this row quarter
    const int rloc = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 256 + hh * 64;
    const uint32_t tO = tmem + lane_off + t * 256 + kHrColO + hh * 32;  // this half's 32 O columns
    const uint32_t tP = tmem + lane_off + t * 256 + kHrColP + hh * 32;
    const float c = p.scale_log2;
    float m = -INFINITY;  // the row's reference maximum, in log2 units (same in both halves)
    float l = 0.f;        // this half's part of the row sum
    bool ok = true;
    // local indices of this CTA's ragged context tiles and the valid keys of this half there
    int rag_j[4], rag_nv[4];
    {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        int end, len;
        seg.bounds(k, end, len);
        const int e = end - 1;
        const int nv = len % kRows;
        rag_nv[k] = min(max(nv - 64 * hh, 0), 64);
        rag_j[k] = (nv != 0 && e >= j0 && e < j1) ? e - j0 : -1;
      }
    }
    bool s_ready = false;  // S(j) was seen complete at the end of tile j-1
    for (int j = 0; j < n_tiles; ++j) {
      if (!s_ready) ok = ok && mbar_wait(smem_u32(s_full + t), j & 1, abort, kWaitNs);
      tc_fence_after();
      if (wq == 0 && lane == 0) PF_TRACE_AT(0, 2 * t + hh, j);
      if (j == 0) PF_TRACE_EV(1);
      uint32_t s[64];
      tmem_ld32(tS + 0, s);
      tmem_ld32(tS + 32, s + 32);
      tmem_wait_ld();
      reg_fence<64>(s);
      if (wq == 0 && lane == 0) PF_TRACE_AT(5, 2 * t + hh, j);
      // S is in registers: hand its columns back so QK(j+1) can start
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(s_free + t));
      if (wq == 0 && lane == 0) PF_TRACE_AT(10, 2 * t + hh, j);
      int nv = 64;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (j == rag_j[k]) nv = rag_nv[k];
      if (nv < 64) {
#pragma unroll
        for (int k = 0; k < 64; ++k)
          if (k >= nv) s[k] = __float_as_uint(-INFINITY);
      }
      if (wq == 0 && lane == 0) PF_TRACE_AT(11, 2 * t + hh, j);
      const float mx_half = row_max64(s);
      if (wq == 0 && lane == 0) PF_TRACE_AT(12, 2 * t + hh, j);
      // the row maximum over both halves: exchange, behind a barrier that also makes the two
      // warps agree on going on (a warp whose wait failed must not leave its partner waiting)
      xch_m[j & 1][t][hh][rloc] = mx_half;
      if (wq == 0 && lane == 0) PF_TRACE_AT(8, 2 * t + hh, j);
      ok = named_bar_and(pair_bar, 64, ok);
      if (!ok) break;
      const float mxs = fmaxf(xch_m[j & 1][t][0][rloc], xch_m[j & 1][t][1][rloc]) * c;
      if (wq == 0 && lane == 0) PF_TRACE_AT(6, 2 * t + hh, j);
      const bool grow = mxs > m + 8.f;  // the same decision in both halves
      // warp-collective TMEM accesses: the whole warp rescales when any of its rows grew
      // (alpha is exactly 1 for the others)
      const bool any_grow = __any_sync(0xffffffffu, grow);
      float alpha = 1.f;
      if (any_grow) {
        alpha = grow ? ex2(m - mxs) : 1.f;
        l *= alpha;
        m = grow ? mxs : m;
      }
      // P(j) may overwrite P(j-1) once PV(j-1) has read it: S(j+1) complete implies it (QK(j+1)
      // was issued after PV(j-1)); the last tile waits for PV(j-1) itself.  Probed half way
      // through the exponentials so the wait is usually over.
      const bool has_next = j + 1 < n_tiles;
      const uint32_t gate = has_next ? smem_u32(s_full + t) : smem_u32(pv_done + t);
      const uint32_t gate_par = has_next ? static_cast<uint32_t>((j + 1) & 1)
                                         : static_cast<uint32_t>((j - 1) & 1);
      bool gate_ok = !has_next && j == 0;  // a single tile: nothing to wait for
      uint32_t pk[32];
      {
        const float2 cc = make_float2(c, c), nm = make_float2(-m, -m);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1])), cc, nm);
          const float2 pe = (k & 7) < kHrPoly ? exp2_poly2(x) : make_float2(ex2(x.x), ex2(x.y));
          acc[k & 3] = __fadd2_rn(acc[k & 3], pe);
          pk[k] = pack_bf16(pe.x, pe.y);
          if (k == 15 && !gate_ok) gate_ok = mbar_test_wait_all(gate, gate_par);
        }
        const float2 a = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
        l += a.x + a.y;
      }
      if (wq == 0 && lane == 0) PF_TRACE_AT(7, 2 * t + hh, j);
      if (!gate_ok) {
        // on failure go on (the abort flag is up): the partner learns of it at the next
        // exchange, and both leave the loop together
        if (!mbar_wait(gate, gate_par, abort, kWaitNs)) ok = false;
        ok = __all_sync(0xffffffffu, ok);
      }
      tc_fence_after();
      if (wq == 0 && lane == 0) PF_TRACE_AT(9, 2 * t + hh, j);
      s_ready = has_next;
      if (any_grow && j > 0) {
        // this half rescales its 32 of the row's 64 O columns (PV(j-1) is complete)
#pragma unroll
        for (int c0 = 0; c0 < 32; c0 += 16) {
          uint32_t o[16];
          tmem_ld16(tO + c0, o);
          tmem_wait_ld();
          reg_fence<16>(o);
#pragma unroll
          for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st16(tO + c0, o);
        }
      }
      tmem_st32(tP, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(p_full + t));
      if (wq == 0 && lane == 0) PF_TRACE_AT(1, 2 * t + hh, j);
    }
    if (!ok && lane == 0) raise_abort(abort, kWdSoftmax);
    {
      bool ok_o = ok && mbar_wait(smem_u32(o_full + t), 0, abort, kWaitNs);
      PF_TRACE_EV(2);
      ok_o = __all_sync(0xffffffffu, ok_o);
      // both halves of the query tile take the same branch (the epilogue has barriers)
      ok_o = named_bar_and(9 + t, 2 * kRows, ok_o);
      if (!ok_o) {
        if (ok && lane == 0) raise_abort(abort, kWdEpilogue);
      } else {
        tc_fence_after();
        grid_dep_wait();  // the output and the workspace may be in use by the previous grid
        const int row = q0 + t * kRows + rloc;
        const bool in_range = row < p.q_rows;
        xch_l[t][hh][rloc] = l;
        named_bar_sync(9 + t, 2 * kRows);
        const float lrow = xch_l[t][0][rloc] + xch_l[t][1][rloc];
        float o[32];
#pragma unroll
        for (int c0 = 0; c0 < 32; c0 += 16) {
          uint32_t a0[16];
          tmem_ld16(tO + c0, a0);
          tmem_wait_ld();
          reg_fence<16>(a0);
#pragma unroll
          for (int k = 0; k < 16; ++k) o[c0 + k] = __uint_as_float(a0[k]);
        }
        // this thread's 32 output columns: 32 hh .. 32 hh + 31
        uint16_t* dst = p.o + ((static_cast<size_t>(b) * p.q_rows + row) * p.heads + hd) * D + 32 * hh;
        if (p.n_split == 1) {
          const float inv = 1.f / lrow;
          if (in_range) {
#pragma unroll
            for (int k = 0; k < 32; k += 8) {
              uint4 w;
              w.x = pack_bf16(o[k + 0] * inv, o[k + 1] * inv);
              w.y = pack_bf16(o[k + 2] * inv, o[k + 3] * inv);
              w.z = pack_bf16(o[k + 4] * inv, o[k + 5] * inv);
              w.w = pack_bf16(o[k + 6] * inv, o[k + 7] * inv);
              *reinterpret_cast<uint4*>(dst + k) = w;
            }
          }
        } else {
          // the last part to finish its loop merges (an arrival counter tells, before anything
          // is stored); the others store their partial and count it written
          const size_t slot_elems = static_cast<size_t>(D + 2) * kRows;
          float* slot0 = p.ws_part + (static_cast<size_t>(pair) * 2 + t) * p.n_split * slot_elems;
          unsigned* cnt = p.ws_cnt + (static_cast<size_t>(pair) * 2 + t) * 2;  // arrived, written
          if (hh == 0 && rloc == 0) s_last[t] = atomicAdd(cnt, 1u) == static_cast<unsigned>(p.n_split - 1);
          named_bar_sync(9 + t, 2 * kRows);
          // every part stores its partial (O row: this thread's 32 of the 64 columns; m, l),
          // column-major -- the merger too, so that the merge reads all parts in part order
          // whichever part merges
          float* mine = slot0 + static_cast<size_t>(part) * slot_elems;
#pragma unroll
          for (int k = 0; k < 32; ++k) mine[(32 * hh + k) * kRows + rloc] = o[k];
          if (hh == 0) {
            mine[D * kRows + rloc] = m;
            mine[(D + 1) * kRows + rloc] = lrow;
          }
          if (!s_last[t]) {
            __threadfence();
            named_bar_sync(9 + t, 2 * kRows);
            PF_TRACE_EV(3);
            if (hh == 0 && rloc == 0) atomicAdd(cnt + 1, 1u);
          } else {
            // the merger: wait (bounded) for the other parts' partials -- they have all arrived,
            // so they are running and wait for nothing -- then reset the counters for the next
            // launch; its own partial is visible to its threads after the barrier
            if (hh == 0 && rloc == 0) {
              const bool ready = wait_count_geq(cnt + 1, static_cast<unsigned>(p.n_split - 1), abort, kWaitNs);
              if (ready) {
                cnt[0] = 0u;
                cnt[1] = 0u;
              } else {
                raise_abort(abort, kWdEpilogue);
              }
              s_last[2 + t] = ready;
            }
            named_bar_sync(9 + t, 2 * kRows);
            PF_TRACE_EV(4);
            if (s_last[2 + t]) {
              // this thread's 32 columns of its row
              float mref, inv;
              merge_stats(slot0 + rloc, slot_elems, D, p.n_split, mref, inv);
              merge_columns<32, 8>(slot0 + rloc, slot_elems, D, p.n_split, 32 * hh, mref, inv, dst, in_range);
              PF_TRACE_EV(5);
              if (p.discard) {
                // every thread of the tile has read all parts' slots: drop them from L2
                named_bar_sync(9 + t, 2 * kRows);
                discard_partials<D>(slot0, p.n_split, hh * kRows + rloc, 2 * kRows);
              }
            }
          }
        }
      }
    }
  } else {
    // softmax warps of a second query tile when the CTA has one: idle
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kHrRegsOther));
  }

  tc_fence_before();
  __syncthreads();
  PF_TRACE_CTA(2);
  if (warp == kHrWarpMma0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Launch an attention kernel with programmatic stream serialization: when the previous
// work on the stream is another attention launch, this grid's CTAs may start while that one
// finishes (it signals with grid_dep_launch); the kernel waits (grid_dep_wait) before it
// reads the K/V buffer or writes the buffer, the output or the workspace.  After any other
// kind of work the launch simply waits for it, as an ordinary launch does.
cudaError_t launch_overlapped(void (*kernel)(AttnParams), const AttnParams& p, int threads, int smem,
                              cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.n_pairs) * static_cast<unsigned>(p.n_split));
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

template <int NQ>
cudaError_t hr_configure_once(int dev) {
  static std::mutex mu;
  static uint64_t done = 0;  // bit per device ordinal
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const uint64_t bit = 1ull << dev;
  std::lock_guard<std::mutex> lock(mu);
  if (done & bit) return cudaSuccess;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, patch_attn_hr_kernel<NQ>);
  if (e != cudaSuccess) return e;
  if (128 * static_cast<long>(kHrRegsOther) + 512 * static_cast<long>(kHrRegsSoftmax) >
      static_cast<long>(kHrThreads) * fa.numRegs)
    return cudaErrorNotSupported;  // the split would wait forever in setmaxnreg.inc
  e = cudaFuncSetAttribute(patch_attn_hr_kernel<NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           hr_smem_bytes<NQ>());
  if (e != cudaSuccess) return e;
  done |= bit;
  return cudaSuccess;
}

template <int NQ>
cudaError_t launch_hr(const AttnParams& p, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = hr_configure_once<NQ>(dev);
  if (e != cudaSuccess) return e;
  return launch_overlapped(patch_attn_hr_kernel<NQ>, p, kHrThreads, hr_smem_bytes<NQ>(), stream);
}

// Epilogue of a softmax thread that owns a whole query row: O (TMEM columns from tO) over l
// to the bf16 output when the call has no key-range split.  Otherwise the last part of the
// query tile to finish its loop (an arrival counter tells, before anything is stored) merges:
// every other part stores its unnormalised row with m and l in its workspace slot and counts
// it written; the merger waits (bounded) for those counts -- the parts it waits for have all
// arrived, so they are running and wait for nothing -- and combines them with its own part,
// which it never stores.  Called by all 128 threads of the query tile's warpgroup (named
// barrier 1 + t).
template <int D>
__device__ __forceinline__ void full_row_epilogue(const AttnParams& p, uint32_t tO, float m, float l,
                                                  int pair, int part, int t, int q0, int hd, int b,
                                                  int wq, int lane, int* s_last, volatile int* abort) {
  constexpr int kMmaN = Dims<D>::kMmaN;
  const int rloc = wq * 32 + lane;
  const int row = q0 + t * kRows + rloc;
  uint16_t* dst = p.o + ((static_cast<size_t>(b) * p.q_rows + row) * p.heads + hd) * D;
  const bool in_range = row < p.q_rows;
  if (p.n_split == 1) {
    const float inv = 1.f / l;
#pragma unroll
    for (int c0 = 0; c0 < kMmaN; c0 += 16) {
      uint32_t o[16];
      tmem_ld16(tO + c0, o);
      tmem_wait_ld();
      reg_fence<16>(o);
      store_row16<D>(dst, c0, o, inv, in_range);
    }
    return;
  }
  const size_t slot_elems = static_cast<size_t>(D + 2) * kRows;
  float* slot0 = p.ws_part + (static_cast<size_t>(pair) * 2 + t) * p.n_split * slot_elems;
  unsigned* cnt = p.ws_cnt + (static_cast<size_t>(pair) * 2 + t) * 2;  // arrived, written
  if (rloc == 0) s_last[t] = atomicAdd(cnt, 1u) == static_cast<unsigned>(p.n_split - 1);
  named_bar_sync(1 + t, kRows);
  // every part stores its partial, O row (d columns), m, l, column-major -- the merger too,
  // so that the merge reads all parts in part order whichever part merges
  float* mine = slot0 + static_cast<size_t>(part) * slot_elems;
#pragma unroll
  for (int c0 = 0; c0 < kMmaN; c0 += 16) {
    uint32_t o[16];
    tmem_ld16(tO + c0, o);
    tmem_wait_ld();
    reg_fence<16>(o);
#pragma unroll
    for (int k = 0; k < 16; ++k)
      if (c0 + k < D) mine[(c0 + k) * kRows + rloc] = __uint_as_float(o[k]);
  }
  mine[D * kRows + rloc] = m;
  mine[(D + 1) * kRows + rloc] = l;
  if (!s_last[t]) {
    __threadfence();
    named_bar_sync(1 + t, kRows);
    if (rloc == 0) atomicAdd(cnt + 1, 1u);
    return;
  }
  // the merger: wait until the other parts' partials are written, then reset the counters
  // for the next launch (every other part has counted both by then); its own partial is
  // visible to its threads after the barrier
  if (rloc == 0) {
    const bool ready = wait_count_geq(cnt + 1, static_cast<unsigned>(p.n_split - 1), abort, kWaitNs);
    if (ready) {
      cnt[0] = 0u;
      cnt[1] = 0u;
    } else {
      raise_abort(abort, kWdEpilogue);
    }
    s_last[2 + t] = ready;
  }
  named_bar_sync(1 + t, kRows);
  if (!s_last[2 + t]) return;
  float mref, inv;
  merge_stats(slot0 + rloc, slot_elems, D, p.n_split, mref, inv);
  merge_columns<D>(slot0 + rloc, slot_elems, D, p.n_split, 0, mref, inv, dst, in_range);
  if (p.discard) {
    // every thread of the tile has read all parts' slots: drop them from L2
    named_bar_sync(1 + t, kRows);
    discard_partials<D>(slot0, p.n_split, rloc, kRows);
  }
}

// ------------------------------------------------------------------ head_dim 72/128: split key tiles
//
// With one thread per query row and P written over S, the next key tile's QK cannot start
// before PV has read P, and PV cannot start before the softmax has written P: per query
// tile the softmax, the PV and the next QK run one after another.  This kernel splits every
// 128-key tile into two 64-key halves, each with its own S columns and its own P over them.
// The softmax thread still owns a whole row and keeps one reference maximum m, one row sum l
// and one O accumulator; it exponentiates half 0 of tile j, hands P_0 to the MMA issuer,
// then exponentiates half 1 while the tensor core runs PV_0(j) and QK_0(j+1).  By the time
// the thread comes back to half 0 of tile j+1, its scores are usually ready.
//
// TMEM, per query tile t: S_0 | S_1 (64 fp32 columns each) at 128 t, O (head_dim padded to
// 16 columns) at 256 + 128 t.  An O rescale (the row maximum grew by more than 2^8) must not
// overlap a PV still accumulating into O: S_h(j) complete implies PV_h(j-1) complete (same
// issuing thread, issued before QK_h(j)), and the rescale also waits for the other half's
// latest PV through its own barrier.
//
// Warps: 0-7 softmax (warp w: query tile w / 4, TMEM lane quarter w % 4), 8 TMEM allocation
// + MMA issuer of query tile 0, 9 TMA producer, 10 scatter, 11 MMA issuer of query tile 1.
template <int D, int NQ>
__global__ void __launch_bounds__(kThreads, 1) patch_attn_sn_kernel(const __grid_constant__ AttnParams p) {
  using Dm = Dims<D>;
  constexpr int S = Dm::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + NQ * Dm::kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + S * Dm::kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + S;
  uint64_t* s_full = kv_empty + S;   // [2 t + h]
  uint64_t* p_full = s_full + 4;     // [2 t + h]
  uint64_t* pv_done = p_full + 4;    // [2 t + h]
  uint64_t* o_full = pv_done + 4;    // [t]
  uint64_t* mma_done = o_full + 2;   // [issuer]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ int s_last[4];  // [t]: this CTA merges query tile t; [2 + t]: the partials are ready

  PF_TRACE_CTA(1);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const CtaWork wk = cta_work(p);
  const int pair = wk.pair, part = wk.part, hd = wk.hd, b = wk.b;
  const int q0 = wk.grp * NQ * kRows;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int st = 0; st < S; ++st) {
      mbar_init(smem_u32(kv_full + st), 1);
      mbar_init(smem_u32(kv_empty + st), NQ);  // one commit per MMA issuer (one per query tile)
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(smem_u32(s_full + i), 1);
      mbar_init(smem_u32(p_full + i), 4);  // one arrival per softmax warp
      mbar_init(smem_u32(pv_done + i), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(o_full + t), 1);
      mbar_init(smem_u32(mma_done + t), 1);
    }
    *abort = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kWarpLoad && lane == 0) {
    prefetch_tmap(&p.tm_q);
    if (p.fresh_rows > 0) {
      prefetch_tmap(&p.tm_kf);
      prefetch_tmap(&p.tm_vf);
    }
    if (p.lo_len > 0) {
      prefetch_tmap(&p.tm_kl);
      prefetch_tmap(&p.tm_vl);
    }
    if (p.hi_len > 0) {
      prefetch_tmap(&p.tm_kb);
      prefetch_tmap(&p.tm_vb);
    }
    if (p.n_txt > 0) {
      prefetch_tmap(&p.tm_kt);
      prefetch_tmap(&p.tm_vt);
    }
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  PF_TRACE_EV(0);
  // the next micro-step may start its CTAs (set-up, Q and fresh K/V loads) on SMs this grid
  // leaves idle; everything that touches memory this grid writes waits (grid_dep_wait)
  grid_dep_launch();

  Segments seg;
  seg.init(p);
  const int n_all = seg.total();
  // part r takes context tiles [ceil(r n / k), ceil((r + 1) n / k)): the first parts take the
  // extra tiles; the walk starts with the call's own tensors (fresh rows, text), which need
  // nothing from earlier micro-steps
  const int j0 = static_cast<int>((static_cast<long long>(part) * n_all + p.n_split - 1) / p.n_split);
  const int j1 = static_cast<int>((static_cast<long long>(part + 1) * n_all + p.n_split - 1) / p.n_split);
  const int n_tiles = j1 - j0;  // this CTA's context tiles: j0 .. j1-1

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
    if (warp == kWarpLoad) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        const uint32_t qbar = smem_u32(q_full);
        mbar_arrive_expect_tx(qbar, NQ * Dm::kTileBytes);
        for (int t = 0; t < NQ; ++t)
          for (int c = 0; c < Dm::kChunks; ++c)
            tma_load_4d(smem_u32(sQ + t * Dm::kTileBytes + c * kChunkBytes), &p.tm_q, c * 64, hd,
                        q0 + t * kRows, b, qbar);
        int issued = 0;
        bool ok = true;
        bool dep_hi = false, dep_lo = false;
        for (int j = 0; j < n_tiles && ok; ++j) {
          int src, row0, nv;
          seg.tile(j0 + j, src, row0, nv);
          if ((src == 1 || src == 3) && !buffer_rows_ready(p, src, dep_hi, dep_lo, abort)) {
            ok = false;
            break;
          }
          for (int kv = 0; kv < 2; ++kv) {
            const int i = 2 * j + kv;
            const int st = i % S;
            if (!mbar_wait(smem_u32(kv_empty + st), ((i / S) & 1) ^ 1, abort, kWaitNs)) {
              ok = false;
              break;
            }
            const CUtensorMap* m = src == 0 ? (kv ? &p.tm_vf : &p.tm_kf)
                                   : src == 1 ? (kv ? &p.tm_vl : &p.tm_kl)
                                   : src == 3 ? (kv ? &p.tm_vb : &p.tm_kb)
                                              : (kv ? &p.tm_vt : &p.tm_kt);
            const uint32_t fb = smem_u32(kv_full + st);
            mbar_arrive_expect_tx(fb, Dm::kTileBytes);
            for (int c = 0; c < Dm::kChunks; ++c)
              tma_load_4d(smem_u32(sKV + st * Dm::kTileBytes + c * kChunkBytes), m, c * 64, hd, row0,
                          b, fb);
            issued = i + 1;
          }
        }
        if (!ok) raise_abort(abort, kWdLoad);
        // drain: every issued copy must land before the CTA exits
        mbar_wait(qbar, 0, nullptr, kWaitNs);
        for (int i = issued > S ? issued - S : 0; i < issued; ++i)
          mbar_wait(smem_u32(kv_full + (i % S)), (i / S) & 1, nullptr, kWaitNs);
        // this CTA has read all it reads of the buffer: count it for later calls' scatters
        count_reads_done(p);
      }
    } else if (warp == kWarpMma || (NQ == 2 && warp == kWarpMma2)) {
      // ------------------------------------------------------------ MMA issuer of query tile t
      if (lane == 0) {
        const int t = warp == kWarpMma ? 0 : 1;
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 64, 0);         // N = 64 keys
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, Dm::kMmaN, 1);  // N = head_dim (padded)
        const uint32_t q_lo = ((smem_u32(sQ) + t * Dm::kTileBytes) >> 4) | desc_lbo_bits(16);
        const uint32_t k_lo = (smem_u32(sKV) >> 4) | desc_lbo_bits(16);
        const uint32_t v_lo = (smem_u32(sKV) >> 4) | desc_lbo_bits(kChunkBytes);
        // S_h = Q_t K[64 h .. 64 h + 63]^T: the half's key rows start 64 * 128 bytes into each
        // 64-column chunk of the K tile
        auto issue_qk = [=](int h, int st) {
          const uint32_t b0 = k_lo + static_cast<uint32_t>((st * Dm::kTileBytes + h * 8192) >> 4);
          const uint32_t d = tmem + t * 128 + h * 64;
#pragma unroll
          for (int kk = 0; kk < Dm::kMmaN / 16; ++kk) {
            const uint32_t off = static_cast<uint32_t>(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
            mma_ss(d, smem_desc_lo(q_lo + off), smem_desc_lo(b0 + off), idesc_qk, kk > 0);
          }
        };
        // O += P_h V[64 h .. 64 h + 63]: P_h from TMEM (over S_h), 16 keys per MMA
        auto issue_pv = [=](int h, int st, bool acc) {
          const uint32_t v0 = v_lo + static_cast<uint32_t>((st * Dm::kTileBytes + h * 8192) >> 4);
          const uint32_t d = tmem + kColO + t * 128;
          const uint32_t a = tmem + t * 128 + h * 64;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(d, a + kk * 8, smem_desc_lo(v0 + static_cast<uint32_t>((kk * 2048) >> 4)), idesc_pv,
                   acc || kk > 0);
        };

        bool ok = mbar_wait(smem_u32(q_full), 0, abort, kWaitNs);
        if (ok && n_tiles > 0) {
          ok = mbar_wait(smem_u32(kv_full + 0), 0, abort, kWaitNs);  // K(0): load 0, stage 0
          tc_fence_after();
          if (ok) {
            issue_qk(0, 0);
            mma_commit(smem_u32(s_full + 2 * t));
            issue_qk(1, 0);
            mma_commit(smem_u32(s_full + 2 * t + 1));
            mma_commit(smem_u32(kv_empty + 0));
          }
        }
        for (int j = 0; j < n_tiles && ok; ++j) {
          const int iV = 2 * j + 1, sV = iV % S;
          if (!(ok = mbar_wait(smem_u32(kv_full + sV), (iV / S) & 1, abort, kWaitNs))) break;
          const bool has_next = j + 1 < n_tiles;
          const int iK = 2 * (j + 1), sK = iK % S;
          if (has_next && !(ok = mbar_wait(smem_u32(kv_full + sK), (iK / S) & 1, abort, kWaitNs))) break;
          PF_TRACE_AT(4, 2 * t, j);
          for (int h = 0; h < 2; ++h) {
            if (!(ok = mbar_wait(smem_u32(p_full + 2 * t + h), j & 1, abort, kWaitNs))) break;
            tc_fence_after();
            PF_TRACE_AT(2, 2 * t + h, j);
            issue_pv(h, sV, j > 0 || h > 0);
            mma_commit(smem_u32(pv_done + 2 * t + h));
            if (has_next) {
              issue_qk(h, sK);
              mma_commit(smem_u32(s_full + 2 * t + h));
            }
            PF_TRACE_AT(3, 2 * t + h, j);
          }
          if (!ok) break;
          if (!has_next) mma_commit(smem_u32(o_full + t));
          mma_commit(smem_u32(kv_empty + sV));
          if (has_next) mma_commit(smem_u32(kv_empty + sK));
        }
        if (!ok) raise_abort(abort, kWdMma);
        // drain every MMA issued by this thread before TMEM is released
        mma_commit(smem_u32(mma_done + t));
        mbar_wait(smem_u32(mma_done + t), 0, nullptr, kWaitNs);
      }
    } else if (warp == kWarpScatter) {
      // ------------------------------------------------------------ buffer scatter
      scatter_share<D>(p, lane);
    }
  } else if (warp < 4 * NQ) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ------------------------------------------------------------ softmax + epilogue
    const int t = warp >> 2;
    const int wq = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + kColO + t * 128;
    const float c = p.scale_log2;
    float m = -INFINITY;  // reference row maximum, in log2 units
    float l = 0.f;
    bool ok = true;
    // local indices of this CTA's ragged context tiles and their valid rows
    int rag_j[4], rag_nv[4];
    {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        int end, len;
        seg.bounds(k, end, len);
        const int e = end - 1;
        rag_nv[k] = len % kRows;
        rag_j[k] = (rag_nv[k] != 0 && e >= j0 && e < j1) ? e - j0 : -1;
      }
    }
    for (int j = 0; j < n_tiles && ok; ++j) {
      int nv = kRows;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (j == rag_j[k]) nv = rag_nv[k];
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        ok = mbar_wait(smem_u32(s_full + 2 * t + h), j & 1, abort, kWaitNs);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        if (wq == 0 && lane == 0) PF_TRACE_AT(0, 2 * t + h, j);
        if (j == 0 && h == 0) PF_TRACE_EV(1);
        uint32_t s[64];
        tmem_ld32(tS + h * 64, s);
        tmem_ld32(tS + h * 64 + 32, s + 32);
        tmem_wait_ld();
        reg_fence<64>(s);
        const int nvh = min(max(nv - 64 * h, 0), 64);
        if (nvh < 64) {
#pragma unroll
          for (int k = 0; k < 64; ++k)
            if (k >= nvh) s[k] = __float_as_uint(-INFINITY);
        }
        uint32_t pk[32];
        float lsum;
        {
          const float mxs = row_max64(s) * c;
          const bool grow = mxs > m + 8.f;
          // warp-collective TMEM accesses: the whole warp rescales when any of its rows grew
          // (alpha is exactly 1 for the others)
          const bool any_grow = __any_sync(0xffffffffu, grow);
          const float alpha = grow ? ex2(m - mxs) : 1.f;
          if (any_grow && (j > 0 || h > 0)) {
            // O holds earlier PVs: PV_h(j-1) is complete (S_h(j) is); wait for the other
            // half's latest one, PV_1(j-1) before half 0, PV_0(j) before half 1
            const uint32_t par = h == 0 ? static_cast<uint32_t>((j - 1) & 1) : static_cast<uint32_t>(j & 1);
            ok = mbar_wait(smem_u32(pv_done + 2 * t + (h ^ 1)), par, abort, kWaitNs);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < Dm::kMmaN; c0 += 16) {
              uint32_t o[16];
              tmem_ld16(tO + c0, o);
              tmem_wait_ld();
              reg_fence<16>(o);
#pragma unroll
              for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st16(tO + c0, o);
            }
          }
          l *= alpha;
          m = grow ? mxs : m;
          exps64<kPolyPairs<D>>(s, c, m, pk, lsum);
        }
        l += lsum;
        if (wq == 0 && lane == 0) PF_TRACE_AT(7, 2 * t + h, j);
        tmem_st32(tS + h * 64, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(p_full + 2 * t + h));
        if (wq == 0 && lane == 0) PF_TRACE_AT(1, 2 * t + h, j);
      }
    }
    if (!ok && lane == 0) raise_abort(abort, kWdSoftmax);
    {
      bool ok_o = ok && mbar_wait(smem_u32(o_full + t), 0, abort, kWaitNs);
      PF_TRACE_EV(2);
      ok_o = __all_sync(0xffffffffu, ok_o);
      // the whole warpgroup takes the same branch (the merge path has barriers)
      ok_o = named_bar_and(1 + t, kRows, ok_o);
      if (!ok_o) {
        if (ok && lane == 0) raise_abort(abort, kWdEpilogue);
      } else {
        tc_fence_after();
        grid_dep_wait();  // the output and the workspace may be in use by the previous grid
        full_row_epilogue<D>(p, tO, m, l, pair, part, t, q0, hd, b, wq, lane, s_last, abort);
      }
    }
  } else {
    // second softmax warpgroup when the CTA has a single query tile: idle
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
  }

  tc_fence_before();
  __syncthreads();
  PF_TRACE_CTA(2);
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int NQ>
cudaError_t sn_configure_once(int dev) {
  static std::mutex mu;
  static uint64_t done = 0;  // bit per device ordinal
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const uint64_t bit = 1ull << dev;
  std::lock_guard<std::mutex> lock(mu);
  if (done & bit) return cudaSuccess;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, patch_attn_sn_kernel<D, NQ>);
  if (e != cudaSuccess) return e;
  if (128 * static_cast<long>(kRegsOther) + 256 * static_cast<long>(kRegsSoftmax) >
      static_cast<long>(kThreads) * fa.numRegs)
    return cudaErrorNotSupported;  // the split would wait forever in setmaxnreg.inc
  e = cudaFuncSetAttribute(patch_attn_sn_kernel<D, NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_bytes<D, NQ>());
  if (e != cudaSuccess) return e;
  done |= bit;
  return cudaSuccess;
}

template <int D, int NQ>
cudaError_t launch_sn(const AttnParams& p, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = sn_configure_once<D, NQ>(dev);
  if (e != cudaSuccess) return e;
  return launch_overlapped(patch_attn_sn_kernel<D, NQ>, p, kThreads, smem_bytes<D, NQ>(), stream);
}

__global__ void zero_u32_kernel(unsigned* p, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    p[i] = 0u;
}

}  // namespace

int attn_tiles_per_cta(int plen) { return plen > kRows ? 2 : 1; }

int attn_context_tiles(int fresh_rows, int lo_len, int hi_len, int n_txt) {
  auto tiles = [](long long n) { return static_cast<int>((n + kRows - 1) / kRows); };
  return tiles(fresh_rows) + tiles(lo_len) + tiles(hi_len) + tiles(n_txt);
}

int attn_choose_split(int n_pairs, int n_tiles, int n_sms, int max_split) {
  // Cost model in units of context tiles.  Launches overlap on the GPU (the per-layer ordering
  // counters let a launch start while earlier ones finish), so a call costs the larger of its
  // share of SM time, n_pairs (n_tiles + k c) / n_sms, and half the length of one CTA,
  // (ceil(n_tiles / k) + c) / 2: a launch is issued only once every CTA of the previous one
  // has started, so short launches of few CTAs leave SMs idle between them (measured: a
  // PixArt-size call of 32 CTAs runs 8-12% slower unsplit than split in two, with either
  // buffer layout).  c is the fixed cost of a CTA (launch, TMEM allocation, Q load, pipeline
  // fill, merge).  Of the splits within 5% of the cheapest the smallest is taken: fewer
  // partials to store and merge.
  constexpr double kOverheadTiles = 6.0;
  const int kmax = max_split < kMaxSplit ? max_split : kMaxSplit;
  double cost[kMaxSplit + 1];
  double best = -1.0;
  int kn = 0;
  for (int k = 1; k <= kmax && k <= n_tiles; ++k) {
    const double sm_time = static_cast<double>(n_pairs) * (n_tiles + k * kOverheadTiles) / n_sms;
    const double cta = 0.5 * ((n_tiles + k - 1) / k + kOverheadTiles);
    cost[k] = sm_time > cta ? sm_time : cta;
    if (best < 0.0 || cost[k] < best) best = cost[k];
    kn = k;
  }
  for (int k = 1; k <= kn; ++k)
    if (cost[k] <= 1.05 * best) return k;
  return 1;
}

size_t attn_workspace_bytes(int n_pairs, int head_dim, int n_split) {
  if (n_split <= 1) return 0;
  const size_t part_bytes = static_cast<size_t>(n_pairs) * 2 * n_split * (head_dim + 2) * kRows * 4;
  const size_t cnt_bytes = static_cast<size_t>(n_pairs) * 2 * 2 * 4;
  return ((part_bytes + 255) / 256) * 256 + cnt_bytes;
}

cudaError_t launch_zero_u32(unsigned* p, size_t n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  size_t blocks = (n + 255) / 256;
  if (blocks > 1024) blocks = 1024;
  zero_u32_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p, n);
  return cudaGetLastError();
}

cudaError_t launch_patch_attn(const AttnParams& p, cudaStream_t stream) {
  const bool two = p.q_rows > kRows;
  switch (p.head_dim) {
    case 64: return two ? launch_hr<2>(p, stream) : launch_hr<1>(p, stream);
    case 72: return two ? launch_sn<72, 2>(p, stream) : launch_sn<72, 1>(p, stream);
    case 128: return two ? launch_sn<128, 2>(p, stream) : launch_sn<128, 1>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

#ifdef PF_TRACE
extern "C" int pf_trace_read(unsigned long long* dst, size_t n) {
  if (n > sizeof(g_trace) / sizeof(g_trace[0])) n = sizeof(g_trace) / sizeof(g_trace[0]);
  return static_cast<int>(cudaMemcpyFromSymbol(dst, g_trace, n * sizeof(unsigned long long)));
}
extern "C" int pf_trace_cta_read(unsigned long long* dst, size_t n) {
  if (n > sizeof(g_cta) / sizeof(g_cta[0])) n = sizeof(g_cta) / sizeof(g_cta[0]);
  return static_cast<int>(cudaMemcpyFromSymbol(dst, g_cta, n * sizeof(unsigned long long)));
}
extern "C" int pf_trace_ev_read(unsigned long long* dst, size_t n) {
  if (n > sizeof(g_cta_ev) / sizeof(g_cta_ev[0])) n = sizeof(g_cta_ev) / sizeof(g_cta_ev[0]);
  return static_cast<int>(cudaMemcpyFromSymbol(dst, g_cta_ev, n * sizeof(unsigned long long)));
}
#endif

namespace {
// One thread waits on an mbarrier that nothing ever arrives at.  The wait gives up after
// limit_ns and records the role in the status word: the path every role of the attention
// kernel takes when one of its bounded waits expires.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    if (!mbar_wait(smem_u32(&bar), 0, nullptr, limit_ns)) atomicOr(&g_watchdog, kWdSelftest);
  }
}
}  // namespace

cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(static_cast<unsigned long long>(limit_ns));
  return cudaGetLastError();
}

cudaError_t read_and_clear_watchdog(unsigned* value) {
  unsigned v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_watchdog, sizeof(v));
  if (e != cudaSuccess) return e;
  *value = v;
  if (v != 0) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_watchdog, &zero, sizeof(zero));
  }
  return e;
}

}  // namespace pf
