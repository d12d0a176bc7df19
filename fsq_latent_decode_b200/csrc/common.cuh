// Shared device/host helpers of the CUDA library (not used by the oracle).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <map>
#include <mutex>
#include <utility>

#include "../../include/fsq.h"

namespace fsq {

// B200: 148 SMs.  Launch planning uses this constant so that workspace sizes
// depend only on the call's arguments (and can be computed without a device).
constexpr int kNumSMs = 148;

// 1/ln(2): scores are kept in the log2 domain so the softmax uses exp2.
constexpr float kLog2e = 1.4426950408889634f;

// Supported level counts L and their code widths b = log2 L ([D] backup frame
// "the grid size is an allocation choice", Table 8: 4, 16 and 256 levels).
constexpr int kMaxLevels = 256;
__host__ __device__ constexpr int bits_of_levels(int L) { return L == 4 ? 2 : L == 16 ? 4 : L == 256 ? 8 : 0; }

// The L-1 ascending fp32 decision thresholds of eq. (2) at L levels.
template <int L>
struct Thresholds {
  float th[L - 1];
};

__device__ __forceinline__ float bf16_to_f32(uint16_t v) {
  return __uint_as_float(((uint32_t)v) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t *>(&b);
}

// Code = number of thresholds at or below u (0..L-1); level = code - L/2.
// Up to 16 levels every threshold is compared; at 256 levels a binary search
// over the ascending table finds the same count (8 comparisons).  Kernels
// take the table as a __grid_constant__ parameter, so indexing it reads the
// parameter space directly.
template <int L>
__device__ __forceinline__ uint32_t fsq_code(float u, const Thresholds<L> &t) {
  uint32_t n = 0;
  if constexpr (L <= 16) {
#pragma unroll
    for (int k = 0; k < L - 1; ++k) n += (u >= t.th[k]) ? 1u : 0u;
  } else {
#pragma unroll
    for (uint32_t step = L / 2; step; step >>= 1)
      if (u >= t.th[n + step - 1]) n += step;  // index <= L - 1 - step
  }
  return n;
}

// Split-merge plan of the absorbed form (merge.cu): CTAs per (kv head, batch
// row), one per slice of G, and the workspace its sliced mode needs.
struct MergePlan {
  int ngq = 1;
  size_t slab_bytes = 0, cnt_bytes = 0;
};
MergePlan merge_plan(int S, int64_t B, int n_q, int n_kv, int G);

// Workspace of the sliced merge: the merged latents of every slice and one
// arrival count per (batch row, kv head), which the query prologue of the
// same call zeroes (ncnt counts; slab and cnt are null in direct mode).
struct MergeScratch {
  float *slab;
  uint32_t *cnt;
  int ncnt;
};

// Workspace header: the device error word lives in the first 4 bytes.
constexpr size_t kWsHeader = 256;

__device__ __forceinline__ void record_error(uint32_t *err, int status) {
  atomicCAS(err, 0u, (uint32_t)(-status));
}

// Cached tokens of batch row b: T, or seq_lens[b] for a ragged batch, clamped
// into [1, T]; a value outside records FSQ_ERR_INVALID_ARG when `report`
// (one thread per row reports, after the call's error word was cleared).
__device__ __forceinline__ int64_t row_len(const int32_t *seq_lens, int64_t b, int64_t T, uint32_t *err,
                                           bool report) {
  if (seq_lens == nullptr) return T;
  const int64_t v = seq_lens[b];
  if (v >= 1 && v <= T) return v;
  if (report) record_error(err, FSQ_ERR_INVALID_ARG);
  return v < 1 ? 1 : T;
}

// Multi-query calls (chunked prefill, speculative decoding) run the n_new
// queries of a cache row as consecutive virtual rows r = b * n_new + i of the
// same kernels.  Query i of cache row b (whose length is L_b, the new tokens
// included) sits at position L_b - n_new + i and attends causally to the
// first L_b - n_new + i + 1 cached tokens.  One thread per cache row reports
// (from its query 0) a row too short for its queries, clamped to length 1.
__device__ __forceinline__ int64_t query_len(const int32_t *seq_lens, int64_t r, int n_new, int64_t T, uint32_t *err,
                                             bool report) {
  const int64_t b = r / n_new;
  const int i = (int)(r - b * n_new);
  const int64_t len = row_len(seq_lens, b, T, err, report && i == 0) - (n_new - 1 - i);
  if (len >= 1) return len;
  if (report && i == 0) record_error(err, FSQ_ERR_INVALID_ARG);
  return 1;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Raise a kernel's dynamic shared-memory limit on the current device, once:
// the attribute is per function and device and stays set, so later calls
// needing no more than the largest limit set so far skip the driver call.
inline cudaError_t ensure_smem_limit(const void *fn, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::map<std::pair<const void *, int>, size_t> done;
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find({fn, dev});
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done[{fn, dev}] = bytes;
  return e;
}

// Programmatic dependent launch.  Kernels launched with launch_pdl may start
// while the previous kernel of the stream is still running, once every CTA of
// that kernel has called pdl_trigger (or exited).  A kernel reads nothing that
// the previous kernels write before pdl_wait, which returns when they have
// completed and their writes are visible.  Every kernel here completes only
// after its own pdl_wait, so waiting for the immediate predecessor also covers
// all kernels before it.  The query prologue triggers only after its wait, so
// the split kernel, which requests code tiles before its own wait, starts
// after the codes are complete; the merge never triggers early, so work after
// a decode call starts once its output is written.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Profiling events around the main kernel.  While the stream is being
// captured into a graph they are recorded as external events (event nodes of
// the graph); otherwise as plain records.
inline void record_prof_event(void *ev, cudaStream_t st) {
  if (!ev) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags((cudaEvent_t)ev, st, cudaEventRecordExternal);
  else
    cudaEventRecord((cudaEvent_t)ev, st);
}

}  // namespace fsq
