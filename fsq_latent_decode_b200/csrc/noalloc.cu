// fsq_decode_attn_noalloc: decode attention for callers that cannot allocate
// device memory themselves.  The scratch that fsq_decode_attn takes as a
// caller-owned workspace lives here in one file-scope device array instead.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"

namespace {

// The library's built-in decode scratch.  Every GPU that loads the library
// holds FSQ_NOALLOC_SCRATCH_BYTES of it until the process exits.  Its name is
// a host-side stand-in in host code: only the address returned by
// cudaGetSymbolAddress (per device context) may be handed to a kernel.
static __device__ __align__(256) unsigned char g_decode_scratch[FSQ_NOALLOC_SCRATCH_BYTES];

// Driver calls that name the current context: its handle, then its unique id
// (ids are never reused, so a device reset, which makes a new primary
// context, also makes a new cache key).
struct CtxApi {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};

const CtxApi &ctx_api() {
  static CtxApi api;
  static std::once_flag once;
  std::call_once(once, []() {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      api.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      api.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  return api;
}

std::mutex g_scratch_mu;
std::map<std::pair<int, unsigned long long>, void *> g_scratch_addr;  // (device, context id) -> address

// Device address of the scratch in the current device's current context,
// looked up once per context with that device current.
fsq_status scratch_on_current_device(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FSQ_ERR_CUDA;
  const CtxApi &api = ctx_api();
  if (!api.get_current || !api.get_id) return FSQ_ERR_CUDA;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (api.get_current(&ctx) != CUDA_SUCCESS) return FSQ_ERR_CUDA;
  if (ctx == nullptr) {
    // no context yet on this thread: make the device's primary context current
    if (cudaSetDevice(dev) != cudaSuccess || api.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
      return FSQ_ERR_CUDA;
  }
  if (api.get_id(ctx, &id) != CUDA_SUCCESS) return FSQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  auto it = g_scratch_addr.find({dev, id});
  if (it == g_scratch_addr.end()) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) return FSQ_ERR_CUDA;
    it = g_scratch_addr.emplace(std::make_pair(dev, id), p).first;
  }
  *out = it->second;
  return FSQ_OK;
}

}  // namespace

extern "C" FSQ_API fsq_status fsq_decode_attn_noalloc(const uint16_t *q, int64_t B, int n_q, int d_h,
                                                      const uint8_t *codes, int64_t code_batch_stride_bytes,
                                                      int64_t T, int G, const uint16_t *W_kv, int n_kv,
                                                      const fsq_attn_opts *opts, void *o, fsq_stream_t stream) {
  const size_t need = fsq_decode_attn_workspace_size(B, T, n_q, n_kv, d_h, G, opts);
  if (B == 0 || need == 0) {
    // empty batch (a no-op) or invalid arguments: the regular entry point
    // returns the same status without touching the device
    return fsq_decode_attn(q, B, n_q, d_h, codes, code_batch_stride_bytes, T, G, W_kv, n_kv, opts, nullptr, 0, o,
                           stream);
  }
  if (need > (size_t)FSQ_NOALLOC_SCRATCH_BYTES) return FSQ_ERR_WORKSPACE;
  void *scratch = nullptr;
  const fsq_status st = scratch_on_current_device(&scratch);
  if (st != FSQ_OK) return st;
  return fsq_decode_attn(q, B, n_q, d_h, codes, code_batch_stride_bytes, T, G, W_kv, n_kv, opts, scratch,
                         (size_t)FSQ_NOALLOC_SCRATCH_BYTES, o, stream);
}

extern "C" FSQ_API fsq_status fsq_decode_attn_noalloc_status(fsq_stream_t stream) {
  void *scratch = nullptr;
  const fsq_status st = scratch_on_current_device(&scratch);
  if (st != FSQ_OK) return st;
  // the error word sits at the start of the scratch, as in a caller's workspace
  return fsq_workspace_status(scratch, (size_t)FSQ_NOALLOC_SCRATCH_BYTES, stream);
}
