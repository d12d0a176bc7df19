// fsq_decode_attn_noalloc: decode attention for callers that cannot allocate
// device memory themselves.  The scratch that fsq_decode_attn takes as a
// caller-owned workspace lives here in one file-scope device array instead.
#include <mutex>

#include "common.cuh"

namespace {

// The library's built-in decode scratch.  Every GPU that loads the library
// holds FSQ_NOALLOC_SCRATCH_BYTES of it until the process exits.  Its name is
// a host-side stand-in in host code: only the address returned by
// cudaGetSymbolAddress (per device) may be handed to a kernel.
static __device__ __align__(256) unsigned char g_decode_scratch[FSQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices];

// Device address of the scratch on the current device, looked up once per
// device with that device current.
fsq_status scratch_on_current_device(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FSQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FSQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) return FSQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
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
