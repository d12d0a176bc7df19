// Append path for decode-step token counts (CUDA cores): u = E x (fp32), FSQ
// threshold count, nibble packing.  Transformer-FSQ summary, Methodology/Architecture eq. (4);
// Theoretical Basis eq. (2); slide deck frame "A wide product code uses four
// bits per coordinate" (ceil(G*b/8) bytes per token).
#include "common.cuh"

namespace fsq {

namespace {

// Few-token append (a decode step appends one token per batch row): one warp
// per (token, byte), i.e. per pair of coordinates (2i, 2i+1); 16-byte loads of
// the token's row and the two encoder rows, fp32 accumulation, warp reduction.
__global__ void __launch_bounds__(256) encode_pack_rows(const uint16_t *__restrict__ x, int64_t n_tok, int64_t ldx,
                                                        int64_t C, const uint16_t *__restrict__ E, int G,
                                                        Thresholds th, uint8_t *__restrict__ codes, int64_t ldc) {
  const int half = G / 2;
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= n_tok * half) return;
  const int64_t t = wid / half;
  const int by = (int)(wid % half);
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + t * ldx);
  const uint4 *e0 = reinterpret_cast<const uint4 *>(E + (int64_t)(2 * by) * C);
  const uint4 *e1 = reinterpret_cast<const uint4 *>(E + (int64_t)(2 * by + 1) * C);
  float a0 = 0.f, a1 = 0.f;
  for (int64_t k = lane; k < C / 8; k += 32) {
    const uint4 xv = xr[k], v0 = e0[k], v1 = e1[k];
    const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
    const uint32_t s0[4] = {v0.x, v0.y, v0.z, v0.w};
    const uint32_t s1[4] = {v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float xl = __uint_as_float(xs[j] << 16), xh = __uint_as_float(xs[j] & 0xFFFF0000u);
      a0 = fmaf(xl, __uint_as_float(s0[j] << 16), a0);
      a0 = fmaf(xh, __uint_as_float(s0[j] & 0xFFFF0000u), a0);
      a1 = fmaf(xl, __uint_as_float(s1[j] << 16), a1);
      a1 = fmaf(xh, __uint_as_float(s1[j] & 0xFFFF0000u), a1);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    a0 += __shfl_xor_sync(0xffffffffu, a0, o);
    a1 += __shfl_xor_sync(0xffffffffu, a1, o);
  }
  if (lane == 0) codes[t * ldc + by] = (uint8_t)(fsq_nibble(a0, th) | (fsq_nibble(a1, th) << 4));
}

// Decode-step append (up to 16 tokens): one CTA per coordinate pair (2i, 2i+1).
// Its 512 threads take interleaved 16-byte chunks of C, so for C <= 4096 every
// load of the kernel is issued at once; E's two rows are read once for all
// tokens.  The 32 per-thread sums (16 tokens x 2 coordinates) are reduced
// across the warp by a transposing butterfly (31 shuffles, lane l ends with
// sum l), then across the 16 warps in shared memory.
constexpr int kFewTok = 16;
constexpr int kFewWarps = 16;
__global__ void __launch_bounds__(kFewWarps * 32, 1)
    encode_pack_few(const uint16_t *__restrict__ x, int n_tok, int64_t ldx, int64_t C,
                    const uint16_t *__restrict__ E, int G, Thresholds th, uint8_t *__restrict__ codes, int64_t ldc) {
  __shared__ float red[kFewWarps][2 * kFewTok];
  const int by = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint4 *e0 = reinterpret_cast<const uint4 *>(E + (int64_t)(2 * by) * C);
  const uint4 *e1 = reinterpret_cast<const uint4 *>(E + (int64_t)(2 * by + 1) * C);
  pdl_wait();
  pdl_trigger();
  float v[2 * kFewTok];  // v[t]: coordinate 2i of token t; v[16 + t]: coordinate 2i+1
#pragma unroll
  for (int i = 0; i < 2 * kFewTok; ++i) v[i] = 0.f;
  for (int64_t k = threadIdx.x; k < C / 8; k += kFewWarps * 32) {
    const uint4 w0 = e0[k], w1 = e1[k];
    uint4 xv[kFewTok];
#pragma unroll
    for (int t = 0; t < kFewTok; ++t)
      xv[t] = t < n_tok ? reinterpret_cast<const uint4 *>(x + (int64_t)t * ldx)[k] : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t s0[4] = {w0.x, w0.y, w0.z, w0.w}, s1[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int t = 0; t < kFewTok; ++t) {
      const uint32_t xs[4] = {xv[t].x, xv[t].y, xv[t].z, xv[t].w};
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const float xl = __uint_as_float(xs[jj] << 16), xh = __uint_as_float(xs[jj] & 0xFFFF0000u);
        v[t] = fmaf(xl, __uint_as_float(s0[jj] << 16), fmaf(xh, __uint_as_float(s0[jj] & 0xFFFF0000u), v[t]));
        v[kFewTok + t] =
            fmaf(xl, __uint_as_float(s1[jj] << 16), fmaf(xh, __uint_as_float(s1[jj] & 0xFFFF0000u), v[kFewTok + t]));
      }
    }
  }
  // butterfly: at offset o a lane keeps the half of its values selected by
  // (lane & o) and adds the partner's copy of that half
#pragma unroll
  for (int o = 16, n = 16; o; o >>= 1, n >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n; ++i) {
      const float send = up ? v[i] : v[i + n];
      const float keep = up ? v[i + n] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  red[warp][lane] = v[0];
  __syncthreads();
  if (threadIdx.x < n_tok) {
    const int t = threadIdx.x;
    float u0 = 0.f, u1 = 0.f;
#pragma unroll
    for (int w = 0; w < kFewWarps; ++w) {
      u0 += red[w][t];
      u1 += red[w][kFewTok + t];
    }
    codes[(int64_t)t * ldc + by] = (uint8_t)(fsq_nibble(u0, th) | (fsq_nibble(u1, th) << 4));
  }
}

__global__ void quantize_pack_f32_kernel(const float *__restrict__ u, int64_t n_tok, int G, Thresholds th,
                                         uint8_t *__restrict__ codes, int64_t ldc) {
  const int half = G / 2;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_tok * half) return;
  int64_t t = i / half;
  int b = (int)(i % half);
  float2 v = *reinterpret_cast<const float2 *>(u + t * G + 2 * b);
  codes[t * ldc + b] = (uint8_t)(fsq_nibble(v.x, th) | (fsq_nibble(v.y, th) << 4));
}

}  // namespace

cudaError_t launch_encode_pack_tc(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C, const uint16_t *E, int G,
                                  const Thresholds &th, uint8_t *codes, int64_t ldc, uint32_t *status,
                                  uint32_t stall_ns, cudaStream_t s);

// Decode-step appends (up to 64 tokens) on CUDA cores; prefill-sized ones on
// the tensor cores (encode_tc.cu).
cudaError_t launch_encode_pack_simt(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C,
                                    const uint16_t *E, int G, const Thresholds &th, uint8_t *codes,
                                    int64_t ldc, uint32_t *status, uint32_t stall_ns, cudaStream_t s) {
  if (n_tok <= kFewTok) {
    return launch_pdl(encode_pack_few, dim3((unsigned)(G / 2)), dim3(kFewWarps * 32), 0, s, x, (int)n_tok, ldx, C, E,
                      G, th, codes, ldc);
  }
  if (n_tok <= 64) {
    const int64_t warps = n_tok * (G / 2);
    encode_pack_rows<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(x, n_tok, ldx, C, E, G, th, codes, ldc);
    return cudaGetLastError();
  }
  return launch_encode_pack_tc(x, n_tok, ldx, C, E, G, th, codes, ldc, status, stall_ns, s);
}

cudaError_t launch_quantize_pack_f32(const float *u, int64_t n_tok, int G, const Thresholds &th,
                                     uint8_t *codes, int64_t ldc, cudaStream_t s) {
  int64_t n = n_tok * (G / 2);
  unsigned blocks = (unsigned)((n + 255) / 256);
  quantize_pack_f32_kernel<<<blocks, 256, 0, s>>>(u, n_tok, G, th, codes, ldc);
  return cudaGetLastError();
}

}  // namespace fsq
