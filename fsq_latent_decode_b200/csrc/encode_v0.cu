// Append path, portable SIMT kernels: u = E x (fp32), FSQ threshold count,
// nibble packing.  Transformer-FSQ summary, Methodology/Architecture eq. (4);
// Theoretical Basis eq. (2); slide deck frame "A wide product code uses four
// bits per coordinate" (ceil(G*b/8) bytes per token).
#include "common.cuh"

namespace fsq {

namespace {

constexpr int kEncTok = 32;  // tokens per CTA
constexpr int kEncK = 32;    // K (= C) chunk

__global__ void __launch_bounds__(256) encode_pack_simt(const uint16_t *__restrict__ x, int64_t n_tok,
                                                        int64_t ldx, int64_t C,
                                                        const uint16_t *__restrict__ E, int G,
                                                        Thresholds th, uint8_t *__restrict__ codes,
                                                        int64_t ldc) {
  __shared__ float xs[kEncTok][kEncK + 1];
  __shared__ float es[kEncK][FSQ_MAX_G];
  __shared__ uint8_t nib[kEncTok][FSQ_MAX_G];
  const int tid = threadIdx.x;
  const int64_t tok0 = (int64_t)blockIdx.x * kEncTok;
  float acc[kEncTok];
#pragma unroll
  for (int i = 0; i < kEncTok; ++i) acc[i] = 0.f;

  for (int64_t k0 = 0; k0 < C; k0 += kEncK) {
    for (int i = tid; i < kEncTok * kEncK; i += blockDim.x) {
      int t = i / kEncK, k = i % kEncK;
      int64_t tt = tok0 + t;
      xs[t][k] = (tt < n_tok) ? bf16_to_f32(x[tt * ldx + k0 + k]) : 0.f;
    }
    for (int i = tid; i < kEncK * G; i += blockDim.x) {
      int g = i / kEncK, k = i % kEncK;
      es[k][g] = bf16_to_f32(E[(int64_t)g * C + k0 + k]);
    }
    __syncthreads();
    if (tid < G) {
#pragma unroll 4
      for (int k = 0; k < kEncK; ++k) {
        float e = es[k][tid];
#pragma unroll
        for (int t = 0; t < kEncTok; ++t) acc[t] = fmaf(xs[t][k], e, acc[t]);
      }
    }
    __syncthreads();
  }
  if (tid < G) {
#pragma unroll
    for (int t = 0; t < kEncTok; ++t) nib[t][tid] = (uint8_t)fsq_nibble(acc[t], th);
  }
  __syncthreads();
  const int half = G / 2;
  for (int i = tid; i < kEncTok * half; i += blockDim.x) {
    int t = i / half, b = i % half;
    int64_t tt = tok0 + t;
    if (tt < n_tok) codes[tt * ldc + b] = (uint8_t)(nib[t][2 * b] | (nib[t][2 * b + 1] << 4));
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

cudaError_t launch_encode_pack_simt(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C,
                                    const uint16_t *E, int G, const Thresholds &th, uint8_t *codes,
                                    int64_t ldc, cudaStream_t s) {
  dim3 grid((unsigned)((n_tok + kEncTok - 1) / kEncTok));
  encode_pack_simt<<<grid, 256, 0, s>>>(x, n_tok, ldx, C, E, G, th, codes, ldc);
  return cudaGetLastError();
}

cudaError_t launch_quantize_pack_f32(const float *u, int64_t n_tok, int G, const Thresholds &th,
                                     uint8_t *codes, int64_t ldc, cudaStream_t s) {
  int64_t n = n_tok * (G / 2);
  unsigned blocks = (unsigned)((n + 255) / 256);
  quantize_pack_f32_kernel<<<blocks, 256, 0, s>>>(u, n_tok, G, th, codes, ldc);
  return cudaGetLastError();
}

}  // namespace fsq
