// Append path for decode-step token counts (CUDA cores): u = E x (fp32), FSQ
// threshold count, bit packing.  Transformer-FSQ summary, Methodology/Architecture eq. (4);
// Theoretical Basis eq. (2); slide deck frame "A wide product code uses four
// bits per coordinate" (ceil(G*b/8) bytes per token) and backup frame "the
// grid size is an allocation choice" (L = 4, 16, 256 at b = 2, 4, 8 bits).
#include "common.cuh"
#include "encode.cuh"

namespace fsq {

namespace {

// Packing constants of L levels: b bits per code, PER codes per byte, and the
// coordinate chunk of the few-token kernel (whole bytes and whole pairs).
template <int L>
struct Pk {
  static constexpr int BITS = bits_of_levels(L);
  static constexpr int PER = 8 / BITS;
  static constexpr int CP = PER < 2 ? 2 : PER;
  static_assert(BITS > 0, "unsupported level count");
};

// Few-token append (a decode step appends one token per batch row): one warp
// per (token, byte), i.e. per group of PER coordinates; 16-byte loads of the
// token's row and the encoder rows, fp32 accumulation, warp reduction.
template <int L>
__global__ void __launch_bounds__(256) encode_pack_rows(const uint16_t *__restrict__ x, int64_t n_tok, int64_t ldx,
                                                        int64_t C, const uint16_t *__restrict__ E, int G,
                                                        const __grid_constant__ Thresholds<L> th,
                                                        const CodeRows dst) {
  constexpr int P = Pk<L>::PER, BITS = Pk<L>::BITS;
  const int rb = G / P;  // bytes per token row
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= n_tok * rb) return;
  const int64_t t = wid / rb;
  const int by = (int)(wid % rb);
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + t * ldx);
  const uint4 *er[P];
#pragma unroll
  for (int c = 0; c < P; ++c) er[c] = reinterpret_cast<const uint4 *>(E + (int64_t)(P * by + c) * C);
  float a[P];
#pragma unroll
  for (int c = 0; c < P; ++c) a[c] = 0.f;
  for (int64_t k = lane; k < C / 8; k += 32) {
    const uint4 xv = xr[k];
    const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int c = 0; c < P; ++c) {
      const uint4 ev = er[c][k];
      const uint32_t es[4] = {ev.x, ev.y, ev.z, ev.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float xl = __uint_as_float(xs[j] << 16), xh = __uint_as_float(xs[j] & 0xFFFF0000u);
        a[c] = fmaf(xl, __uint_as_float(es[j] << 16), a[c]);
        a[c] = fmaf(xh, __uint_as_float(es[j] & 0xFFFF0000u), a[c]);
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1)
#pragma unroll
    for (int c = 0; c < P; ++c) a[c] += __shfl_xor_sync(0xffffffffu, a[c], o);
  if (lane == 0) {
    uint32_t v = 0;
#pragma unroll
    for (int c = 0; c < P; ++c) v |= fsq_code<L>(a[c], th) << (BITS * c);
    dst.row(t)[by] = (uint8_t)v;
  }
}

// Decode-step append (up to 16 tokens): one CTA per chunk of CP coordinates
// (whole bytes, taken a pair (2i, 2i+1) at a time).  Its 512 threads take
// interleaved 16-byte chunks of C, so for C <= 4096 every load of a pair is
// issued at once; E's rows are read once for all tokens.  The 32 per-thread
// sums of a pair (16 tokens x 2 coordinates) are reduced across the warp by a
// transposing butterfly (31 shuffles, lane l ends with sum l), then across
// the 16 warps in shared memory.
constexpr int kFewTok = 16;
constexpr int kFewWarps = 16;
template <int L>
__global__ void __launch_bounds__(kFewWarps * 32, 1)
    encode_pack_few(const uint16_t *__restrict__ x, int n_tok, int64_t ldx, int64_t C,
                    const uint16_t *__restrict__ E, int G, const __grid_constant__ Thresholds<L> th,
                    const CodeRows dst) {
  constexpr int P = Pk<L>::PER, BITS = Pk<L>::BITS, CP = Pk<L>::CP, NPAIR = CP / 2;
  __shared__ float red[NPAIR][kFewWarps][2 * kFewTok];
  const int c0 = blockIdx.x * CP;  // first coordinate of this chunk
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
#pragma unroll 1
  for (int pp = 0; pp < NPAIR; ++pp) {
    const uint4 *e0 = reinterpret_cast<const uint4 *>(E + (int64_t)(c0 + 2 * pp) * C);
    const uint4 *e1 = reinterpret_cast<const uint4 *>(E + (int64_t)(c0 + 2 * pp + 1) * C);
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
          v[kFewTok + t] = fmaf(xl, __uint_as_float(s1[jj] << 16),
                                fmaf(xh, __uint_as_float(s1[jj] & 0xFFFF0000u), v[kFewTok + t]));
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
    red[pp][warp][lane] = v[0];
  }
  __syncthreads();
  if (threadIdx.x < n_tok) {
    const int t = threadIdx.x;
    uint32_t cw[CP];
#pragma unroll
    for (int pp = 0; pp < NPAIR; ++pp) {
      float u0 = 0.f, u1 = 0.f;
#pragma unroll
      for (int w = 0; w < kFewWarps; ++w) {
        u0 += red[pp][w][t];
        u1 += red[pp][w][kFewTok + t];
      }
      cw[2 * pp] = fsq_code<L>(u0, th);
      cw[2 * pp + 1] = fsq_code<L>(u1, th);
    }
#pragma unroll
    for (int by = 0; by < CP / P; ++by) {
      uint32_t v = 0;
#pragma unroll
      for (int c = 0; c < P; ++c) v |= cw[by * P + c] << (BITS * c);
      dst.row(t)[c0 / P + by] = (uint8_t)v;
    }
  }
}

// One thread per output byte: its PER consecutive coordinates of u.
template <int L>
__global__ void quantize_pack_f32_kernel(const float *__restrict__ u, int64_t n_tok, int G,
                                         const __grid_constant__ Thresholds<L> th, uint8_t *__restrict__ codes,
                                         int64_t ldc) {
  constexpr int P = Pk<L>::PER, BITS = Pk<L>::BITS;
  const int rb = G / P;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_tok * rb) return;
  const int64_t t = i / rb;
  const int by = (int)(i % rb);
  const float *ur = u + t * G + P * by;
  uint32_t v = 0;
#pragma unroll
  for (int c = 0; c < P; ++c) v |= fsq_code<L>(ur[c], th) << (BITS * c);
  codes[t * ldc + by] = (uint8_t)v;
}

template <int L>
Thresholds<L> table_of(const float *th) {
  Thresholds<L> t;
  for (int k = 0; k < L - 1; ++k) t.th[k] = th[k];
  return t;
}

}  // namespace

template <int L>
cudaError_t launch_encode_pack_tc(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C, const uint16_t *E, int G,
                                  const Thresholds<L> &th, const CodeRows &dst, uint32_t *status,
                                  uint32_t stall_ns, cudaStream_t s);

namespace {
// Decode-step appends (up to 64 tokens) on CUDA cores; prefill-sized ones on
// the tensor cores (encode_tc.cu).
template <int L>
cudaError_t encode_levels(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C, const uint16_t *E, int G,
                          const float *th_host, const CodeRows &dst, uint32_t *status, uint32_t stall_ns,
                          cudaStream_t s) {
  const Thresholds<L> th = table_of<L>(th_host);
  if (n_tok <= kFewTok) {
    return launch_pdl(encode_pack_few<L>, dim3((unsigned)(G / Pk<L>::CP)), dim3(kFewWarps * 32), 0, s, x, (int)n_tok,
                      ldx, C, E, G, th, dst);
  }
  if (n_tok <= 64) {
    const int64_t warps = n_tok * (G / Pk<L>::PER);
    encode_pack_rows<L><<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(x, n_tok, ldx, C, E, G, th, dst);
    return cudaGetLastError();
  }
  return launch_encode_pack_tc<L>(x, n_tok, ldx, C, E, G, th, dst, status, stall_ns, s);
}

template <int L>
cudaError_t quantize_levels(const float *u, int64_t n_tok, int G, const float *th_host, uint8_t *codes, int64_t ldc,
                            cudaStream_t s) {
  const int64_t n = n_tok * (G / Pk<L>::PER);
  const unsigned blocks = (unsigned)((n + 255) / 256);
  quantize_pack_f32_kernel<L><<<blocks, 256, 0, s>>>(u, n_tok, G, table_of<L>(th_host), codes, ldc);
  return cudaGetLastError();
}
}  // namespace

// th: the levels-1 thresholds of fsq_thresholds; per_row / row_stride: the
// grouping of the destination rows (CodeRows; per_row = 0: one stride ldc).
cudaError_t launch_encode_pack(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C, const uint16_t *E, int G,
                               int levels, const float *th, uint8_t *codes, int64_t ldc, int64_t per_row,
                               int64_t row_stride, uint32_t *status, uint32_t stall_ns, cudaStream_t s) {
  const CodeRows dst{codes, ldc, per_row, row_stride};
  switch (levels) {
    case 4: return encode_levels<4>(x, n_tok, ldx, C, E, G, th, dst, status, stall_ns, s);
    case 16: return encode_levels<16>(x, n_tok, ldx, C, E, G, th, dst, status, stall_ns, s);
    case 256: return encode_levels<256>(x, n_tok, ldx, C, E, G, th, dst, status, stall_ns, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_quantize_pack_f32(const float *u, int64_t n_tok, int G, int levels, const float *th,
                                     uint8_t *codes, int64_t ldc, cudaStream_t s) {
  switch (levels) {
    case 4: return quantize_levels<4>(u, n_tok, G, th, codes, ldc, s);
    case 16: return quantize_levels<16>(u, n_tok, G, th, codes, ldc, s);
    case 256: return quantize_levels<256>(u, n_tok, G, th, codes, ldc, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace fsq
