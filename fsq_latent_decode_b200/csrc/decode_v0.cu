// Decode attention over packed FSQ codes — portable SIMT kernels.
//
// These are the straightforward forms of the two variants:
//  * ABSORBED: q'_h = W_k^(j)T q_h (prologue), per split s_t = q'_h . z_t,
//    online softmax, acc_h = sum_t p_t z_t; the merge applies W_v^(j) once
//    (Transformer-FSQ summary, Key Design Innovation eq. (6); slide deck frame
//    "Attention pools codes before decoding values").
//  * EXPAND: per tile k_t = W_k^(j) z_t (optionally RoPE_t(N_k(.))) and
//    v_t = W_v^(j) z_t, then standard GQA online-softmax attention
//    (summary eq. (5)).
// The code of a coordinate is b = log2 L bits wide (L = 4, 16 or 256 levels;
// slide deck backup frame "the grid size is an allocation choice"): a byte of
// a row holds 8/b consecutive coordinates, the first in its lowest bits, and a
// level is code - L/2.
// Long contexts are split over token ranges; each split emits (m, l, acc)
// in the log2 domain and a merge kernel combines them by log-sum-exp
// (slide deck frame "The kernel reads codes and never writes reconstructed
// K/V": "merge partials and apply W_v once").
#include "common.cuh"

namespace fsq {

namespace {

constexpr int kNT = 32;        // tokens per tile (absorbed)
constexpr int kMaxNQ = 64;     // query heads per batch row supported here
constexpr int kNTx = 16;       // tokens per tile (expand)
constexpr int kMaxGrp = 16;    // query heads per kv head supported here

// ---------------------------------------------------------------- prologue
// qa[b][h][g] = c * sum_d W_k[j*d_h + d][g] * q[b][h][d],  c = scale*log2(e)
__global__ void absorb_query_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ W_kv,
                                    int n_q, int n_kv, int d_h, int G, float c, float *__restrict__ qa,
                                    uint32_t *err, MergeScratch ms) {
  __shared__ float qs[FSQ_HEAD_DIM];
  const int h = blockIdx.x, b = blockIdx.y;
  const int j = h / (n_q / n_kv);
  if (blockIdx.x == 0 && blockIdx.y == 0) {
    if (threadIdx.x == 0) *err = 0u;
    for (int i = threadIdx.x; i < ms.ncnt; i += blockDim.x) ms.cnt[i] = 0u;
  }
  for (int d = threadIdx.x; d < d_h; d += blockDim.x) qs[d] = bf16_to_f32(q[((int64_t)b * n_q + h) * d_h + d]);
  __syncthreads();
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    float s = 0.f;
    const uint16_t *w = W_kv + (int64_t)j * d_h * G + g;
    for (int d = 0; d < d_h; ++d) s = fmaf(bf16_to_f32(w[(int64_t)d * G]), qs[d], s);
    qa[((int64_t)b * n_q + h) * G + g] = c * s;
  }
}

// ---------------------------------------------------------------- absorbed split
// part layout: [B][S][n_q][2 + G]  (m, l, acc[G]), log2 domain.
__global__ void __launch_bounds__(256) absorbed_split_simt(const float *__restrict__ qa,
                                                           const uint8_t *__restrict__ codes, int64_t bstride,
                                                           int64_t T, const int32_t *__restrict__ seq_lens,
                                                           int n_new, int G, int bits, int n_q, int64_t tps,
                                                           float *__restrict__ part, uint32_t *err) {
  extern __shared__ float sm[];
  float *qs = sm;                                   // [n_q][G]
  float *acc = qs + n_q * G;                        // [n_q][G]
  float *cs = acc + n_q * G;                        // [kNT][G+1]
  float *ps = cs + kNT * (G + 1);                   // [kNT][n_q]
  float *ms = ps + kNT * n_q;                       // [n_q]
  float *ls = ms + n_q;                             // [n_q]
  float *cr = ls + n_q;                             // [n_q]
  const int tid = threadIdx.x, nth = blockDim.x;
  const int s = blockIdx.x, b = blockIdx.y, S = gridDim.x;
  const int64_t t0 = (int64_t)s * tps;
  // empty past the row's end (ragged batch, causal query); grid row b reads cache row b / n_new
  const int64_t t1 = min(query_len(seq_lens, b, n_new, T, err, s == 0 && tid == 0), t0 + tps);
  const int per = 8 / bits, rb = G / per;  // coordinates per byte, bytes per row
  const uint32_t mask = (1u << bits) - 1u;
  const float off = (float)(1 << (bits - 1));  // L/2
  const uint8_t *cb = codes + (int64_t)(b / n_new) * bstride;

  for (int i = tid; i < n_q * G; i += nth) {
    qs[i] = qa[(int64_t)b * n_q * G + i];
    acc[i] = 0.f;
  }
  for (int h = tid; h < n_q; h += nth) {
    ms[h] = -INFINITY;
    ls[h] = 0.f;
  }
  __syncthreads();

  for (int64_t tt = t0; tt < t1; tt += kNT) {
    const int nv = (int)min((int64_t)kNT, t1 - tt);
    for (int i = tid; i < kNT * rb; i += nth) {
      const int t = i / rb, by = i % rb;
      const uint32_t v = t < nv ? cb[(tt + t) * rb + by] : 0u;
      for (int c = 0; c < per; ++c)
        cs[t * (G + 1) + per * by + c] = t < nv ? (float)((v >> (bits * c)) & mask) - off : 0.f;
    }
    __syncthreads();
    for (int i = tid; i < kNT * n_q; i += nth) {
      int t = i % kNT, h = i / kNT;
      float sc = -INFINITY;
      if (t < nv) {
        sc = 0.f;
        const float *c = cs + t * (G + 1);
        const float *qq = qs + h * G;
        for (int g = 0; g < G; ++g) sc = fmaf(c[g], qq[g], sc);
      }
      ps[t * n_q + h] = sc;
    }
    __syncthreads();
    for (int h = tid; h < n_q; h += nth) {
      float mx = ms[h];
      for (int t = 0; t < nv; ++t) mx = fmaxf(mx, ps[t * n_q + h]);
      float corr = exp2f(ms[h] - mx);  // exp2(-inf) = 0 on the first tile
      float l = ls[h] * corr;
      for (int t = 0; t < kNT; ++t) {
        float p = (t < nv) ? exp2f(ps[t * n_q + h] - mx) : 0.f;
        ps[t * n_q + h] = p;
        l += p;
      }
      ms[h] = mx;
      ls[h] = l;
      cr[h] = corr;
    }
    __syncthreads();
    for (int i = tid; i < n_q * G; i += nth) {
      int h = i / G, g = i % G;
      float a = acc[i] * cr[h];
      for (int t = 0; t < nv; ++t) a = fmaf(ps[t * n_q + h], cs[t * (G + 1) + g], a);
      acc[i] = a;
    }
    __syncthreads();
  }
  float *out = part + (((int64_t)b * S + s) * n_q) * (2 + G);
  for (int h = tid; h < n_q; h += nth) {
    out[h * (2 + G)] = ms[h];
    out[h * (2 + G) + 1] = ls[h];
  }
  for (int i = tid; i < n_q * G; i += nth) {
    int h = i / G, g = i % G;
    out[h * (2 + G) + 2 + g] = acc[i];
  }
}

// ---------------------------------------------------------------- merge + W_v
// o[b][h][d] = W_v^(j)[d] . (sum_s w_s acc_s) / (sum_s w_s l_s),  w_s = 2^(m_s - m)
__global__ void merge_absorbed_kernel(const float *__restrict__ part, int S, int n_q, int n_kv, int d_h, int G,
                                      const uint16_t *__restrict__ W_kv, void *o, int out_fp32) {
  __shared__ float ab[FSQ_MAX_G];
  __shared__ float wsh[1024];
  __shared__ float linv;
  const int h = blockIdx.x, b = blockIdx.y;
  const int j = h / (n_q / n_kv);
  const float *pb = part + ((int64_t)b * S * n_q + h) * (2 + G);
  const int64_t sstride = (int64_t)n_q * (2 + G);
  if (threadIdx.x == 0) {
    float m = -INFINITY;
    for (int s = 0; s < S; ++s) m = fmaxf(m, pb[s * sstride]);
    float l = 0.f;
    for (int s = 0; s < S; ++s) {
      float w = exp2f(pb[s * sstride] - m);
      wsh[s] = w;
      l += w * pb[s * sstride + 1];
    }
    linv = 1.f / l;
  }
  __syncthreads();
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    float a = 0.f;
    for (int s = 0; s < S; ++s) a = fmaf(wsh[s], pb[s * sstride + 2 + g], a);
    ab[g] = a * linv;
  }
  __syncthreads();
  for (int d = threadIdx.x; d < d_h; d += blockDim.x) {
    const uint16_t *w = W_kv + ((int64_t)(n_kv + j) * d_h + d) * G;
    float v = 0.f;
    for (int g = 0; g < G; ++g) v = fmaf(bf16_to_f32(w[g]), ab[g], v);
    int64_t oi = ((int64_t)b * n_q + h) * d_h + d;
    if (out_fp32) reinterpret_cast<float *>(o)[oi] = v;
    else reinterpret_cast<uint16_t *>(o)[oi] = f32_to_bf16_rn(v);
  }
}

// ---------------------------------------------------------------- expand split
// grid (S, B, n_kv), 128 threads (thread = output dimension d).
// part layout: [B][S][n_q][2 + d_h].
__global__ void __launch_bounds__(128) expand_split_simt(const uint16_t *__restrict__ q,
                                                         const uint8_t *__restrict__ codes, int64_t bstride,
                                                         int64_t T, const int32_t *__restrict__ seq_lens,
                                                         int n_new, int G, int bits, int n_q, int n_kv,
                                                         const uint16_t *__restrict__ W_kv,
                                                         float c, int64_t tps, int rope_knorm, float rope_base,
                                                         const uint16_t *__restrict__ gain, float eps,
                                                         float *__restrict__ part, uint32_t *err) {
  constexpr int D = FSQ_HEAD_DIM;
  extern __shared__ float sm[];
  uint16_t *wk = reinterpret_cast<uint16_t *>(sm);          // [G][D]
  uint16_t *wv = wk + G * D;                                  // [G][D]
  float *cs = reinterpret_cast<float *>(wv + G * D);          // [kNTx][G]
  float *ks = cs + kNTx * G;                                  // [kNTx][D]
  float *qs = ks + kNTx * D;                                  // [grp][D]
  float *ss = qs + kMaxGrp * D;                               // [grp][kNTx]
  float *red = ss + kMaxGrp * kNTx;                           // [kNTx][4]
  const int d = threadIdx.x, warp = d / 32, lane = d % 32;
  const int s = blockIdx.x, b = blockIdx.y, j = blockIdx.z, S = gridDim.x;
  const int grp = n_q / n_kv;
  const int64_t t0 = (int64_t)s * tps;
  const int64_t t1 = min(query_len(seq_lens, b, n_new, T, err, s == 0 && j == 0 && d == 0), t0 + tps);
  const int per = 8 / bits, rb = G / per;  // coordinates per byte, bytes per row
  const uint32_t mask = (1u << bits) - 1u;
  const float off = (float)(1 << (bits - 1));  // L/2
  const uint8_t *cb = codes + (int64_t)(b / n_new) * bstride;

  for (int i = d; i < G * D; i += D) {
    int dd = i / G, g = i % G;
    wk[g * D + dd] = W_kv[((int64_t)j * D + dd) * G + g];
    wv[g * D + dd] = W_kv[((int64_t)(n_kv + j) * D + dd) * G + g];
  }
  for (int hh = 0; hh < grp; ++hh) qs[hh * D + d] = bf16_to_f32(q[((int64_t)b * n_q + j * grp + hh) * D + d]);
  const float gd = (rope_knorm && gain) ? bf16_to_f32(gain[d]) : 1.f;
  // RoPE frequency of this dimension (half-split pairing: d and d +/- D/2)
  const double inv_freq = pow((double)rope_base, -2.0 * (double)(d % (D / 2)) / (double)D);
  float o[kMaxGrp], m[kMaxGrp], l[kMaxGrp];
#pragma unroll
  for (int hh = 0; hh < kMaxGrp; ++hh) { o[hh] = 0.f; m[hh] = -INFINITY; l[hh] = 0.f; }
  __syncthreads();

  for (int64_t tt = t0; tt < t1; tt += kNTx) {
    const int nv = (int)min((int64_t)kNTx, t1 - tt);
    for (int i = d; i < kNTx * rb; i += D) {
      const int t = i / rb, by = i % rb;
      const uint32_t v = t < nv ? cb[(tt + t) * rb + by] : 0u;
      for (int c = 0; c < per; ++c)
        cs[t * G + per * by + c] = t < nv ? (float)((v >> (bits * c)) & mask) - off : 0.f;
    }
    __syncthreads();
    float vr[kNTx];
#pragma unroll
    for (int t = 0; t < kNTx; ++t) {
      float kk = 0.f, vv = 0.f;
      const float *cz = cs + t * G;
      for (int g = 0; g < G; ++g) {
        float z = cz[g];
        kk = fmaf(bf16_to_f32(wk[g * D + d]), z, kk);
        vv = fmaf(bf16_to_f32(wv[g * D + d]), z, vv);
      }
      ks[t * D + d] = kk;
      vr[t] = vv;
    }
    __syncthreads();
    if (rope_knorm) {
      // N_k: RMS norm over d, per token
#pragma unroll
      for (int t = 0; t < kNTx; ++t) {
        float x = ks[t * D + d];
        float sq = x * x;
        for (int off = 16; off; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
        if (lane == 0) red[t * 4 + warp] = sq;
      }
      __syncthreads();
      float kn[kNTx];
#pragma unroll
      for (int t = 0; t < kNTx; ++t) {
        float ms2 = (red[t * 4] + red[t * 4 + 1] + red[t * 4 + 2] + red[t * 4 + 3]) / (float)D;
        kn[t] = ks[t * D + d] * gd * rsqrtf(ms2 + eps);
      }
      __syncthreads();
#pragma unroll
      for (int t = 0; t < kNTx; ++t) ks[t * D + d] = kn[t];
      __syncthreads();
      // RoPE_t at position t (cache index)
#pragma unroll
      for (int t = 0; t < kNTx; ++t) {
        double ang = (double)(tt + t) * inv_freq;
        double sn, cn;
        sincos(ang, &sn, &cn);
        float a = ks[t * D + (d % (D / 2))], bq = ks[t * D + (d % (D / 2)) + D / 2];
        kn[t] = (d < D / 2) ? (float)(a * cn - bq * sn) : (float)(a * sn + bq * cn);
      }
      __syncthreads();
#pragma unroll
      for (int t = 0; t < kNTx; ++t) ks[t * D + d] = kn[t];
      __syncthreads();
    }
    // scores: warp w handles (head, token) pairs w, w+4, ...
    for (int pi = warp; pi < grp * kNTx; pi += 4) {
      int hh = pi / kNTx, t = pi % kNTx;
      float sc = 0.f;
      for (int dd = lane; dd < D; dd += 32) sc = fmaf(qs[hh * D + dd], ks[t * D + dd], sc);
      for (int off = 16; off; off >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, off);
      if (lane == 0) ss[hh * kNTx + t] = (t < nv) ? sc * c : -INFINITY;
    }
    __syncthreads();
    for (int hh = 0; hh < grp; ++hh) {
      float mx = m[hh];
      for (int t = 0; t < nv; ++t) mx = fmaxf(mx, ss[hh * kNTx + t]);
      float corr = exp2f(m[hh] - mx);
      float acc = o[hh] * corr, ll = l[hh] * corr;
#pragma unroll
      for (int t = 0; t < kNTx; ++t) {
        float p = (t < nv) ? exp2f(ss[hh * kNTx + t] - mx) : 0.f;
        ll += p;
        acc = fmaf(p, vr[t], acc);
      }
      o[hh] = acc;
      l[hh] = ll;
      m[hh] = mx;
    }
    __syncthreads();
  }
  for (int hh = 0; hh < grp; ++hh) {
    const int h = j * grp + hh;
    float *out = part + (((int64_t)b * S + s) * n_q + h) * (2 + D);
    if (d == 0) {
      out[0] = m[hh];
      out[1] = l[hh];
    }
    out[2 + d] = o[hh];
  }
}

__global__ void merge_expand_kernel(const float *__restrict__ part, int S, int n_q, int d_h, void *o,
                                    int out_fp32) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const float *pb = part + ((int64_t)b * S * n_q + h) * (2 + d_h);
  const int64_t sstride = (int64_t)n_q * (2 + d_h);
  float m = -INFINITY;
  for (int s = 0; s < S; ++s) m = fmaxf(m, pb[s * sstride]);
  float l = 0.f, a = 0.f;
  for (int s = 0; s < S; ++s) {
    float w = exp2f(pb[s * sstride] - m);
    l = fmaf(w, pb[s * sstride + 1], l);
    a = fmaf(w, pb[s * sstride + 2 + d], a);
  }
  float v = a / l;
  int64_t oi = ((int64_t)b * n_q + h) * d_h + d;
  if (out_fp32) reinterpret_cast<float *>(o)[oi] = v;
  else reinterpret_cast<uint16_t *>(o)[oi] = f32_to_bf16_rn(v);
}

__global__ void clear_err_kernel(uint32_t *err) { *err = 0u; }

}  // namespace

bool merge_grouped_supported(int n_q, int n_kv);
cudaError_t merge_grouped_launch(const float *part, int S, int64_t B, int n_q, int n_kv, int G,
                                 const uint16_t *W_kv, void *o, int out_fp32, float *slab, uint32_t *cnt,
                                 cudaStream_t st, int fold_bytes);

// Group sizes 1, 2, 4, 8, 16 share W_v^(j) reads across the group (merge.cu);
// others take one CTA per query head.  fold_bytes: the partials carry 8-bit
// codes read as nibble pairs (G of them = 2 x the latent width; grouped merge only).
cudaError_t merge_absorbed_launch(const float *part, int S, int64_t B, int n_q, int n_kv, int d_h, int G,
                                  const uint16_t *W_kv, void *o, int out_fp32, MergeScratch ms, cudaStream_t st,
                                  int fold_bytes) {
  if (merge_grouped_supported(n_q, n_kv))
    return merge_grouped_launch(part, S, B, n_q, n_kv, G, W_kv, o, out_fp32, ms.slab, ms.cnt, st, fold_bytes);
  if (fold_bytes) return cudaErrorInvalidValue;
  merge_absorbed_kernel<<<dim3(n_q, (unsigned)B), 256, 0, st>>>(part, S, n_q, n_kv, d_h, G, W_kv, o, out_fp32);
  return cudaGetLastError();
}

// Log-sum-exp merge of expanded-value partials [B][S][n_q][2 + d_h].
cudaError_t merge_expand_launch(const float *part, int S, int64_t B, int n_q, int d_h, void *o, int out_fp32,
                                cudaStream_t st) {
  merge_expand_kernel<<<dim3(n_q, (unsigned)B), d_h, 0, st>>>(part, S, n_q, d_h, o, out_fp32);
  return cudaGetLastError();
}

size_t absorbed_simt_smem(int n_q, int G) {
  return sizeof(float) * (2 * (size_t)n_q * G + kNT * (G + 1) + kNT * n_q + 3 * n_q);
}

size_t expand_simt_smem(int G) {
  return 2 * sizeof(uint16_t) * (size_t)G * FSQ_HEAD_DIM +
         sizeof(float) * (kNTx * G + kNTx * FSQ_HEAD_DIM + kMaxGrp * FSQ_HEAD_DIM + kMaxGrp * kNTx + kNTx * 4);
}

int simt_max_nq() { return kMaxNQ; }
int simt_max_grp() { return kMaxGrp; }

cudaError_t launch_absorbed_simt(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int n_new,
                                 int64_t T, const int32_t *seq_lens, int n_q, int n_kv, int d_h, int G, int bits,
                                 const uint16_t *W_kv,
                                 float scale, int S, int64_t tps, float *qa, float *part, uint32_t *err,
                                 MergeScratch ms, void *o, int out_fp32, void *const *prof, cudaStream_t st) {
  absorb_query_kernel<<<dim3(n_q, (unsigned)B), 256, 0, st>>>(q, W_kv, n_q, n_kv, d_h, G, scale * kLog2e, qa, err,
                                                              ms);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  size_t smem = absorbed_simt_smem(n_q, G);
  e = ensure_smem_limit((const void *)absorbed_split_simt, smem);
  if (e != cudaSuccess) return e;
  record_prof_event(prof[0], st);
  absorbed_split_simt<<<dim3(S, (unsigned)B), 256, smem, st>>>(qa, codes, bstride, T, seq_lens, n_new, G, bits,
                                                                n_q, tps, part, err);
  e = cudaGetLastError();
  record_prof_event(prof[1], st);
  if (e != cudaSuccess) return e;
  return merge_absorbed_launch(part, S, B, n_q, n_kv, d_h, G, W_kv, o, out_fp32, ms, st, 0);
}

cudaError_t launch_expand_simt(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int n_new,
                               int64_t T, const int32_t *seq_lens, int n_q, int n_kv, int d_h, int G, int bits,
                               const uint16_t *W_kv,
                               float scale, int S, int64_t tps, int rope_knorm, float rope_base,
                               const uint16_t *gain, float eps, float *part, uint32_t *err, void *o, int out_fp32,
                               void *const *prof, cudaStream_t st) {
  clear_err_kernel<<<1, 1, 0, st>>>(err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  size_t smem = expand_simt_smem(G);
  e = ensure_smem_limit((const void *)expand_split_simt, smem);
  if (e != cudaSuccess) return e;
  record_prof_event(prof[0], st);
  expand_split_simt<<<dim3(S, (unsigned)B, n_kv), FSQ_HEAD_DIM, smem, st>>>(
      q, codes, bstride, T, seq_lens, n_new, G, bits, n_q, n_kv, W_kv, scale * kLog2e, tps, rope_knorm, rope_base,
      gain, eps, part, err);
  e = cudaGetLastError();
  record_prof_event(prof[1], st);
  if (e != cudaSuccess) return e;
  merge_expand_kernel<<<dim3(n_q, (unsigned)B), d_h, 0, st>>>(part, S, n_q, d_h, o, out_fp32);
  return cudaGetLastError();
}

}  // namespace fsq
