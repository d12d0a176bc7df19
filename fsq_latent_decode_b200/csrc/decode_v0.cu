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
                                    uint32_t *err) {
  __shared__ float qs[FSQ_HEAD_DIM];
  const int h = blockIdx.x, b = blockIdx.y;
  const int j = h / (n_q / n_kv);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *err = 0u;
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
                                                           int64_t T, int G, int n_q, int64_t tps,
                                                           float *__restrict__ part) {
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
  const int64_t t1 = min(T, t0 + tps);
  const int half = G / 2;
  const uint8_t *cb = codes + (int64_t)b * bstride;

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
    for (int i = tid; i < kNT * half; i += nth) {
      int t = i / half, by = i % half;
      float lo = 0.f, hi = 0.f;
      if (t < nv) {
        uint32_t v = cb[(tt + t) * half + by];
        lo = (float)(int)(v & 15u) - 8.f;
        hi = (float)(int)(v >> 4) - 8.f;
      }
      cs[t * (G + 1) + 2 * by] = lo;
      cs[t * (G + 1) + 2 * by + 1] = hi;
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
                                                         int64_t T, int G, int n_q, int n_kv,
                                                         const uint16_t *__restrict__ W_kv, float c, int64_t tps,
                                                         int rope_knorm, float rope_base,
                                                         const uint16_t *__restrict__ gain, float eps,
                                                         float *__restrict__ part) {
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
  const int64_t t0 = (int64_t)s * tps, t1 = min(T, t0 + tps);
  const int half = G / 2;
  const uint8_t *cb = codes + (int64_t)b * bstride;

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
    for (int i = d; i < kNTx * half; i += D) {
      int t = i / half, by = i % half;
      float lo = 0.f, hi = 0.f;
      if (t < nv) {
        uint32_t v = cb[(tt + t) * half + by];
        lo = (float)(int)(v & 15u) - 8.f;
        hi = (float)(int)(v >> 4) - 8.f;
      }
      cs[t * G + 2 * by] = lo;
      cs[t * G + 2 * by + 1] = hi;
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

// Split merge + W_v for one GQA group, one CTA per (kv head j, batch row b).
// The group's heads share W_v^(j): it is staged once in shared memory by
// cp.async, issued first so the copy overlaps the partial reads, in rows of
// WS = 8 x odd elements so that a warp's 16-byte reads of 32 consecutive rows
// fall on distinct bank groups.  Then abar_h = sum_s w_s acc_s / l over the
// splits, and one thread per output (d, heads) forms o_h[d] = W_v[d] . abar_h
// with 16-byte shared reads (abar is a broadcast).
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s), "l"(gmem) : "memory");
}

struct MergeShape {
  int GP;   // G rounded up to 8 (abar row, zero tail)
  int WS;   // W_v row stride in shared memory: 8 x odd >= GP
  size_t off_abar, off_w, bytes;
};

inline MergeShape merge_shape(int G, int d_h, int grp, int S) {
  MergeShape m;
  m.GP = (G + 7) / 8 * 8;
  m.WS = m.GP % 16 ? m.GP : m.GP + 8;
  m.off_abar = sizeof(uint16_t) * (size_t)d_h * m.WS;
  m.off_w = m.off_abar + sizeof(float) * (size_t)grp * m.GP;
  m.bytes = m.off_w + sizeof(float) * (size_t)grp * S;
  return m;
}

template <int GRP>
struct MergeThreads {
  static constexpr int HT = GRP < 4 ? GRP : 4;   // head slices, one thread per (d, slice)
  static constexpr int H = GRP / HT;             // heads per thread
  static constexpr int NT = FSQ_HEAD_DIM * HT;
};

template <int GRP>
__global__ void __launch_bounds__(MergeThreads<GRP>::NT)
    merge_absorbed_group_kernel(const float *__restrict__ part, int S, int n_q, int n_kv, int G,
                                const uint16_t *__restrict__ W_kv, void *o, int out_fp32, MergeShape ms) {
  constexpr int D = FSQ_HEAD_DIM;
  constexpr int H = MergeThreads<GRP>::H;
  extern __shared__ __align__(16) unsigned char msm[];
  uint16_t *wv = reinterpret_cast<uint16_t *>(msm);                     // [D][WS]
  float *abar = reinterpret_cast<float *>(msm + ms.off_abar);           // [GRP][GP]
  float *wts = reinterpret_cast<float *>(msm + ms.off_w);               // [GRP][S]
  const int j = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int GP = ms.GP, WS = ms.WS;
  {  // W_v^(j): D contiguous rows of G bf16 starting at row (n_kv + j) D
    const uint16_t *src = W_kv + (int64_t)(n_kv + j) * D * G;
    if (G % 8 == 0) {
      const int cpr = G / 8;
      for (int i = threadIdx.x; i < D * cpr; i += blockDim.x) {
        const int r = i / cpr, c8 = i % cpr;
        cp_async16(wv + r * WS + 8 * c8, src + (int64_t)r * G + 8 * c8);
      }
    } else {
      const int cpr = G / 2;
      for (int i = threadIdx.x; i < D * cpr; i += blockDim.x) {
        const int r = i / cpr, c2 = i % cpr;
        cp_async4(wv + r * WS + 2 * c2, src + (int64_t)r * G + 2 * c2);
      }
      for (int i = threadIdx.x; i < D * (GP - G); i += blockDim.x) wv[(i / (GP - G)) * WS + G + i % (GP - G)] = 0;
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  pdl_wait();  // the partials come from the split kernel
  pdl_trigger();
  const int64_t sstride = (int64_t)n_q * (2 + G);
  const float *pbase = part + ((int64_t)b * S * n_q + j * GRP) * (2 + G);
  if (warp < GRP) {  // split weights for head `warp`, 1/l folded in
    const float *pb = pbase + (int64_t)warp * (2 + G);
    float m = -INFINITY;
    for (int s = lane; s < S; s += 32) m = fmaxf(m, pb[s * sstride]);
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.f;
    for (int s = lane; s < S; s += 32) {
      const float w = exp2f(pb[s * sstride] - m);
      wts[warp * S + s] = w;
      l = fmaf(w, pb[s * sstride + 1], l);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    const float inv = 1.f / l;
    __syncwarp();
    for (int s = lane; s < S; s += 32) wts[warp * S + s] *= inv;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < GRP * GP; idx += blockDim.x) {
    const int hh = idx / GP, g = idx % GP;
    float a0 = 0.f, a1 = 0.f;
    if (g < G) {
      const float *pb = pbase + (int64_t)hh * (2 + G) + 2 + g;
      const float *ws = wts + hh * S;
      int s = 0;
      for (; s + 8 <= S; s += 8) {  // eight independent loads in flight
        float pv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) pv[u] = pb[(s + u) * sstride];
#pragma unroll
        for (int u = 0; u < 8; u += 2) {
          a0 = fmaf(ws[s + u], pv[u], a0);
          a1 = fmaf(ws[s + u + 1], pv[u + 1], a1);
        }
      }
      for (; s < S; ++s) a0 = fmaf(ws[s], pb[s * sstride], a0);
    }
    abar[idx] = a0 + a1;
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  const int d = threadIdx.x % D, h0 = (threadIdx.x / D) * H;
  const uint16_t *wr = wv + d * WS;
  float acc[H];
#pragma unroll
  for (int i = 0; i < H; ++i) acc[i] = 0.f;
#pragma unroll 2
  for (int g0 = 0; g0 < GP; g0 += 8) {
    const uint4 wq = *reinterpret_cast<const uint4 *>(wr + g0);
    const uint32_t wp[4] = {wq.x, wq.y, wq.z, wq.w};
    float wf[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      wf[2 * i] = __uint_as_float(wp[i] << 16);
      wf[2 * i + 1] = __uint_as_float(wp[i] & 0xFFFF0000u);
    }
#pragma unroll
    for (int i = 0; i < H; ++i) {
      const float4 lo = *reinterpret_cast<const float4 *>(abar + (h0 + i) * GP + g0);
      const float4 hi = *reinterpret_cast<const float4 *>(abar + (h0 + i) * GP + g0 + 4);
      acc[i] = fmaf(wf[0], lo.x, fmaf(wf[1], lo.y, fmaf(wf[2], lo.z, fmaf(wf[3], lo.w, acc[i]))));
      acc[i] = fmaf(wf[4], hi.x, fmaf(wf[5], hi.y, fmaf(wf[6], hi.z, fmaf(wf[7], hi.w, acc[i]))));
    }
  }
#pragma unroll
  for (int i = 0; i < H; ++i) {
    const int64_t oi = ((int64_t)b * n_q + j * GRP + h0 + i) * D + d;
    if (out_fp32) reinterpret_cast<float *>(o)[oi] = acc[i];
    else reinterpret_cast<uint16_t *>(o)[oi] = f32_to_bf16_rn(acc[i]);
  }
}

template <int GRP>
cudaError_t merge_group_launch(const float *part, int S, int64_t B, int n_q, int n_kv, int d_h, int G,
                               const uint16_t *W_kv, void *o, int out_fp32, cudaStream_t st) {
  const MergeShape ms = merge_shape(G, d_h, GRP, S);
  cudaError_t e = ensure_smem_limit((const void *)merge_absorbed_group_kernel<GRP>, ms.bytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(merge_absorbed_group_kernel<GRP>, dim3(n_kv, (unsigned)B), dim3(MergeThreads<GRP>::NT), ms.bytes,
                    st, part, S, n_q, n_kv, G, W_kv, o, out_fp32, ms);
}

}  // namespace

cudaError_t merge_absorbed_launch(const float *part, int S, int64_t B, int n_q, int n_kv, int d_h, int G,
                                  const uint16_t *W_kv, void *o, int out_fp32, cudaStream_t st) {
  switch (n_q / n_kv) {
    case 1: return merge_group_launch<1>(part, S, B, n_q, n_kv, d_h, G, W_kv, o, out_fp32, st);
    case 2: return merge_group_launch<2>(part, S, B, n_q, n_kv, d_h, G, W_kv, o, out_fp32, st);
    case 4: return merge_group_launch<4>(part, S, B, n_q, n_kv, d_h, G, W_kv, o, out_fp32, st);
    case 8: return merge_group_launch<8>(part, S, B, n_q, n_kv, d_h, G, W_kv, o, out_fp32, st);
    case 16: return merge_group_launch<16>(part, S, B, n_q, n_kv, d_h, G, W_kv, o, out_fp32, st);
    default: break;
  }
  merge_absorbed_kernel<<<dim3(n_q, (unsigned)B), 256, 0, st>>>(part, S, n_q, n_kv, d_h, G, W_kv, o, out_fp32);
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

cudaError_t launch_absorbed_simt(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int64_t T,
                                 int n_q, int n_kv, int d_h, int G, const uint16_t *W_kv, float scale,
                                 int S, int64_t tps, float *qa, float *part, uint32_t *err, void *o,
                                 int out_fp32, void *const *prof, cudaStream_t st) {
  absorb_query_kernel<<<dim3(n_q, (unsigned)B), 256, 0, st>>>(q, W_kv, n_q, n_kv, d_h, G, scale * kLog2e, qa, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  size_t smem = absorbed_simt_smem(n_q, G);
  e = ensure_smem_limit((const void *)absorbed_split_simt, smem);
  if (e != cudaSuccess) return e;
  record_prof_event(prof[0], st);
  absorbed_split_simt<<<dim3(S, (unsigned)B), 256, smem, st>>>(qa, codes, bstride, T, G, n_q, tps, part);
  e = cudaGetLastError();
  record_prof_event(prof[1], st);
  if (e != cudaSuccess) return e;
  return merge_absorbed_launch(part, S, B, n_q, n_kv, d_h, G, W_kv, o, out_fp32, st);
}

cudaError_t launch_expand_simt(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int64_t T,
                               int n_q, int n_kv, int d_h, int G, const uint16_t *W_kv, float scale, int S,
                               int64_t tps, int rope_knorm, float rope_base, const uint16_t *gain, float eps,
                               float *part, uint32_t *err, void *o, int out_fp32, void *const *prof,
                               cudaStream_t st) {
  clear_err_kernel<<<1, 1, 0, st>>>(err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  size_t smem = expand_simt_smem(G);
  e = ensure_smem_limit((const void *)expand_split_simt, smem);
  if (e != cudaSuccess) return e;
  record_prof_event(prof[0], st);
  expand_split_simt<<<dim3(S, (unsigned)B, n_kv), FSQ_HEAD_DIM, smem, st>>>(
      q, codes, bstride, T, G, n_q, n_kv, W_kv, scale * kLog2e, tps, rope_knorm, rope_base, gain, eps, part);
  e = cudaGetLastError();
  record_prof_event(prof[1], st);
  if (e != cudaSuccess) return e;
  merge_expand_kernel<<<dim3(n_q, (unsigned)B), d_h, 0, st>>>(part, S, n_q, d_h, o, out_fp32);
  return cudaGetLastError();
}

}  // namespace fsq
