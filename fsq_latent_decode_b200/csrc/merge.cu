// Split merge and value decode of the absorbed form.
//
// Every split s of a batch row leaves, per query head h, its running max m_s
// (log2 domain), its weight sum l_s and its pooled latent acc_s[g] =
// sum_t 2^(x_t - m_s) z_t[g].  The merge forms ([S] eq. (6); slide deck frame
// "The kernel reads codes and never writes reconstructed K/V": merge partials
// and apply W_v once)
//   m = max_s m_s,  w_s = 2^(m_s - m) / sum_s' 2^(m_s' - m) l_s'
//   abar_h[g] = sum_s w_s acc_s[g]
//   o_h = W_v^(j) abar_h
// for the GRP query heads of kv head j, per batch row b.
//
// Direct mode (few splits): one CTA per (j, b) does all of it, with W_v^(j)
// staged in shared memory before the wait for the split kernel.  Sliced mode
// (long contexts, many splits): the CTAs of a (j, b) pair cut the G
// coordinates into 32-wide slices and the splits into chunks; each writes its
// share of abar to a slab in the workspace, and the last of them to finish
// (an atomic count, zeroed by the query prologue of the same call) adds the
// shares and applies W_v.
#include <algorithm>

#include "common.cuh"

namespace fsq {

namespace {

constexpr int kMT = 256;           // threads per CTA: two per output row d of W_v
constexpr int kGsl = 32;           // G coordinates per slice (sliced mode)
constexpr int kSplitsPerCta = 32;  // splits per chunk (sliced mode)
constexpr size_t kDirectBytes = 48 * 1024;  // partial bytes of a (j, b) pair that one CTA reads
static_assert(kMT == 2 * FSQ_HEAD_DIM, "the W_v pass maps (half, d) to threads");

__host__ __device__ inline int g_pad(int G) { return (G + 31) / 32 * 32; }
__host__ __device__ inline int w_stride(int G) { return g_pad(G) + 8; }  // bf16: 16-byte rows, odd x 16 B

struct MergeSmem {
  size_t off_abar, off_wts, off_scr, bytes;
};

inline MergeSmem merge_smem(int G, int grp, int S) {
  MergeSmem m;
  size_t off = sizeof(uint16_t) * (size_t)FSQ_HEAD_DIM * w_stride(G);  // W_v^(j), bf16
  m.off_abar = off;
  off += sizeof(float) * (size_t)grp * g_pad(G);
  m.off_wts = off;
  off += sizeof(float) * (size_t)grp * S;
  m.off_scr = off;  // l_s scratch, then the halves of the W_v pass
  off += sizeof(float) * std::max((size_t)grp * S, (size_t)grp * FSQ_HEAD_DIM);
  m.bytes = align_up(off, 16);
  return m;
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// W_v^(j) (D rows of G bf16) -> shared memory, rows padded to w_stride, zero
// tail; asynchronous copies, all in flight at once (cp_async_wait_all and a
// barrier before use)
__device__ __forceinline__ void stage_wv(uint16_t *wv, const uint16_t *__restrict__ src, int G) {
  constexpr int D = FSQ_HEAD_DIM;
  const int WS = w_stride(G), GP = g_pad(G);
  if (G % 8 == 0) {
    const int cpr = G / 8;
    for (int i = threadIdx.x; i < D * cpr; i += kMT) {
      const int r = i / cpr, c = i % cpr;
      cp_async16(wv + r * WS + 8 * c, src + (int64_t)r * G + 8 * c);
    }
  } else {
    const int cpr = G / 2;
    for (int i = threadIdx.x; i < D * cpr; i += kMT) {
      const int r = i / cpr, c = i % cpr;
      cp_async4(wv + r * WS + 2 * c, src + (int64_t)r * G + 2 * c);
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int i = threadIdx.x; i < D * (GP - G); i += kMT) wv[(i / (GP - G)) * WS + G + i % (GP - G)] = 0;
}

// o_h[d] = W_v[d, :] . abar_h for the GRP heads; thread (half, d) covers half
// of the coordinates for every head, so each W_v value read serves GRP heads
template <int GRP>
__device__ __forceinline__ void apply_wv(const uint16_t *wv, const float *abar, float *scr, int G, int64_t obase,
                                         void *o, int out_fp32) {
  constexpr int D = FSQ_HEAD_DIM;
  const int GP = g_pad(G), WS = w_stride(G);
  const int d = threadIdx.x % D, half = threadIdx.x / D;
  const int gh = GP / 2;  // a multiple of 16
  const uint16_t *wr = wv + d * WS + half * gh;
  float acc[GRP];
#pragma unroll
  for (int h = 0; h < GRP; ++h) acc[h] = 0.f;
  for (int g8 = 0; g8 < gh; g8 += 8) {
    const uint4 wq = *reinterpret_cast<const uint4 *>(wr + g8);
    const uint32_t wp[4] = {wq.x, wq.y, wq.z, wq.w};
    float wf[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      wf[2 * e] = __uint_as_float(wp[e] << 16);
      wf[2 * e + 1] = __uint_as_float(wp[e] & 0xFFFF0000u);
    }
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      const float4 lo = *reinterpret_cast<const float4 *>(abar + h * GP + half * gh + g8);
      const float4 hi = *reinterpret_cast<const float4 *>(abar + h * GP + half * gh + g8 + 4);
      acc[h] = fmaf(wf[0], lo.x, fmaf(wf[1], lo.y, fmaf(wf[2], lo.z, fmaf(wf[3], lo.w, acc[h]))));
      acc[h] = fmaf(wf[4], hi.x, fmaf(wf[5], hi.y, fmaf(wf[6], hi.z, fmaf(wf[7], hi.w, acc[h]))));
    }
  }
  if (half == 1) {
#pragma unroll
    for (int h = 0; h < GRP; ++h) scr[h * D + d] = acc[h];
  }
  __syncthreads();
  if (half == 0) {
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      const float v = acc[h] + scr[h * D + d];
      const int64_t oi = obase + (int64_t)h * D + d;
      if (out_fp32) reinterpret_cast<float *>(o)[oi] = v;
      else reinterpret_cast<uint16_t *>(o)[oi] = f32_to_bf16_rn(v);
    }
  }
}

template <int GRP>
__global__ void __launch_bounds__(kMT) merge_absorbed_grouped(const float *__restrict__ part, int S, int n_q,
                                                              int n_kv, int G, const uint16_t *__restrict__ W_kv,
                                                              void *o, int out_fp32, int ngq, int nsq,
                                                              float *__restrict__ slab, uint32_t *__restrict__ cnt,
                                                              MergeSmem L) {
  constexpr int D = FSQ_HEAD_DIM;
  extern __shared__ __align__(16) unsigned char msm[];
  uint16_t *wv = reinterpret_cast<uint16_t *>(msm);           // [D][WS] bf16
  float *abar = reinterpret_cast<float *>(msm + L.off_abar);  // [GRP][GP]
  float *wts = reinterpret_cast<float *>(msm + L.off_wts);    // [GRP][S]
  float *scr = reinterpret_cast<float *>(msm + L.off_scr);
  __shared__ uint32_t last;
  const int gq = blockIdx.x % ngq, sq = blockIdx.x / ngq;
  const int j = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool direct = ngq * nsq == 1;
  const int GP = g_pad(G);
  const uint16_t *wsrc = W_kv + (int64_t)(n_kv + j) * D * G;
  if (direct) stage_wv(wv, wsrc, G);  // W_v is not written by the split kernel
  // the partials come from the split kernel; no early trigger: whatever
  // follows the call starts once o is complete
  pdl_wait();

  const int64_t hstride = 2 + (int64_t)G;          // floats per (split, head) record
  const int64_t sstride = (int64_t)n_q * hstride;  // floats per split
  const float *pbase = part + ((int64_t)b * S * n_q + (int64_t)j * GRP) * hstride;

  // split weights of each head, 1/l folded in; (m_s, l_s) is one 8-byte
  // load, eight of them in flight per lane
  for (int h = warp; h < GRP; h += kMT / 32) {
    const float *ph = pbase + (int64_t)h * hstride;
    float m = -INFINITY;
    for (int s8 = 0; s8 < S; s8 += 256) {
      float2 ml[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int s = s8 + 32 * u + lane;
        ml[u] = s < S ? *reinterpret_cast<const float2 *>(ph + (int64_t)s * sstride) : make_float2(-INFINITY, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int s = s8 + 32 * u + lane;
        if (s < S) {
          wts[h * S + s] = ml[u].x;
          scr[h * S + s] = ml[u].y;
        }
        m = fmaxf(m, ml[u].x);
      }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.f;
    for (int s = lane; s < S; s += 32) {
      const float w = exp2f(wts[h * S + s] - m);
      wts[h * S + s] = w;
      l = fmaf(w, scr[h * S + s], l);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    const float inv = 1.f / l;
    __syncwarp();
    for (int s = lane; s < S; s += 32) wts[h * S + s] *= inv;
  }
  __syncthreads();

  // this CTA's coordinates and splits; a pair of coordinates per 8-byte load
  // (records start 8-byte aligned), up to eight loads in flight per thread
  const int gc0 = direct ? 0 : gq * kGsl, gcn = direct ? G : min(kGsl, G - gc0);
  const int s0 = direct ? 0 : sq * kSplitsPerCta, s1 = direct ? S : min(S, s0 + kSplitsPerCta);
  const int npair = gcn / 2;  // G is even, so are gc0 and gcn
  for (int t = tid; t < GRP * npair; t += kMT) {
    const int h = t / npair, gi = 2 * (t % npair);
    const float *pg = pbase + (int64_t)h * hstride + 2 + gc0 + gi;
    const float *w = wts + h * S;
    float2 a = make_float2(0.f, 0.f);
    for (int s = s0; s < s1; s += 8) {
      float2 pv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        pv[u] = s + u < s1 ? *reinterpret_cast<const float2 *>(pg + (int64_t)(s + u) * sstride) : make_float2(0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float wu = s + u < s1 ? w[s + u] : 0.f;
        a.x = fmaf(wu, pv[u].x, a.x);
        a.y = fmaf(wu, pv[u].y, a.y);
      }
    }
    if (direct) {
      abar[h * GP + gi] = a.x;
      abar[h * GP + gi + 1] = a.y;
    } else {  // slab[b][j][sq][h][g]
      float *dst = slab + ((((int64_t)b * n_kv + j) * nsq + sq) * GRP + h) * GP + gc0 + gi;
      *reinterpret_cast<float2 *>(dst) = a;
    }
  }
  if (direct) {
    for (int i = tid; i < GRP * (GP - G); i += kMT) abar[(i / (GP - G)) * GP + G + i % (GP - G)] = 0.f;
  } else {
    // the last CTA of the (j, b) pair adds the shares of all chunks
    __threadfence();
    __syncthreads();
    if (tid == 0) last = atomicAdd(cnt + (int64_t)b * n_kv + j, 1u) == (uint32_t)(ngq * nsq - 1) ? 1u : 0u;
    __syncthreads();
    if (!last) return;
    __threadfence();
    stage_wv(wv, wsrc, G);
    const float *sl = slab + ((int64_t)b * n_kv + j) * nsq * GRP * GP;
    for (int i = tid; i < GRP * GP; i += kMT) {
      float a = 0.f;
      if (i % GP < G)
        for (int c0 = 0; c0 < nsq; c0 += 8) {  // eight loads in flight
          float v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] = c0 + u < nsq ? __ldcg(sl + (int64_t)(c0 + u) * GRP * GP + i) : 0.f;
#pragma unroll
          for (int u = 0; u < 8; ++u) a += v[u];
        }
      abar[i] = a;
    }
  }
  cp_async_wait_all();
  __syncthreads();
  apply_wv<GRP>(wv, abar, scr, G, ((int64_t)b * n_q + (int64_t)j * GRP) * D, o, out_fp32);
}

template <int GRP>
cudaError_t merge_launch(const float *part, int S, int64_t B, int n_q, int n_kv, int G, const uint16_t *W_kv, void *o,
                         int out_fp32, const MergePlan &mp, float *slab, uint32_t *cnt, cudaStream_t st) {
  const MergeSmem L = merge_smem(G, GRP, S);
  auto kern = merge_absorbed_grouped<GRP>;
  cudaError_t e = ensure_smem_limit((const void *)kern, L.bytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3((unsigned)(mp.ngq * mp.nsq), (unsigned)n_kv, (unsigned)B), dim3(kMT), L.bytes, st,
                    part, S, n_q, n_kv, G, W_kv, o, out_fp32, mp.ngq, mp.nsq, slab, cnt, L);
}

}  // namespace

bool merge_grouped_supported(int n_q, int n_kv) {
  const int grp = n_q / n_kv;
  return grp == 1 || grp == 2 || grp == 4 || grp == 8 || grp == 16;
}

// Direct mode when one CTA's share of partials is small; else G slices of 32
// and split chunks of kSplitsPerCta.
MergePlan merge_plan(int S, int64_t B, int n_q, int n_kv, int G) {
  MergePlan mp;
  const int grp = n_q / n_kv;
  const size_t bytes = sizeof(float) * (size_t)S * grp * (2 + G);
  if (merge_grouped_supported(n_q, n_kv) && bytes > kDirectBytes) {
    mp.ngq = (G + kGsl - 1) / kGsl;
    mp.nsq = (S + kSplitsPerCta - 1) / kSplitsPerCta;
    mp.slab_bytes = sizeof(float) * (size_t)B * n_q * mp.nsq * g_pad(G);
    mp.cnt_bytes = sizeof(uint32_t) * (size_t)B * n_kv;
  }
  return mp;
}

cudaError_t merge_grouped_launch(const float *part, int S, int64_t B, int n_q, int n_kv, int G,
                                 const uint16_t *W_kv, void *o, int out_fp32, float *slab, uint32_t *cnt,
                                 cudaStream_t st) {
  if (B > 65535 || n_kv > 65535 || G > FSQ_MAX_G) return cudaErrorInvalidValue;
  const MergePlan mp = merge_plan(S, B, n_q, n_kv, G);
  if (mp.ngq * mp.nsq > 1 && (!slab || !cnt)) return cudaErrorInvalidValue;
  switch (n_q / n_kv) {
    case 1: return merge_launch<1>(part, S, B, n_q, n_kv, G, W_kv, o, out_fp32, mp, slab, cnt, st);
    case 2: return merge_launch<2>(part, S, B, n_q, n_kv, G, W_kv, o, out_fp32, mp, slab, cnt, st);
    case 4: return merge_launch<4>(part, S, B, n_q, n_kv, G, W_kv, o, out_fp32, mp, slab, cnt, st);
    case 8: return merge_launch<8>(part, S, B, n_q, n_kv, G, W_kv, o, out_fp32, mp, slab, cnt, st);
    case 16: return merge_launch<16>(part, S, B, n_q, n_kv, G, W_kv, o, out_fp32, mp, slab, cnt, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fsq
