// Split merge and value decode of the absorbed form.
//
// Every split s of a batch row leaves, per query head h, its running max m_s
// (log2 domain), its weight sum l_s and its pooled latent acc_s[g] =
// sum_t 2^(x_t - m_s) z_t[g].  The merge forms ([S] eq. (6); slide deck frame
// "The kernel reads codes and never writes reconstructed K/V": merge partials
// and apply W_v once)
//   m = max_s m_s,  L = sum_s 2^(m_s - m) l_s,  abar_h = sum_s 2^(m_s - m) acc_s / L
//   o_h = W_v^(j) abar_h
// for the GRP query heads of kv head j, per batch row b.  Each thread owns a
// pair of coordinates of one head and folds the splits into a running
// (max, sum, pair) by log-sum-exp, so all of its loads - the (m_s, l_s)
// records and the accumulator pairs - are independent of each other and are
// issued sixteen splits at a time.
//
// When a CTA has more threads than pairs, its threads also split the range of
// splits (interleaved) and their running states are combined, by the same
// log-sum-exp, in shared memory.
//
// Direct mode (few splits): one CTA per (j, b) does all of it, with W_v^(j)
// staged in shared memory (cp.async) before the wait for the split kernel.
// Sliced mode (long contexts, many splits): the CTAs of a (j, b) pair take
// 32-coordinate slices of G over all splits, write their slices of abar to a
// slab in the workspace, and the last to finish (an arrival count, zeroed by
// the query prologue of the same call) applies W_v.
//
// Byte fold: with 256-level codes the split kernel pools each 8-bit code as
// its two nibbles (coordinates 2i and 2i+1 of G = 2 x the latent width, levels
// lo - 8 and hi - 8).  The code's level is (lo - 8) + 16 (hi - 8) + 8, and the
// merged weights sum to one, so abar_i = abar'_2i + 16 abar'_2i+1 + 8: the
// pair a thread merges is exactly one byte, folded as it is written.  W_v^(j)
// then has G/2 columns.
#include <algorithm>

#include "common.cuh"

namespace fsq {
namespace {

constexpr int kMT = 512;                    // threads per CTA
constexpr int kParts = kMT / FSQ_HEAD_DIM;  // W_v pass: threads per output row d
constexpr int kGsl = 32;                    // G coordinates per slice (sliced mode)
constexpr int kBatch = 16;                  // splits whose loads a thread issues at once
constexpr int kMaxSub = 16;                 // threads sharing one pair (split ranges)
constexpr size_t kDirectBytes = 64 * 1024;  // partial bytes of a (j, b) pair that one CTA reads
static_assert(kMT % FSQ_HEAD_DIM == 0, "the W_v pass maps (part, d) to threads");

// Padded G: a multiple of 8 * kParts, so that each part of the W_v pass
// covers whole 8-element pieces.
__host__ __device__ inline int g_pad(int G) { return (G + 8 * kParts - 1) / (8 * kParts) * (8 * kParts); }
__host__ __device__ inline int w_stride(int G) { return g_pad(G) + 8; }  // bf16: 16-byte rows, odd x 16 B

struct MergeSmem {
  size_t off_abar, off_scr, off_lse, bytes;
};

inline MergeSmem merge_smem(int G, int grp) {
  MergeSmem m;
  size_t off = sizeof(uint16_t) * (size_t)FSQ_HEAD_DIM * w_stride(G);  // W_v^(j), bf16
  m.off_abar = off;
  off += sizeof(float) * (size_t)grp * g_pad(G);
  m.off_scr = off;  // partial outputs of parts 1.. of the W_v pass
  off += sizeof(float) * (size_t)(kParts - 1) * grp * FSQ_HEAD_DIM;
  off = align_up(off, 16);
  m.off_lse = off;  // running states of the threads of a pair: [sub][pair] x (m, l, a.x, a.y)
  off += sizeof(float4) * (size_t)kMT;
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

// o_h[d] = W_v[d, :] . abar_h for the GRP heads; thread (part, d) covers a
// kParts-th of the coordinates for every head, so each W_v value read serves
// GRP heads (the abar reads are broadcasts)
template <int GRP>
__device__ __forceinline__ void apply_wv(const uint16_t *wv, const float *abar, float *scr, int G, int64_t obase,
                                         void *o, int out_fp32) {
  constexpr int D = FSQ_HEAD_DIM;
  const int GP = g_pad(G), WS = w_stride(G);
  const int d = threadIdx.x % D, part = threadIdx.x / D;
  const int gq = GP / kParts;  // a multiple of 8
  const uint16_t *wr = wv + d * WS + part * gq;
  // even and odd coordinates accumulate in the two lanes of packed fp32x2 FMAs
  float2 acc2[GRP];
#pragma unroll
  for (int h = 0; h < GRP; ++h) acc2[h] = make_float2(0.f, 0.f);
  for (int g8 = 0; g8 < gq; g8 += 8) {
    const uint4 wq = *reinterpret_cast<const uint4 *>(wr + g8);
    const uint32_t wp[4] = {wq.x, wq.y, wq.z, wq.w};
    float2 wf[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) wf[e] = make_float2(__uint_as_float(wp[e] << 16), __uint_as_float(wp[e] & 0xFFFF0000u));
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      const float4 lo = *reinterpret_cast<const float4 *>(abar + h * GP + part * gq + g8);
      const float4 hi = *reinterpret_cast<const float4 *>(abar + h * GP + part * gq + g8 + 4);
      acc2[h] = __ffma2_rn(wf[0], make_float2(lo.x, lo.y), acc2[h]);
      acc2[h] = __ffma2_rn(wf[1], make_float2(lo.z, lo.w), acc2[h]);
      acc2[h] = __ffma2_rn(wf[2], make_float2(hi.x, hi.y), acc2[h]);
      acc2[h] = __ffma2_rn(wf[3], make_float2(hi.z, hi.w), acc2[h]);
    }
  }
  float acc[GRP];
#pragma unroll
  for (int h = 0; h < GRP; ++h) acc[h] = acc2[h].x + acc2[h].y;
  if (part > 0) {
#pragma unroll
    for (int h = 0; h < GRP; ++h) scr[((part - 1) * GRP + h) * D + d] = acc[h];
  }
  __syncthreads();
  if (part == 0) {
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      float v = acc[h];
#pragma unroll
      for (int p = 1; p < kParts; ++p) v += scr[((p - 1) * GRP + h) * D + d];
      const int64_t oi = obase + (int64_t)h * D + d;
      if (out_fp32) reinterpret_cast<float *>(o)[oi] = v;
      else reinterpret_cast<uint16_t *>(o)[oi] = f32_to_bf16_rn(v);
    }
  }
}

// Running log-sum-exp state of one coordinate pair: max m, weight sum l, pair a.
struct Lse {
  float m, l;
  float2 a;
};

// 2^x on the special-function unit (x <= 0 here; -inf gives 0)
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Fold splits s0, s0 + ds, ... below S of one head's records (rec: the
// head's record in split 0; sstride: floats between splits; gi: the pair's
// offset) into st.  A batch of up to kBatch splits is folded at once: its
// maximum first, then one exponential per split, so the weighted sums of the
// batch do not wait on one another.
template <int NB>
__device__ __forceinline__ void fold_batch(Lse &st, const float *__restrict__ rec, int64_t sstride, int gi, int s,
                                           int ds, int S) {
  float2 ml[NB], av[NB];
#pragma unroll
  for (int u = 0; u < NB; ++u) {
    const bool in = s + u * ds < S;
    const float *r = rec + (int64_t)(s + u * ds) * sstride;
    ml[u] = in ? *reinterpret_cast<const float2 *>(r) : make_float2(-INFINITY, 0.f);
    av[u] = in ? *reinterpret_cast<const float2 *>(r + 2 + gi) : make_float2(0.f, 0.f);
  }
  float mn = st.m;
#pragma unroll
  for (int u = 0; u < NB; ++u) mn = fmaxf(mn, ml[u].x);
  if (mn == -INFINITY) return;  // nothing folded yet and only empty splits
  const float co = ex2_fast(st.m - mn);
  float l = st.l * co, ax = st.a.x * co, ay = st.a.y * co;
#pragma unroll
  for (int u = 0; u < NB; ++u) {
    const float cs = ex2_fast(ml[u].x - mn);  // 0 for an empty slot
    l = fmaf(ml[u].y, cs, l);
    ax = fmaf(av[u].x, cs, ax);
    ay = fmaf(av[u].y, cs, ay);
  }
  st.m = mn;
  st.l = l;
  st.a = make_float2(ax, ay);
}
__device__ __forceinline__ void fold_splits(Lse &st, const float *__restrict__ rec, int64_t sstride, int gi, int s0,
                                            int ds, int S) {
  const int n = (S - s0 + ds - 1) / ds;  // splits this thread folds
  if (n <= 4) {
    fold_batch<4>(st, rec, sstride, gi, s0, ds, S);
  } else if (n <= 8) {
    fold_batch<8>(st, rec, sstride, gi, s0, ds, S);
  } else {
    for (int s = s0; s < S; s += kBatch * ds) fold_batch<kBatch>(st, rec, sstride, gi, s, ds, S);
  }
}

__device__ __forceinline__ void fold_state(Lse &st, const float4 &o) {
  const float mn = fmaxf(st.m, o.x);
  if (mn == -INFINITY) return;
  const float co = ex2_fast(st.m - mn), cs = ex2_fast(o.x - mn);
  st.l = fmaf(st.l, co, o.y * cs);
  st.a.x = fmaf(st.a.x, co, o.z * cs);
  st.a.y = fmaf(st.a.y, co, o.w * cs);
  st.m = mn;
}

template <int GRP>
__global__ void __launch_bounds__(kMT) merge_absorbed_grouped(const float *__restrict__ part, int S, int n_q,
                                                              int n_kv, int G, const uint16_t *__restrict__ W_kv,
                                                              void *o, int out_fp32, int ngq,
                                                              float *__restrict__ slab, uint32_t *__restrict__ cnt,
                                                              MergeSmem L, int fold) {
  constexpr int D = FSQ_HEAD_DIM;
  extern __shared__ __align__(16) unsigned char msm[];
  uint16_t *wv = reinterpret_cast<uint16_t *>(msm);           // [D][WS] bf16
  float *abar = reinterpret_cast<float *>(msm + L.off_abar);  // [GRP][GP]
  float *scr = reinterpret_cast<float *>(msm + L.off_scr);
  __shared__ uint32_t last;
  const int gq = blockIdx.x;
  const int j = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const bool direct = ngq == 1;
  const int GW = fold ? G / 2 : G;  // latent width: columns of W_v^(j), entries of abar
  const int GP = g_pad(GW);
  const uint16_t *wsrc = W_kv + (int64_t)(n_kv + j) * D * GW;
  if (direct) stage_wv(wv, wsrc, GW);  // W_v is not written by the split kernel
  // the partials come from the split kernel; no early trigger: whatever
  // follows the call starts once o is complete
  pdl_wait();

  const int64_t hstride = 2 + (int64_t)G;          // floats per (split, head) record
  const int64_t sstride = (int64_t)n_q * hstride;  // floats per split
  const float *pbase = part + ((int64_t)b * S * n_q + (int64_t)j * GRP) * hstride;
  // sliced mode: slab[b][j][h][GP] holds abar; CTA gq writes coordinates gq*32 ..
  float *sl = slab + ((int64_t)b * n_kv + j) * GRP * GP;
  const int gc0 = direct ? 0 : gq * kGsl, gcn = direct ? G : min(kGsl, G - gc0);
  const int npair = gcn / 2;  // G is even, so are gc0 and gcn
  const int items = GRP * npair;
  const int nsub = items >= kMT ? 1 : min(kMaxSub, kMT / items);  // threads per pair
  float4 *lse = reinterpret_cast<float4 *>(msm + L.off_lse);       // [nsub][items]
  for (int t0 = 0; t0 < items * nsub; t0 += kMT) {
    const int t = t0 + tid;
    const int it = t % items, sub = t / items;
    const int h = it / npair, gi = gc0 + 2 * (it % npair);
    Lse st{-INFINITY, 0.f, make_float2(0.f, 0.f)};
    if (t < items * nsub) fold_splits(st, pbase + (int64_t)h * hstride, sstride, gi, sub, nsub, S);
    if (nsub > 1) {  // combine the sub-ranges of a pair (all of them lie in this round)
      lse[tid] = make_float4(st.m, st.l, st.a.x, st.a.y);
      __syncthreads();
      if (sub == 0 && t < items)
        for (int k = 1; k < nsub; ++k) fold_state(st, lse[k * items + it]);
    }
    if (sub == 0 && t < items) {
      const float inv = 1.f / st.l;
      const float2 v = make_float2(st.a.x * inv, st.a.y * inv);
      if (fold) {
        const float f = fmaf(16.f, v.y, v.x) + 8.f;  // nibbles lo, hi of byte gi / 2
        (direct ? abar : sl)[h * GP + gi / 2] = f;
      } else if (direct) {
        *reinterpret_cast<float2 *>(abar + h * GP + gi) = v;
      } else {
        *reinterpret_cast<float2 *>(sl + h * GP + gi) = v;
      }
    }
  }
  if (direct) {
    for (int i = tid; i < GRP * (GP - GW); i += kMT) abar[(i / (GP - GW)) * GP + GW + i % (GP - GW)] = 0.f;
  } else {
    // the last CTA of the (j, b) pair gathers abar and applies W_v
    __threadfence();
    __syncthreads();
    if (tid == 0) last = atomicAdd(cnt + (int64_t)b * n_kv + j, 1u) == (uint32_t)(ngq - 1) ? 1u : 0u;
    __syncthreads();
    if (!last) return;
    __threadfence();
    stage_wv(wv, wsrc, GW);
    for (int i = tid; i < GRP * GP; i += kMT) abar[i] = i % GP < GW ? __ldcg(sl + i) : 0.f;
  }
  cp_async_wait_all();
  __syncthreads();
  apply_wv<GRP>(wv, abar, scr, GW, ((int64_t)b * n_q + (int64_t)j * GRP) * D, o, out_fp32);
}

template <int GRP>
cudaError_t merge_launch(const float *part, int S, int64_t B, int n_q, int n_kv, int G, const uint16_t *W_kv, void *o,
                         int out_fp32, const MergePlan &mp, float *slab, uint32_t *cnt, cudaStream_t st, int fold) {
  const MergeSmem L = merge_smem(fold ? G / 2 : G, GRP);
  auto kern = merge_absorbed_grouped<GRP>;
  cudaError_t e = ensure_smem_limit((const void *)kern, L.bytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3((unsigned)mp.ngq, (unsigned)n_kv, (unsigned)B), dim3(kMT), L.bytes, st, part, S, n_q,
                    n_kv, G, W_kv, o, out_fp32, mp.ngq, slab, cnt, L, fold);
}

}  // namespace

bool merge_grouped_supported(int n_q, int n_kv) {
  const int grp = n_q / n_kv;
  return grp == 1 || grp == 2 || grp == 4 || grp == 8 || grp == 16;
}

// Direct mode when one CTA's share of partials is small; else G slices of 32.
MergePlan merge_plan(int S, int64_t B, int n_q, int n_kv, int G) {
  MergePlan mp;
  const int grp = n_q / n_kv;
  const size_t bytes = sizeof(float) * (size_t)S * grp * (2 + G);
  if (merge_grouped_supported(n_q, n_kv) && bytes > kDirectBytes) {
    mp.ngq = (G + kGsl - 1) / kGsl;
    mp.slab_bytes = sizeof(float) * (size_t)B * n_q * g_pad(G);
    mp.cnt_bytes = sizeof(uint32_t) * (size_t)B * n_kv;
  }
  return mp;
}

// G: coordinates of the partials (with fold, two nibbles per 8-bit code).
cudaError_t merge_grouped_launch(const float *part, int S, int64_t B, int n_q, int n_kv, int G,
                                 const uint16_t *W_kv, void *o, int out_fp32, float *slab, uint32_t *cnt,
                                 cudaStream_t st, int fold) {
  if (B > 65535 || n_kv > 65535 || G > 2 * FSQ_MAX_G || (!fold && G > FSQ_MAX_G)) return cudaErrorInvalidValue;
  const MergePlan mp = merge_plan(S, B, n_q, n_kv, G);
  if (mp.ngq > 1 && (!slab || !cnt)) return cudaErrorInvalidValue;
  switch (n_q / n_kv) {
    case 1: return merge_launch<1>(part, S, B, n_q, n_kv, G, W_kv, o, out_fp32, mp, slab, cnt, st, fold);
    case 2: return merge_launch<2>(part, S, B, n_q, n_kv, G, W_kv, o, out_fp32, mp, slab, cnt, st, fold);
    case 4: return merge_launch<4>(part, S, B, n_q, n_kv, G, W_kv, o, out_fp32, mp, slab, cnt, st, fold);
    case 8: return merge_launch<8>(part, S, B, n_q, n_kv, G, W_kv, o, out_fp32, mp, slab, cnt, st, fold);
    case 16: return merge_launch<16>(part, S, B, n_q, n_kv, G, W_kv, o, out_fp32, mp, slab, cnt, st, fold);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fsq
