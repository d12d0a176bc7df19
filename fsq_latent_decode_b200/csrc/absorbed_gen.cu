// Decode attention over packed FSQ codes on the tensor cores, absorbed form,
// for any code width (2-, 4- or 8-bit codes: 4, 16 or 256 levels) and any even
// latent width G whose tiles fit in shared memory.
//
// Per 128-token tile of one batch row and token split ([S] Key Design
// Innovation eq. (6); slide deck frame "The kernel reads codes and never
// writes reconstructed K/V": read codes, unpack, tensor cores, online softmax,
// merge partials, apply W_v once):
//   bulk copy of the packed rows into shared memory (two buffers)
//   -> all threads unpack the codes into Z [128 tokens x G] in shared memory:
//      each code n becomes the fp16 subnormal (n - L/2) 2^-24 (its bit pattern
//      n, minus (L/2) 2^-24 by one exact fp16 subtraction per pair), so Z holds
//      the signed levels and the products of both MMAs have either sign (the
//      fp32 sums of a long split do not drift one way), in 8 x 8 blocks (8 tokens x 8 coordinates, 128 bytes).  Read along the
//      coordinates that block is a K-major core matrix of the score MMA's A;
//      read along the tokens it is an MN-major core matrix of the pooling
//      MMA's A (Z^T), so one copy serves both products with no transpose.
//      The unpack also writes each token's row of Z to TMEM (lane = token),
//      the A operand of the score MMA, so that product reads only Q' from
//      shared memory.
//   -> S [128 x 2 NQ] = Z . Q'^T on tcgen05 (kind::f16, fp32 in TMEM), Q' the
//      absorbed query weights as two fp16 terms (hi, lo) per head, stacked
//      along N: the score is 2^24 (S_hi + S_lo), with about 22 significant bits
//      of q'.
//   -> online softmax on the CUDA cores (lazy rescale at 2^8, log2 domain),
//      P [128 x NQ] fp16 into shared memory.
//   -> ACC [G x NQ] += Z^T . P on tcgen05, in blocks of 128 coordinates.
// The epilogue writes the split's (m, l, ACC) partial in latent units, and the
// grouped merge applies W_v.
//
// The steps of a tile run in sequence, all 256 threads taking part (one
// thread issues the MMAs); the next tile's codes are copied meanwhile.  Every
// wait is bounded: a wait that gives up records FSQ_ERR_TIMEOUT, every thread
// leaves the tile loop together (the vote that follows each wait), and the CTA
// lets its issued copies and MMAs finish before it frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc_decode.cuh"
#include "tc_ptx.cuh"

namespace fsq {
namespace tc {
namespace gen {

constexpr int kTile = 128;

// Threads of a CTA (NT) and the softmax's head groups: 128 token rows x HG
// groups of NH heads (NH >= 8: the P stores cover 8 heads).  At n_q = 32 a CTA
// runs 512 threads when one CTA fills an SM (the unpack and the softmax spread
// over twice the warps) and 256 when two fit (their steps then overlap).
template <int NQ, int NT>
struct Shape {
  // CTAs per SM the register budget is set for (__launch_bounds__): two
  // 256-thread CTAs at n_q <= 32 (<= 128 registers per thread)
  static constexpr int MINB = (NT == 256 && NQ <= 32) ? 2 : 1;
  static constexpr int NW = NT / 32;
  static constexpr int HG = NT / 128;
  static constexpr int NH = NQ / HG;
  static_assert(NH >= 8 && NH % 8 == 0, "softmax head groups of whole 8-head blocks");
};
constexpr float kTau = 8.f;                       // rescale when a score exceeds the running max by 2^8
constexpr uint64_t kWaitNs = 1000000000ull;       // 1 s per wait
constexpr uint64_t kDrainNs = 1000000000ull;      // 1 s for in-flight copies and MMAs on the error path
constexpr size_t kSmemMax = 227 * 1024;
constexpr int kMiscBytes = 4096;

// Shared-memory plan of one CTA (host and device agree on it).  The pooling's
// copy of Z holds the unpacked tile in one piece (nch = 1) or, when that does
// not fit, in two chunks of whole 128-coordinate blocks (nch = 2): the first
// nmb0 blocks, then the rest.  The pooling runs on the resident second chunk,
// then on the first chunk unpacked again (the scores read Z from TMEM).
struct Plan {
  int G, Gp, NMB, RB;            // latent width, width padded to 16, 128-coordinate blocks, code bytes per row
  int nq, nch, nmb0;
  size_t off_z, off_q, off_p, off_c, off_misc, total;
  int tmem_cols, off_za;          // TMEM: S [0, 2 nq), ACC [2 nq, 2 nq + NMB nq), Z (score A) from off_za
};
__host__ __device__ inline Plan plan_with(int G, int nq, int bits, int nch) {
  Plan p;
  p.G = G;
  p.Gp = (G + 15) / 16 * 16;
  p.NMB = (G + 127) / 128;
  p.RB = G * bits / 8;
  p.nq = nq;
  p.nch = nch;
  p.nmb0 = nch == 1 ? p.NMB : (p.NMB + 1) / 2;
  const int zc = nch == 1 ? p.Gp : 128 * p.nmb0;  // coordinates Z holds at once
  size_t off = 0;
  p.off_z = off;                                           // Z: zc coordinates x 128 tokens, fp16
  off += (size_t)zc * kTile * 2;
  p.off_q = off;                                           // Q': 2 nq rows x Gp, fp16, K-major blocks
  off += (size_t)p.Gp * 2 * nq * 2;
  p.off_p = off;                                           // P: 128 tokens x nq, fp16, MN-major blocks
  off += (size_t)kTile * nq * 2;
  p.off_c = off;                                           // two code-tile buffers (+16 bytes each)
  off += 2 * (((size_t)kTile * p.RB + 16 + 127) / 128 * 128);
  p.off_misc = off;
  off += kMiscBytes;
  // The last pooling block of a chunk reads 128 coordinates from its start:
  // past Z's end it reads the regions that follow (its rows past G are
  // discarded), which must lie inside the allocation.
  const size_t zread = (size_t)p.nmb0 * 128 * kTile * 2;
  p.total = off > zread ? off : zread;
  p.off_za = 2 * nq + p.NMB * nq;
  const int cols = p.off_za + p.Gp / 2;  // Z as fp16 pairs: Gp / 2 columns
  int c = 32;
  while (c < cols) c *= 2;
  p.tmem_cols = c;
  return p;
}
__host__ __device__ inline Plan plan_of(int G, int nq, int bits) {
  const Plan one = plan_with(G, nq, bits, 1);
  return (one.total <= kSmemMax || one.NMB < 2) ? one : plan_with(G, nq, bits, 2);
}
__host__ __device__ inline size_t code_buf_bytes(const Plan &p) { return ((size_t)kTile * p.RB + 16 + 127) / 128 * 128; }

struct Params {
  const uint8_t *codes;
  int64_t bstride, T, tps;
  int S, n_new, levels;
  const uint8_t *qbuf;     // per grid row: Q' in the score MMA's B layout (Gp x 4 nq bytes)
  float *part;             // [R][S][nq][2 + G]
  uint32_t *err;
  const int32_t *seq_lens;
  uint32_t stall_ns;
};

template <int NQ, int NW>
struct Misc {
  uint64_t full[2], s_mid, s_full, p_mid, p_done, q_full, done, never;
  uint32_t tmem_base;
  uint32_t abort;
  float cneg[NQ];          // -(running max), per head
  float red[NW][NQ];       // per-warp partial maxima / sums
};
static_assert(sizeof(Misc<16, 8>) <= kMiscBytes && sizeof(Misc<32, 16>) <= kMiscBytes &&
                  sizeof(Misc<64, 8>) <= kMiscBytes,
              "Misc block exceeds its reservation");

// Code word -> fp16 bit patterns (value n 2^-24) of its codes, two per 32-bit
// word in coordinate order.  BITS = 8: four codes -> two words (byte permute);
// 4: eight -> four; 2 (low 16 bits): eight -> four.  to_level() then
// subtracts L/2.
template <int BITS>
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t *o) {
  if constexpr (BITS == 8) {
    o[0] = __byte_perm(w, 0u, 0x4140);
    o[1] = __byte_perm(w, 0u, 0x4342);
  } else if constexpr (BITS == 4) {
    const uint32_t e = w & 0x0F0F0F0Fu, d = (w >> 4) & 0x0F0F0F0Fu;  // even / odd coordinates
    // result byte 0 <- byte k of e (coordinate 2k), byte 2 <- byte k of d
    // (coordinate 2k + 1); bytes 1 and 3 are masked off
    o[0] = __byte_perm(e, d, 0x7470) & 0x00FF00FFu;                  // coords 0, 1
    o[1] = __byte_perm(e, d, 0x7571) & 0x00FF00FFu;                  // coords 2, 3
    o[2] = __byte_perm(e, d, 0x7672) & 0x00FF00FFu;                  // coords 4, 5
    o[3] = __byte_perm(e, d, 0x7773) & 0x00FF00FFu;                  // coords 6, 7
  } else {
    // 2-bit codes: the eight codes of the word's low 16 bits, code k in bits 2k, 2k+1
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t t = w >> (4 * k);
      o[k] = (t & 3u) | ((t << 14) & 0x30000u);
    }
  }
}

// 32 lanes x 32 bit, 4 consecutive columns: thread i <-> lane (base + i)
__device__ __forceinline__ void tmem_st4(uint32_t taddr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r0), "r"(r1), "r"(r2),
               "r"(r3)
               : "memory");
}

// (n 2^-24, m 2^-24) -> ((n - L/2) 2^-24, (m - L/2) 2^-24): an fp16 subtraction
// of subnormals whose result is a subnormal, so exact
template <int BITS>
__device__ __forceinline__ uint32_t to_level(uint32_t w) {
  constexpr uint32_t h = 1u << (BITS - 1);  // L/2 as a subnormal's bit pattern
  const __half2 c = *reinterpret_cast<const __half2 *>(&(const uint32_t &)(h | (h << 16)));
  __half2 v = *reinterpret_cast<const __half2 *>(&w);
  v = __hsub2(v, c);
  return *reinterpret_cast<const uint32_t *>(&v);
}

template <int NQ, int NT, int BITS>
__global__ void __launch_bounds__(NT, Shape<NQ, NT>::MINB) absorbed_split_gen(Params p, int G) {
  constexpr int kThreads = NT;
  constexpr int NH = Shape<NQ, NT>::NH;      // heads of one softmax thread
  const Plan pl = plan_of(G, NQ, BITS);
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *zs = smem + pl.off_z;
  uint8_t *qs = smem + pl.off_q;
  uint8_t *ps = smem + pl.off_p;
  uint8_t *cs = smem + pl.off_c;
  Misc<NQ, NT / 32> &ms = *reinterpret_cast<Misc<NQ, NT / 32> *>(smem + pl.off_misc);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, b = blockIdx.y;
  const int64_t t0 = (int64_t)split * p.tps;
  const int64_t t1 = min(query_len(p.seq_lens, b, p.n_new, p.T, p.err, false), t0 + p.tps);
  float *out = p.part + (((size_t)b * p.S + split) * NQ) * (2 + G);
  if (t1 <= t0) {  // a split wholly past its row's length: an empty partial
    pdl_wait();
    for (int i = tid; i < NQ * (2 + G); i += kThreads) out[i] = (i % (2 + G)) == 0 ? -INFINITY : 0.f;
    return;
  }
  const int n_tiles = (int)((t1 - t0 + kTile - 1) / kTile);
  const int crow = b / p.n_new;
  const uint8_t *gcodes = p.codes + (int64_t)crow * p.bstride + t0 * pl.RB;
  const size_t cbb = code_buf_bytes(pl);
  const uint32_t tile_bytes = (uint32_t)(kTile * pl.RB);  // a multiple of 16 (128 x RB, RB >= 1)
  volatile uint32_t *abort = &ms.abort;
  const int KB = pl.Gp / 8;                 // 8-coordinate blocks holding codes

  if (tid == 0) {
    mbar_init(&ms.full[0], 1);
    mbar_init(&ms.full[1], 1);
    mbar_init(&ms.s_mid, 1);
    mbar_init(&ms.s_full, 1);
    mbar_init(&ms.p_mid, 1);
    mbar_init(&ms.p_done, 1);
    mbar_init(&ms.q_full, 1);
    mbar_init(&ms.done, 1);
    mbar_init(&ms.never, 1);  // completed by nothing: the test-only stall waits on it
    ms.abort = 0u;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&ms.tmem_base, pl.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ms.tmem_base;
  const uint64_t pol = p.n_new > 1 ? l2_evict_normal() : l2_evict_first();
  auto tile_rows = [&](int i) { return (int)min((int64_t)kTile, t1 - (t0 + (int64_t)i * kTile)); };
  // full tiles come by bulk copy (thread 0); the ragged last tile by bounded plain loads (all threads)
  int pend[2] = {-1, -1};  // thread 0: the tile whose copy into buffer k is issued and not yet consumed
  auto issue_copy = [&](int i) {
    if (tid == 0 && i < n_tiles && tile_rows(i) == kTile) {
      mbar_arrive_expect_tx(&ms.full[i & 1], tile_bytes);
      bulk_g2s_hint(cs + (i & 1) * cbb, gcodes + (int64_t)i * kTile * pl.RB, tile_bytes, &ms.full[i & 1], pol);
      pend[i & 1] = i;
    }
  };
  issue_copy(0);  // the codes were written before the query prologue ran
  issue_copy(1);
  pdl_trigger();  // the merge kernel may start staging W_v
  pdl_wait();     // Q' and the offsets come from the query prologue
  if (tid == 0) {
    mbar_arrive_expect_tx(&ms.q_full, (uint32_t)(pl.Gp * 4 * NQ));
    bulk_g2s(qs, p.qbuf + (size_t)b * pl.Gp * 4 * NQ, (uint32_t)(pl.Gp * 4 * NQ), &ms.q_full);
  }
  if (tid < NQ) ms.cneg[tid] = 0.f;  // provisional m = 0; the first tile rescales
  if (split == 0 && tid == 0) query_len(p.seq_lens, b, p.n_new, p.T, p.err, true);

  bool ok = true;
  auto fail = [&]() {
    record_error(p.err, FSQ_ERR_TIMEOUT);
    *abort = 1u;
  };
  if (!wait_bar(&ms.q_full, 0, abort, kWaitNs)) ok = false;
  // test-only stall: a wait that runs out on purpose (nothing completes `never`)
  if (p.stall_ns != 0u && !wait_bar(&ms.never, 0, abort, p.stall_ns)) ok = false;
  if (!ok) fail();

  // this thread's softmax rows and heads: warp w holds TMEM lanes 32 (w % 4) ..
  // (its tokens) and head group w / 4, heads (w / 4) NH ..
  const int q4 = warp & 3, hh = warp >> 2;
  const int r = 32 * q4 + lane;
  float lsum[NH];
#pragma unroll
  for (int k = 0; k < NH; ++k) lsum[k] = 0.f;
  const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
  constexpr uint32_t id_s = idesc_f16(128, 2 * NQ, 0, 0);  // A (TMEM) and B K-major
  constexpr uint32_t id_p = idesc_f16(128, NQ, 1, 1);
  const uint32_t z_a = smem_u32(zs), q_a = smem_u32(qs), p_a = smem_u32(ps);

  // chunk c of the coordinates: 128-blocks [mb_lo(c), mb_hi(c))
  const int nch = pl.nch;
  auto mb_lo = [&](int c) { return c == 0 ? 0 : pl.nmb0; };
  auto mb_hi = [&](int c) { return (c == 0 && nch == 2) ? pl.nmb0 : pl.NMB; };
  // unpack chunk c of the tile's codes into Z: thread -> token (tid % 128) and
  // every NP-th 8-coordinate block; a warp covers 32 consecutive tokens of one
  // block (512 contiguous bytes of Z)
  auto unpack = [&](const uint8_t *ct, int c, bool to_tmem, bool to_smem) {
    const uint32_t za = tm + ((uint32_t)(32 * (warp & 3)) << 16) + pl.off_za;  // this warp's lanes of Z in TMEM
    constexpr int NP = kThreads / kTile;
    constexpr int U = 4;                       // blocks whose code loads are issued together
    const int t = tid & (kTile - 1);
    const int part = tid / kTile;
    const uint8_t *row = ct + t * pl.RB;       // rows hold an even number of bytes: 2-byte aligned loads
    const int cbA = 16 * mb_lo(c), cbB = min(16 * mb_hi(c), KB);
    uint8_t *zt = zs + (t >> 3) * 128 + (t & 7) * 16;  // token t's row in the chunk's first block
    const int KBf = min(G / 8, cbB);           // blocks wholly inside G
    for (int c0 = cbA + part; c0 < KBf; c0 += U * NP) {
      uint32_t w[U][2];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int cb = c0 + u * NP;
        w[u][0] = 0u;
        w[u][1] = 0u;
        if (cb < KBf) {
          if constexpr (BITS == 8) {
            w[u][0] = lds_u32_a2(row + 8 * cb);
            w[u][1] = lds_u32_a2(row + 8 * cb + 4);
          } else if constexpr (BITS == 4) {
            w[u][0] = lds_u32_a2(row + 4 * cb);
          } else {
            w[u][0] = *reinterpret_cast<const uint16_t *>(row + 2 * cb);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int cb = c0 + u * NP;
        if (cb < KBf) {
          uint32_t o[4];
          unpack_word<BITS>(w[u][0], o);
          if constexpr (BITS == 8) unpack_word<8>(w[u][1], o + 2);
#pragma unroll
          for (int e = 0; e < 4; ++e) o[e] = to_level<BITS>(o[e]);
          if (to_smem)
            *reinterpret_cast<uint4 *>(zt + (size_t)(cb - cbA) * (kTile / 8) * 128) = make_uint4(o[0], o[1], o[2], o[3]);
          if (to_tmem) tmem_st4(za + 4 * cb, o[0], o[1], o[2], o[3]);  // warp-uniform: cb is the warp's
        }
      }
    }
    // blocks reaching past G (when G % 8 != 0, or Gp - G >= 8): codes past G count as 0
    for (int cb = max(KBf, cbA) + part; cb < cbB; cb += NP) {
      uint32_t v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int g = 8 * cb + e;
        v[e] = g < G ? (row[g * BITS / 8] >> ((g * BITS) % 8)) & ((1u << BITS) - 1u) : 0u;
      }
      const uint32_t o0 = to_level<BITS>(v[0] | (v[1] << 16)), o1 = to_level<BITS>(v[2] | (v[3] << 16));
      const uint32_t o2 = to_level<BITS>(v[4] | (v[5] << 16)), o3 = to_level<BITS>(v[6] | (v[7] << 16));
      if (to_smem) *reinterpret_cast<uint4 *>(zt + (size_t)(cb - cbA) * (kTile / 8) * 128) = make_uint4(o0, o1, o2, o3);
      if (to_tmem) tmem_st4(za + 4 * cb, o0, o1, o2, o3);
    }
    if (to_smem) fence_proxy_async_smem();
    if (to_tmem) tmem_st_wait();
  };
  // S = Z . Q'^T over all Gp coordinates: A from TMEM (8 columns per 16 coordinates), B from shared memory (thread 0)
  auto score_mmas = [&]() {
    tc_fence_after();
#pragma unroll 1
    for (int k = 0; k < pl.Gp / 16; ++k) {
      const uint64_t db = smem_desc(q_a + (uint32_t)(k * 2 * (2 * NQ / 8) * 128), (2 * NQ / 8) * 128, 128);
      mma_ts(tm, tm + pl.off_za + 8 * k, db, id_s, k > 0 ? 1u : 0u);
    }
  };
  // ACC[mb] += Z^T[mb] . P over the tile's 128 tokens for the 128-blocks of chunk c (thread 0)
  auto pool_mmas = [&](int c, int i) {
    tc_fence_after();
#pragma unroll 1
    for (int mb = mb_lo(c); mb < mb_hi(c); ++mb) {
#pragma unroll
      for (int k = 0; k < kTile / 16; ++k) {
        const uint64_t da =
            smem_desc(z_a + (uint32_t)((mb - mb_lo(c)) * 16 * (kTile / 8) * 128 + k * 256), 128, (kTile / 8) * 128);
        const uint64_t db = smem_desc(p_a + (uint32_t)(k * 256), 128, (kTile / 8) * 128);
        mma_ss(tm + 2 * NQ + mb * NQ, da, db, id_p, (i > 0 || k > 0) ? 1u : 0u);
      }
    }
  };

  // softmax of tile i (every thread: one token row, NH heads) and its P in
  // shared memory.  The previous tile's pooling must be complete (P is one
  // buffer; a rescale scales ACC).  Returns false when a failed wait ends the
  // tile loop (every thread the same).
  auto softmax_tile = [&](int i, int rows) -> bool {
      // ---- softmax (every thread: one token row, NH heads)
      float x[NH];
      {
        uint32_t sv[2 * NH];
        if constexpr (NH == 32) {
          tmem_ld32(tm + lane_base + hh * 2 * NH, sv);
          tmem_ld32(tm + lane_base + hh * 2 * NH + 32, sv + 32);
        } else if constexpr (NH == 16) {
          tmem_ld32(tm + lane_base + hh * 2 * NH, sv);
        } else {
          tmem_ld16(tm + lane_base + hh * 2 * NH, sv);
        }
        tmem_ld_wait();
        const bool valid = r < rows;
  #pragma unroll
        for (int k = 0; k < NH; ++k) {
          const float s = __uint_as_float(sv[k]) + __uint_as_float(sv[NH + k]);
          x[k] = valid ? fmaf(s, 16777216.f, ms.cneg[hh * NH + k]) : -INFINITY;
        }
      }
      float xm = -INFINITY;
  #pragma unroll
      for (int k = 0; k < NH; ++k) xm = fmaxf(xm, x[k]);
      // the rescale decision is the CTA's (every token of a head shares one max);
      // a failed wait ends the loop for every thread (two barriers, in this order)
      const int vote = __syncthreads_count((i == 0 || xm > kTau) ? 1 : 0);
      if (__syncthreads_or(!ok)) return false;
      if (vote > 0) {
        // raise the running max of each head: m <- m + max(0, tile max of x) (the first tile: its max)
  #pragma unroll
        for (int k = 0; k < NH; ++k) {
          float v = x[k];
  #pragma unroll
          for (int off = 16; off; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
          if (lane == 0) ms.red[warp][hh * NH + k] = v;
        }
        __syncthreads();
        float f[NH];
  #pragma unroll
        for (int k = 0; k < NH; ++k) {
          const int h = hh * NH + k;
          const int w0 = 4 * hh;  // the four warps holding head h's tokens
          const float d = fmaxf(fmaxf(ms.red[w0][h], ms.red[w0 + 1][h]), fmaxf(ms.red[w0 + 2][h], ms.red[w0 + 3][h]));
          const float sh = (i == 0) ? (d == -INFINITY ? 0.f : d) : fmaxf(d, 0.f);
          f[k] = (i == 0) ? 0.f : exp2f(-sh);
          x[k] -= sh;
          lsum[k] *= f[k];
          if (q4 == 0 && lane == 0) ms.cneg[h] -= sh;
        }
        if (i > 0) {
          // ACC holds every earlier tile (its pooling is done): scale this warp's lanes of its heads
  #pragma unroll 1
          for (int mb = 0; mb < pl.NMB; ++mb) {
            uint32_t a[NH];
            const uint32_t ta = tm + lane_base + 2 * NQ + mb * NQ + hh * NH;
            if constexpr (NH == 32) tmem_ld32(ta, a);
            else if constexpr (NH == 16) tmem_ld16(ta, a);
            else tmem_ld8(ta, a);
            tmem_ld_wait();
  #pragma unroll
            for (int k = 0; k < NH; ++k) a[k] = __float_as_uint(__uint_as_float(a[k]) * f[k]);
            if constexpr (NH == 32) tmem_st32(ta, a);
            else if constexpr (NH == 16) tmem_st16(ta, a);
            else tmem_st8(ta, a);
          }
          tmem_st_wait();
        }
      }
      // P row of this token (fp16, MN-major blocks: 8 tokens x 8 heads); the sum
      // takes the rounded weights the pooling MMA sees
  #pragma unroll
      for (int k8 = 0; k8 < NH / 8; ++k8) {
        uint32_t hv[4];
  #pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int k = 8 * k8 + 2 * e;
          const __half2 h2 = __floats2half2_rn(ex2_approx(x[k]), ex2_approx(x[k + 1]));
          const float2 back = __half22float2(h2);
          lsum[k] += back.x;
          lsum[k + 1] += back.y;
          hv[e] = *reinterpret_cast<const uint32_t *>(&h2);
        }
        const int hb = (hh * NH) / 8 + k8;
        *reinterpret_cast<uint4 *>(ps + ((size_t)hb * (kTile / 8) + (r >> 3)) * 128 + (r & 7) * 16) =
            make_uint4(hv[0], hv[1], hv[2], hv[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
    return true;
  };
  // the tile's codes (full tiles: the bulk copy; the ragged last tile: plain loads, zero past its rows)
  auto take_codes = [&](int i) -> bool {
    const int rows = tile_rows(i);
    if (rows == kTile && !wait_bar(&ms.full[i & 1], (uint32_t)(i >> 1) & 1u, abort, kWaitNs)) ok = false;
    if (__syncthreads_or(!ok)) return false;
    if (pend[i & 1] == i) pend[i & 1] = -1;  // every thread saw the copy complete
    if (rows < kTile) {
      // ragged last tile: its buffer is free (no copy was issued into it)
      uint8_t *dst = cs + (i & 1) * cbb;
      const uint8_t *src = gcodes + (int64_t)i * kTile * pl.RB;
      const int nb = rows * pl.RB;
      for (int k = tid; k < kTile * pl.RB; k += kThreads) dst[k] = k < nb ? src[k] : (uint8_t)0;
      __syncthreads();
    }
    return true;
  };

  int i = 0;
  for (; i < n_tiles; ++i) {
    if (__syncthreads_or(!ok)) break;
    const uint8_t *ct = cs + (i & 1) * cbb;
    // Z is free once the previous tile's pooling is done
    if (i > 0 && !wait_bar(&ms.p_done, (uint32_t)(i - 1) & 1u, abort, kWaitNs)) ok = false;
    if (!take_codes(i)) break;
    // Z to TMEM for the scores and to shared memory for the pooling (with two
    // chunks, shared memory keeps the second)
    if (nch == 1) {
      unpack(ct, 0, true, true);
      issue_copy(i + 2);  // this tile's code buffer has been read
    } else {
      unpack(ct, 0, true, false);
      unpack(ct, 1, true, true);
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      score_mmas();
      tc_commit(&ms.s_full);
    }
    if (!wait_bar(&ms.s_full, (uint32_t)i & 1u, abort, kWaitNs)) ok = false;
    tc_fence_after();
    if (!softmax_tile(i, tile_rows(i))) break;
    if (nch == 1) {
      if (tid == 0) {
        pool_mmas(0, i);
        tc_commit(&ms.p_done);
      }
    } else {
      // the resident second chunk first, then the first chunk unpacked again
      if (tid == 0) {
        pool_mmas(1, i);
        tc_commit(&ms.p_mid);
      }
      if (!wait_bar(&ms.p_mid, (uint32_t)i & 1u, abort, kWaitNs)) ok = false;
      if (__syncthreads_or(!ok)) break;
      unpack(ct, 0, false, true);
      __syncthreads();
      issue_copy(i + 2);  // this tile's code buffer has been read
      if (tid == 0) {
        pool_mmas(0, i);
        tc_commit(&ms.p_done);
      }
    }
  }
  // ---- epilogue: ACC -> partials (m, l, ACC) in latent units
  bool good = ok && i == n_tiles;
  if (good && !wait_bar(&ms.p_done, (uint32_t)(n_tiles - 1) & 1u, abort, kWaitNs)) good = false;
  if (__syncthreads_or(!good)) {
    if (tid == 0) {
      fail();
      // let every issued MMA and copy finish before TMEM is freed and the CTA exits
      tc_commit(&ms.done);
      mbar_wait_fixed(&ms.done, 0, kDrainNs);
      for (int k = 0; k < 2; ++k)
        if (pend[k] >= 0) mbar_wait_fixed(&ms.full[k], (uint32_t)(pend[k] >> 1) & 1u, kDrainNs);
    }
  } else {
    tc_fence_after();
    // l per head: the rounded weights of every token of the split
#pragma unroll
    for (int k = 0; k < NH; ++k) {
      float v = lsum[k];
#pragma unroll
      for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) ms.red[warp][hh * NH + k] = v;
    }
    __syncthreads();
    if (tid < NQ) {
      const int h = tid, w0 = 4 * (h / NH);
      const float lt = (ms.red[w0][h] + ms.red[w0 + 1][h]) + (ms.red[w0 + 2][h] + ms.red[w0 + 3][h]);
      out[(size_t)h * (2 + G)] = -ms.cneg[h];
      out[(size_t)h * (2 + G) + 1] = lt;
    }
#pragma unroll 1
    for (int mb = 0; mb < pl.NMB; ++mb) {
      uint32_t a[NH];
      const uint32_t ta = tm + lane_base + 2 * NQ + mb * NQ + hh * NH;
      if constexpr (NH == 32) tmem_ld32(ta, a);
      else if constexpr (NH == 16) tmem_ld16(ta, a);
      else tmem_ld8(ta, a);
      tmem_ld_wait();
      const int g = 128 * mb + r;  // TMEM lane = coordinate within the block
      if (g < G) {
#pragma unroll
        for (int k = 0; k < NH; ++k) {
          const int h = hh * NH + k;
          out[(size_t)h * (2 + G) + 2 + g] = __uint_as_float(a[k]) * 16777216.f;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, pl.tmem_cols);
  }
}

// ---------------------------------------------------------------- prologue
// Per (kv head j, grid row b): q'_h[g] = c sum_d W_k[j d_h + d][g] q_h[d]
// (c = scale log2 e) for the group's heads, split into fp16 hi + lo, written
// in the score MMA's B layout: row n = (h / NH) 2 NH + term NH + h % NH, 8 x 8
// blocks (rows x coordinates) at ((g / 8) (2 NQ / 8) + n / 8) 128 bytes; the
// coordinates in [G, Gp) are zero.  Also clears the error word and the merge's
// arrival counts.
template <int NQ, int NH>
__global__ void __launch_bounds__(256) gen_query(const uint16_t *__restrict__ q, const uint16_t *__restrict__ W_kv,
                                                 int n_kv, int G, float c, uint8_t *__restrict__ qbuf, uint32_t *err,
                                                 MergeScratch msc) {
  constexpr int D = FSQ_HEAD_DIM;
  __shared__ float qsm[16][D];
  const int j = blockIdx.x, b = blockIdx.y;
  const int grp = NQ / n_kv;
  const int Gp = (G + 15) / 16 * 16;
  if (j == 0 && b == 0) {
    if (threadIdx.x == 0) *err = 0u;
    for (int i = threadIdx.x; i < msc.ncnt; i += blockDim.x) msc.cnt[i] = 0u;
  }
  for (int i = threadIdx.x; i < grp * D; i += blockDim.x)
    qsm[i / D][i % D] = bf16_to_f32(q[((int64_t)b * NQ + j * grp) * D + i]);
  __syncthreads();
  uint8_t *dst = qbuf + (size_t)b * Gp * 4 * NQ;
  for (int g = threadIdx.x; g < Gp; g += blockDim.x) {
    float v[16];
#pragma unroll
    for (int hh = 0; hh < 16; ++hh) v[hh] = 0.f;
    if (g < G) {
      const uint16_t *w = W_kv + (int64_t)j * D * G + g;
      for (int d = 0; d < D; ++d) {
        const float wd = bf16_to_f32(w[(int64_t)d * G]);
#pragma unroll
        for (int hh = 0; hh < 16; ++hh)
          if (hh < grp) v[hh] = fmaf(wd, qsm[hh][d], v[hh]);
      }
    }
#pragma unroll
    for (int hh = 0; hh < 16; ++hh) {
      if (hh >= grp) break;
      const int h = j * grp + hh;
      const float qv = v[hh] * c;
      const __half hi = __float2half_rn(qv);
      const __half lo = __float2half_rn(qv - __half2float(hi));
      const int n_hi = (h / NH) * 2 * NH + (h % NH), n_lo = n_hi + NH;
      *reinterpret_cast<__half *>(dst + ((size_t)(g >> 3) * (2 * NQ / 8) + (n_hi >> 3)) * 128 + (n_hi & 7) * 16 +
                                  (g & 7) * 2) = hi;
      *reinterpret_cast<__half *>(dst + ((size_t)(g >> 3) * (2 * NQ / 8) + (n_lo >> 3)) * 128 + (n_lo & 7) * 16 +
                                  (g & 7) * 2) = lo;
    }
  }
  pdl_wait();
  pdl_trigger();  // the split kernel may start its prologue and code loads
}

template <int NQ, int NT, int BITS>
cudaError_t launch_t(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t R, int n_new, int64_t T,
                     const int32_t *seq_lens, int n_kv, int G, int levels, const uint16_t *W_kv, float scale, int S,
                     int64_t tps, uint8_t *qbuf, float *part, uint32_t *err, MergeScratch ms, uint32_t stall_ns,
                     void *const *prof, cudaStream_t st) {
  cudaError_t e = launch_pdl(gen_query<NQ, Shape<NQ, NT>::NH>, dim3(n_kv, (unsigned)R), dim3(256), 0, st, q, W_kv,
                             n_kv, G, scale * kLog2e, qbuf, err, ms);
  if (e != cudaSuccess) return e;
  const Plan pl = plan_of(G, NQ, BITS);
  const size_t smem = pl.total;
  auto kern = absorbed_split_gen<NQ, NT, BITS>;
  e = ensure_smem_limit((const void *)kern, smem);
  if (e != cudaSuccess) return e;
  Params p{codes, bstride, T, tps, S, n_new, levels, qbuf, part, err, seq_lens, stall_ns};
  record_prof_event(prof[0], st);
  e = launch_pdl(kern, dim3(S, (unsigned)R), dim3(NT), smem, st, p, G);
  record_prof_event(prof[1], st);
  return e;
}

}  // namespace gen
}  // namespace tc

// The generic tensor-core absorbed kernel covers n_q in {16, 32, 64} (N of the
// MMAs), any supported level count, rows of an even number of bytes (its code
// loads are 2-byte aligned), and widths whose shared-memory plan fits.
bool absorbed_gen_supported(int n_q, int n_kv, int G, int levels) {
  if (!(n_q == 16 || n_q == 32 || n_q == 64) || n_kv < 1 || n_q % n_kv || n_q / n_kv > 16) return false;
  const int bits = bits_of_levels(levels);
  if (!bits || G < 2 || G % 2 || G > FSQ_MAX_G || (G * bits / 8) % 2) return false;
  const tc::gen::Plan pl = tc::gen::plan_of(G, n_q, bits);
  return pl.total <= tc::gen::kSmemMax && pl.tmem_cols <= 512;
}

size_t absorbed_gen_qbuf_bytes(int n_q, int G) { return (size_t)((G + 15) / 16 * 16) * 4 * n_q; }

// CTAs of the split kernel that one SM holds at once (the split planner fills
// all of them in one wave, so one CTA's sequential steps overlap another's):
// bounded by shared memory (228 KB per SM, 1 KB reserved per CTA), TMEM (512
// columns) and registers (64 K per SM: the 256-thread kernels are built for
// two CTAs per SM at n_q <= 32, one at n_q = 64).
static int gen_fit(int n_q, int G, int levels) {
  const tc::gen::Plan pl = tc::gen::plan_of(G, n_q, bits_of_levels(levels));
  const int by_smem = (int)((228 * 1024) / (pl.total + 1024));
  const int by_tmem = 512 / pl.tmem_cols;
  const int by_regs = n_q >= 64 ? 1 : 2;
  int c = by_smem < by_tmem ? by_smem : by_tmem;
  c = c < by_regs ? c : by_regs;
  return c < 1 ? 1 : c;
}
// Threads per CTA: 512 at n_q = 32 when a single 256-thread CTA fills an SM.
static int gen_threads(int n_q, int G, int levels) { return n_q == 32 && gen_fit(n_q, G, levels) < 2 ? 512 : 256; }
int absorbed_gen_ctas_per_sm(int n_q, int G, int levels) {
  return gen_threads(n_q, G, levels) == 512 ? 1 : gen_fit(n_q, G, levels);
}

cudaError_t merge_absorbed_launch(const float *part, int S, int64_t B, int n_q, int n_kv, int d_h, int G,
                                  const uint16_t *W_kv, void *o, int out_fp32, MergeScratch ms, cudaStream_t st,
                                  int fold_bytes);

// R: grid rows (cache rows x n_new queries).
cudaError_t launch_absorbed_gen(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t R, int n_new,
                                int64_t T, const int32_t *seq_lens, int n_q, int n_kv, int d_h, int G, int levels,
                                const uint16_t *W_kv, float scale, int S, int64_t tps, uint8_t *qbuf, float *part,
                                uint32_t *err, MergeScratch ms, void *o, int out_fp32, uint32_t stall_ns,
                                void *const *prof, cudaStream_t st) {
  const int bits = bits_of_levels(levels);
  cudaError_t e = cudaErrorInvalidValue;
  const int nt = gen_threads(n_q, G, levels);
#define FSQ_GEN(NN, TT, BB)                                                                                           \
  tc::gen::launch_t<NN, TT, BB>(q, codes, bstride, R, n_new, T, seq_lens, n_kv, G, levels, W_kv, scale, S, tps, qbuf, \
                                part, err, ms, stall_ns, prof, st)
#define FSQ_GEN_NQ(NN, TT)                     \
  if (bits == 2) e = FSQ_GEN(NN, TT, 2);       \
  else if (bits == 4) e = FSQ_GEN(NN, TT, 4);  \
  else if (bits == 8) e = FSQ_GEN(NN, TT, 8);
  if (n_q == 16) { FSQ_GEN_NQ(16, 256) }
  else if (n_q == 32 && nt == 512) { FSQ_GEN_NQ(32, 512) }
  else if (n_q == 32) { FSQ_GEN_NQ(32, 256) }
  else if (n_q == 64) { FSQ_GEN_NQ(64, 256) }
#undef FSQ_GEN_NQ
#undef FSQ_GEN
  if (e != cudaSuccess) return e;
  return merge_absorbed_launch(part, S, R, n_q, n_kv, d_h, G, W_kv, o, out_fp32, ms, st, 0);
}

}  // namespace fsq
