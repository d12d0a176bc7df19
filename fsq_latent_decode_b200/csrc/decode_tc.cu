// Decode attention over packed FSQ codes on the 5th-generation tensor cores
// (tcgen05 / TMEM), absorbed form.
//
// Per batch row and token split, every query head shares the same latent code
// tile, so both contractions are dense ([S] Architecture: one latent serves all
// KV heads; [D] frame "Attention pools codes before decoding values"):
//   S   [128 tokens x n_q]  = Z [128 x G]      . Q'^T [G x n_q]   (Q' = (W_k^T q) * scale * log2 e)
//   ACC [G x n_q]          += Z^T [G x 128]     . P [128 x n_q]    (P = online-softmax weights)
// and W_v is applied once to ACC / l after the split merge ([S] eq. 6).
//
// Data path per 128-token tile (slide deck frame "The kernel reads codes and
// never writes reconstructed K/V": read packed codes, unpack in registers,
// tensor cores, online softmax, merge partials):
//   bulk copy (1-D, 16-B aligned) of the packed rows into a shared-memory ring
//   -> score-dequant warps unpack each token's nibbles in registers into
//      token-major Z in TMEM (A of the score MMA, double-buffered)
//   -> pool-dequant warps build coordinate-major Z^T in TMEM (A of the pooling
//      MMA, in two 64-token chunks): the still-packed 16-bit groups of four
//      nibbles are read transposed in 8x8 blocks (ldmatrix.trans; movmatrix
//      when rows are not 16-byte aligned), then unpacked, so one transpose
//      serves four coordinates
//   -> three issuer threads (score MMAs; pooling MMAs of each 128-row half or
//      chunk) keep the tensor core fed: a single issuing thread cannot issue
//      small-N MMAs as fast as the tensor core retires them
//   -> softmax warps read S from TMEM, keep the running max, write P (fp16)
//      to shared memory, rescale ACC in TMEM when the max grows.
//
// Score MMA (kind::i8): the codes enter as unsigned bytes n = level + 8 (one
// LOP3 or SHF+LOP3 per four nibbles), and Q' is split per head into two int8
// terms, Q' ~ sigma (128 a + b), stacked along N (2 n_q columns), so the score
// is exact integer arithmetic on a 15-bit Q': s = sigma (128 S_a + S_b) minus a
// per-head offset for the -8 level shift.  Pooling MMA (kind::f16): one LOP3
// per pair (plus a shift shared by two pairs) leaves each nibble in place in
// the mantissa of an fp16 subnormal, n 2^-24 or n 2^-20; the products with the
// fp16 weights are exact, the pooled sums carry no bias, and the epilogue
// scales them back and removes the level offset (8 l per head).
//
// Warps (24): 0 loads code tiles and owns TMEM; 1 issues score MMAs; 2-3 issue
// pooling MMAs; 4-7 score dequant; 12-15 and 16-19 pooling dequant for the
// first and second 64-token chunk of every tile; 8-11 and 20-23 softmax for
// the first and second half of the heads (each group of four covers TMEM
// sub-partitions 0-3).  Every wait is
// bounded; on a timeout the CTA records FSQ_ERR_TIMEOUT in the workspace error
// word and all roles drain and exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "tc_decode.cuh"
#include "tc_ptx.cuh"

namespace fsq {
namespace tc {

using namespace ptx;

constexpr int kTile = 128;
constexpr int kMaxStages = 16;                     // code-tile ring depth bound (barrier arrays)
constexpr int kSmemBudget = 224 * 1024;            // shared memory a CTA plans for
// The pooled products are all non-negative (nibbles n = level + 8) and the
// tensor core's fp32 accumulation is not round-to-nearest, so one MMA chain
// over a long split drifts by a bias that grows with its length; the
// epilogue's -8 l correction cancels most of the sum and magnifies it (1.45 %
// on a flat softmax over 131k tokens).  Splits of up to kFoldAbove tokens
// (every one-wave plan of the benchmarked shapes) stay within 0.15 %; longer
// ones run the FOLD instance, whose softmax warps move the accumulator into
// fp32 sums of their own every kFlushTiles tiles while the pooling MMAs start
// a fresh chain.  The folding code costs the hot loop about 10 %, so the
// shorter splits run without it.
constexpr int kFlushTiles = 64;
constexpr int64_t kFoldAbove = 16384;
constexpr int kQAfterTiles = 4;                    // code tiles requested before Q' (and its wait)
constexpr float kTau = 8.f;                        // rescale when a score exceeds the running max by 2^8
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s per hand-off wait
constexpr uint64_t kDrainNs = 1000000000ull;       // 1 s for in-flight copies and MMAs on the error path
constexpr int kMiscBytes = 12288;                  // shared-memory reservation for the Misc block
constexpr int kPBufs = 8;                          // ring of softmax-weight (P) tiles in shared memory

template <int G, int NQ>
struct Cfg {
  static constexpr int HALF = G / 2;                 // bytes per token row
  // softmax: NSG groups of four warps, each group owning HQ = 8 heads
  static constexpr int NSG = NQ / 8;
  static constexpr int HQ = NQ / NSG;
  static constexpr int NSMX = 4 * NSG;               // softmax warps
  static constexpr int THREADS = (16 + NSMX) * 32;
  static constexpr int KPAD = (G + 31) / 32 * 32;    // K of the score MMA (32 per kind::i8 step)
  static constexpr int KW = KPAD / 8;                // 32-bit code words (8 coordinates) per padded row
  static constexpr int SCOLS = KPAD / 4;             // TMEM columns of token-major Z (4 bytes per column)
  static constexpr int NS = 2 * NQ;                  // score-MMA N: the a and b terms of every head
  static constexpr int NH = (G + 127) / 128;         // 128-row halves of the pooling MMA
  static constexpr int TILE_BYTES = kTile * HALF;
  // G=256: 128-byte rows arrive by a 2-D TMA copy in 128-byte-swizzle mode, so
  // that both dequant access patterns are free of shared-memory bank conflicts.
  // Other G: 1-D bulk copy of the contiguous rows (+16 bytes for over-reads).
  static constexpr bool TMA = (HALF == 128);
  static constexpr int STAGE_BYTES = TMA ? TILE_BYTES : (TILE_BYTES + 16 + 127) / 128 * 128;
  static constexpr int Q_BYTES = NS * KPAD;          // int8 Q' terms in the K-major no-swizzle layout
  static constexpr int P_BYTES = kTile * NQ * 2;     // P in the MN-major no-swizzle layout
  // TMEM columns: Z (score A) x2 | Z^T 64-token chunks (pool A) x NCP | S x2 | ACC
  static constexpr int CS_COLS = (SCOLS + 15) / 16 * 16;
  static constexpr int CP_CHUNK = NH * 32;           // one 64-token chunk of Z^T
  static constexpr int OFF_CS = 0;
  static constexpr int ACC_COLS = 2 * NQ;            // NH=2: one per half; NH=1: one per chunk
  // Z^T chunk ring: four chunks (two tiles) when TMEM allows, else three
  static constexpr int NCP = (2 * CS_COLS + 4 * CP_CHUNK + 2 * NS + ACC_COLS) <= 512 ? 4 : 3;
  static constexpr int OFF_CP = 2 * CS_COLS;
  static constexpr int OFF_S = OFF_CP + NCP * CP_CHUNK;  // two S buffers
  static constexpr int OFF_ACC = OFF_S + 2 * NS;
  static constexpr int TMEM_USED = OFF_ACC + ACC_COLS;
  static constexpr int TMEM_COLS = TMEM_USED <= 256 ? 256 : 512;
  static_assert(TMEM_USED <= 512, "TMEM plan exceeds 512 columns");
  // shared memory
  static constexpr int SM_CODES = 0;
  // Code-tile ring: as deep as the shared memory left over allows (bytes in
  // flight per SM hide the load latency), at most kMaxStages
  static constexpr int FL_BYTES = 16 * NSMX * 32 * 4;   // 16 flushed fp32 sums per softmax thread
  static constexpr int OTHER_BYTES = Q_BYTES + kPBufs * P_BYTES + kMiscBytes + FL_BYTES;
  static constexpr int STAGES_FIT = (kSmemBudget - OTHER_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT < kMaxStages ? STAGES_FIT : kMaxStages;
  static_assert(STAGES >= 4, "code-tile ring too shallow");
  static constexpr int SM_Q = SM_CODES + STAGES * STAGE_BYTES;
  static constexpr int SM_P = SM_Q + Q_BYTES;
  static constexpr int SM_MISC = SM_P + kPBufs * P_BYTES;
  static constexpr int SM_FL = SM_MISC + kMiscBytes;
  static constexpr int SM_TOTAL = SM_FL + FL_BYTES;
  static constexpr int LBO_Q = (NS / 8) * 128;       // 16-byte K-chunk stride of Q'
  static constexpr int SBO_P = (kTile / 8) * 128;    // N-group stride of P
};

struct Params {
  const uint8_t *codes;
  int64_t bstride;
  int64_t T;
  int64_t tps;
  int S;
  const uint8_t *qphys;  // per batch row: Q' bytes in the shared-memory layout
  const float *corr;     // per batch row: [NQ] sigma, then [NQ] score offsets
  float *part;           // [B][S][NQ][2 + G]
  uint32_t *err;
  uint64_t wait_ns;      // limit of every hand-off wait
  const int32_t *seq_lens;  // per-row lengths (ragged batch) or null
  uint32_t stall_ns;     // test-only: > 0 makes the softmax wait on `never` first
  int n_new;             // queries per cache row: grid row r reads cache row r / n_new (causal)
};

struct Misc {
  uint64_t full[kMaxStages], empty[kMaxStages];
  uint64_t cs_ready[2], cs_free[2];
  uint64_t cp_ready[4], cp_free[4];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[kPBufs], p_free[kPBufs];
  uint64_t acc_full, q_full, done[5], never;
  uint32_t tmem_base;
  uint32_t abort;
  float red[4][64];
  float fac[16][64];
  float m[64];
  float lt[64];
  __align__(16) float cm[16][64];  // per softmax warp: -(score offset + running max), per head
  float corr[64];
  __align__(16) float sig[64];
};

// Score operand bytes from one packed word: even coordinates, then odd ones.
static_assert(sizeof(Misc) <= kMiscBytes, "Misc block exceeds its shared-memory reservation");

__device__ __forceinline__ uint32_t nib_even(uint32_t w) { return w & 0x0F0F0F0Fu; }
__device__ __forceinline__ uint32_t nib_odd(uint32_t w) { return (w >> 4) & 0x0F0F0F0Fu; }

// Instruction descriptor for kind::i8: D s32, A unsigned, B signed.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_ts_i8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
template <int G, int NQ, bool FOLD>
__global__ void __launch_bounds__(Cfg<G, NQ>::THREADS, 1) absorbed_split_tc(const __grid_constant__ CUtensorMap tmap, Params p) {
  using C = Cfg<G, NQ>;
  extern __shared__ __align__(1024) uint8_t smem[];
  Misc &ms = *reinterpret_cast<Misc *>(smem + C::SM_MISC);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, b = blockIdx.y;
  const int64_t t0 = (int64_t)split * p.tps;
  const int64_t t1 = min(query_len(p.seq_lens, b, p.n_new, p.T, p.err, false), t0 + p.tps);
  if (t1 <= t0) {
    // this split lies wholly past its row's length (ragged batch, causal query): an empty
    // partial, which the merge weighs by 2^-inf = 0
    pdl_wait();
    float *out = p.part + (((size_t)b * p.S + split) * NQ) * (2 + G);
    for (int i = tid; i < NQ * (2 + G); i += C::THREADS) out[i] = (i % (2 + G)) == 0 ? -INFINITY : 0.f;
    return;
  }
  const int n_tiles = (int)((t1 - t0 + kTile - 1) / kTile);
  const int crow = b / p.n_new;  // cache row
  const uint8_t *gcodes = p.codes + (int64_t)crow * p.bstride + t0 * C::HALF;
  volatile uint32_t *abort = &ms.abort;
  constexpr uint32_t kPoolIssuers = 2;

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&ms.full[s], 1);
      mbar_init(&ms.empty[s], 12);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ms.cs_ready[i], 4);
      mbar_init(&ms.cs_free[i], 1);
    }
    for (int i = 0; i < kPBufs; ++i) {
      mbar_init(&ms.p_full[i], C::NSMX);
      mbar_init(&ms.p_free[i], kPoolIssuers);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&ms.cp_ready[i], 4);
      mbar_init(&ms.cp_free[i], C::NH == 2 ? 2 : 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ms.s_full[i], 1);
      mbar_init(&ms.s_free[i], C::NSMX);
    }
    mbar_init(&ms.acc_full, kPoolIssuers);
    mbar_init(&ms.q_full, 1);
    for (int i = 0; i < 5; ++i) mbar_init(&ms.done[i], 1);
    mbar_init(&ms.never, 1);  // completed by nothing: the test-only stall waits on it
    ms.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&ms.tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ms.tmem_base;
  pdl_trigger();  // the merge kernel may start staging W_v

  auto fail = [&]() {
    record_error(p.err, FSQ_ERR_TIMEOUT);
    *abort = 1u;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint8_t *ring = smem + C::SM_CODES;
    // The codes were written before the query prologue kernel started, so the
    // first ring-full of tiles is requested before waiting for that kernel;
    // Q' (its output) right after, before the first wait for a free stage.
    const uint64_t pol = p.n_new > 1 ? l2_evict_normal() : l2_evict_first();
    auto load_q = [&]() {
      if (lane == 0) {
        pdl_wait();
        mbar_arrive_expect_tx(&ms.q_full, C::Q_BYTES);
        bulk_g2s(smem + C::SM_Q, p.qphys + (size_t)b * C::Q_BYTES, C::Q_BYTES, &ms.q_full);
      }
    };
    int issued = 0;
    bool ok = true, q_loaded = false;
    for (int i = 0; i < n_tiles; ++i) {
      const int st = i % C::STAGES;
      const uint32_t ph = (uint32_t)(i / C::STAGES) & 1u;
      if (i == kQAfterTiles) {
        load_q();
        q_loaded = true;
      }
      if (!wait_bar(&ms.empty[st], ph ^ 1u, abort, p.wait_ns)) {
        ok = false;
        break;
      }
      const int64_t rows = min((int64_t)kTile, t1 - (t0 + (int64_t)i * kTile));
      uint8_t *dst = ring + st * C::STAGE_BYTES;
      const uint8_t *src = gcodes + (int64_t)i * kTile * C::HALF;
      if constexpr (C::TMA) {
        // rows past T arrive as zeros; rows past this split's end are masked by the softmax
        if (lane == 0) {
          mbar_arrive_expect_tx(&ms.full[st], C::TILE_BYTES);
          tma_load_3d(dst, &tmap, 0, (int)(t0 + (int64_t)i * kTile), crow, &ms.full[st], pol);
        }
      } else if (rows == kTile) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&ms.full[st], C::TILE_BYTES);
          bulk_g2s_hint(dst, src, C::TILE_BYTES, &ms.full[st], pol);
        }
      } else {
        // ragged tail: plain bounded loads, zero fill
        const int nb = (int)rows * C::HALF;
        for (int k = lane; k < C::STAGE_BYTES; k += 32) dst[k] = (k < nb) ? src[k] : (uint8_t)0;
        __syncwarp();
        if (lane == 0) mbar_arrive(&ms.full[st]);
      }
      issued = i + 1;
    }
    if (!q_loaded) load_q();
    if (!ok) {
      if (lane == 0) fail();
      // let the copies still in flight land before the CTA exits
      for (int i = max(0, issued - C::STAGES); i < issued; ++i)
        drain_bar(&ms.full[i % C::STAGES], (uint32_t)(i / C::STAGES) & 1u, kDrainNs);
      drain_bar(&ms.q_full, 0, kDrainNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ score-MMA issuer (whole warp, one lane issues)
    constexpr uint32_t id_s = idesc_i8(128, C::NS);
    const uint64_t qd0 = smem_desc(smem_u32(smem + C::SM_Q), C::LBO_Q, 128);
    bool ok = wait_bar(&ms.q_full, 0, abort, p.wait_ns);
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int sb = i & 1;
      // S(i) is released to the softmax only once P buffer i % kPBufs is free
      // again (pooling of tile i - kPBufs done), so the softmax never waits for it
      ok = wait_bars(&ms.cs_ready[sb], (uint32_t)(i >> 1) & 1u, &ms.s_free[sb], ((uint32_t)(i >> 1) & 1u) ^ 1u,
                     &ms.p_free[i % kPBufs], ((uint32_t)(i / kPBufs) & 1u) ^ 1u, abort, p.wait_ns);
      if (!ok) break;
      tc_fence_after();
      const uint32_t a0 = tm + C::OFF_CS + sb * C::CS_COLS;
      const uint32_t d = tm + C::OFF_S + sb * C::NS;
      if (elect_one()) {  // one lane issues the tile's MMAs and both commits
#pragma unroll
        for (int k = 0; k < C::KPAD / 32; ++k)
          mma_ts_i8(d, a0 + k * 8, qd0 + (uint64_t)((k * 2 * C::LBO_Q) >> 4), id_s, k > 0 ? 1u : 0u);
        tc_commit(&ms.s_full[sb]);
        tc_commit(&ms.cs_free[sb]);
      }
      __syncwarp();
    }
    if (!ok && lane == 0) fail();
    // every MMA of this warp completes before TMEM is freed, error or not
    tc_commit_elect(&ms.done[0]);
    drain_bar(&ms.done[0], 0, kDrainNs);
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ pooling-MMA issuers (whole warp, one lane issues)
    const int k_iss = warp - 2;  // NH=2: half k_iss, both chunks; NH=1: chunk k_iss
    constexpr uint32_t id_p = idesc_f16(128, NQ, 0, 1);
    const uint64_t pd0 = smem_desc(smem_u32(smem + C::SM_P), 128, C::SBO_P);
    const int h = C::NH == 2 ? k_iss : 0;
    const uint32_t d = tm + C::OFF_ACC + k_iss * NQ;
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int pb = i % kPBufs;
      ok = wait_bar(&ms.p_full[pb], (uint32_t)(i / kPBufs) & 1u, abort, p.wait_ns);
      if (!ok) break;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (C::NH == 1 && c != k_iss) continue;
        const int kc = 2 * i + c;  // chunk index; ring buffer kc % NCP, use kc / NCP
        const int cb = kc % C::NCP;
        if (!wait_bar(&ms.cp_ready[cb], (uint32_t)(kc / C::NCP) & 1u, abort, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a0 = tm + C::OFF_CP + cb * C::CP_CHUNK + h * 32;
        const uint64_t bd0 = pd0 + (uint64_t)((pb * C::P_BYTES + 4 * c * 256) >> 4);
        if (elect_one()) {  // one lane issues the chunk's MMAs and its commit
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const bool first = (FOLD ? i % kFlushTiles == 0 : i == 0) && (C::NH == 1 ? kk == 0 : (c == 0 && kk == 0));
            mma_ts(d, a0 + kk * 8, bd0 + (uint64_t)(kk * 16), id_p, first ? 0u : 1u);
          }
          tc_commit(&ms.cp_free[cb]);
        }
        __syncwarp();
      }
      if (!ok) break;
      tc_commit_elect(&ms.p_free[pb]);
    }
    if (ok) tc_commit_elect(&ms.acc_full);
    else if (lane == 0) fail();
    tc_commit_elect(&ms.done[2 + k_iss]);
    drain_bar(&ms.done[2 + k_iss], 0, kDrainNs);
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ score dequant: token row -> TMEM lane
    const int q = warp - 4;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      const int st = i % C::STAGES, sb = i & 1;
      const uint8_t *tile = smem + C::SM_CODES + st * C::STAGE_BYTES;
      if (!wait_bars(&ms.full[st], (uint32_t)(i / C::STAGES) & 1u, &ms.cs_free[sb], ((uint32_t)(i >> 1) & 1u) ^ 1u,
                     abort, p.wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint8_t *row = tile + (32 * q + lane) * C::HALF;
      const uint32_t cbase = tm + lane_base + C::OFF_CS + sb * C::CS_COLS;
      // word k (coordinates 8k..8k+7) -> TMEM columns 2k (even coordinates) and 2k+1 (odd)
#pragma unroll
      for (int c0 = 0; c0 < C::KW; c0 += 16) {
        const int nw = (C::KW - c0) < 16 ? (C::KW - c0) : 16;
        uint32_t r[32];
        if constexpr (C::TMA) {
          const int rr = 32 * q + lane;
#pragma unroll
          for (int hv = 0; hv < 2; ++hv) {
            uint32_t r16[16];
#pragma unroll
            for (int v2 = 0; v2 < 2; ++v2) {
              const int v = 2 * hv + v2;
              const uint4 u = *reinterpret_cast<const uint4 *>(tile + swz(rr, c0 / 4 + v));
              r16[8 * v2 + 0] = nib_even(u.x); r16[8 * v2 + 1] = nib_odd(u.x);
              r16[8 * v2 + 2] = nib_even(u.y); r16[8 * v2 + 3] = nib_odd(u.y);
              r16[8 * v2 + 4] = nib_even(u.z); r16[8 * v2 + 5] = nib_odd(u.z);
              r16[8 * v2 + 6] = nib_even(u.w); r16[8 * v2 + 7] = nib_odd(u.w);
            }
            tmem_st16(cbase + 2 * c0 + 16 * hv, r16);
          }
          continue;
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int kw = c0 + k;
            uint32_t w = 0u;
            if (4 * kw + 4 <= C::HALF) w = lds_u32_a2(row + 4 * kw);
            else if (4 * kw + 2 <= C::HALF) w = *reinterpret_cast<const uint16_t *>(row + 4 * kw);
            r[2 * k] = nib_even(w);
            r[2 * k + 1] = nib_odd(w);
          }
        }
        if (nw == 16) {
          tmem_st32(cbase + 2 * c0, r);
        } else {
          if (nw >= 8) tmem_st16(cbase + 2 * c0, r);
          if (nw % 8 == 4) tmem_st8(cbase + 2 * c0 + 2 * (nw - 4), r + 2 * (nw - 4));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.empty[st]);  // this warp is done with the stage
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.cs_ready[sb]);
    }
    if (!ok && lane == 0) fail();
  } else if (warp >= 12 && warp < 20) {
    // ------------------------------------------------------------ pooling dequant: coordinates -> TMEM lanes
    // group c = 0 / 1 builds 64-token chunk c of every tile (chunk index 2i + c) into ring buffer (2i + c) % NCP
    const int q = warp & 3;
    const int c = (warp - 12) >> 2;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int st = i % C::STAGES;
      const int kc = 2 * i + c;
      const int cb = kc % C::NCP;
      const uint8_t *tile = smem + C::SM_CODES + st * C::STAGE_BYTES;
      if (!wait_bars(&ms.full[st], (uint32_t)(i / C::STAGES) & 1u, &ms.cp_free[cb], ((uint32_t)(kc / C::NCP) & 1u) ^ 1u,
                     abort, p.wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < C::NH; ++h) {
        const int byte0 = 64 * h + 16 * q;  // first byte of this warp's 32 coordinates
        if (byte0 >= C::HALF) continue;
        uint32_t lo[16];
        // y[2j + e]: the 8x8 block of 16-bit groups (four nibbles of one token)
        // of tokens 8 tb .. 8 tb + 7, tb = 8c + 2j + e, transposed, so this
        // thread holds one group (four coordinates) of two tokens
        uint32_t y[8];
        if constexpr (C::TMA) {
          const uint32_t t0a = smem_u32(tile);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int rr = 8 * (8 * c + 4 * hf + (lane >> 3)) + (lane & 7);
            uint32_t r4[4];
            ldmatrix_x4_trans(t0a + (uint32_t)swz(rr, byte0 >> 4), r4);
#pragma unroll
            for (int m = 0; m < 4; ++m) y[4 * hf + m] = r4[m];
          }
        } else {
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int rr = 8 * (8 * c + m) + (lane >> 2);
            y[m] = movmatrix_trans(lds_u32_a2(tile + rr * C::HALF + byte0 + 4 * (lane & 3)));
          }
        }
        // nibbles 0, 1 of each group (n 2^-24, n 2^-20) to lanes +0..15, then
        // nibbles 2, 3 to lanes +16..31: 16 live results at a time
        const uint32_t cbase = tm + lane_base + C::OFF_CP + cb * C::CP_CHUNK + h * 32;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            lo[4 * j + e] = y[2 * j + e] & 0x000F000Fu;
            lo[4 * j + 2 + e] = y[2 * j + e] & 0x00F000F0u;
          }
        }
        tmem_st_16x256b_x4(cbase, lo);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            lo[4 * j + e] = (y[2 * j + e] >> 8) & 0x000F000Fu;
            lo[4 * j + 2 + e] = (y[2 * j + e] >> 8) & 0x00F000F0u;
          }
        }
        tmem_st_16x256b_x4(cbase + (16u << 16), lo);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.empty[st]);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.cp_ready[cb]);
    }
    if (!ok && lane == 0) fail();
  } else if ((warp >= 8 && warp < 12) || warp >= 20) {
    // ------------------------------------------------------------ softmax
    // NSG groups of four warps (8-11, then 20-23, 24-27, ...); group hh owns
    // heads hh*HQ .. hh*HQ+HQ-1, warp q of a group TMEM lanes 32q .. 32q+31
    constexpr int HQ = C::HQ;
    const int q = warp & 3;
    const int hh = warp < 12 ? 0 : 1 + ((warp - 20) >> 2);  // head group
    const int h0 = hh * HQ;             // first head of this warp
    const int sw = 4 * hh + q;          // softmax warp index
    const int gtid = 32 * q + lane;     // thread index within the group
    const int barid = 1 + hh;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    if (gtid < HQ) {
      pdl_wait();  // corr comes from the query prologue kernel
      ms.sig[h0 + gtid] = p.corr[(size_t)b * 2 * NQ + h0 + gtid];
      ms.corr[h0 + gtid] = p.corr[(size_t)b * 2 * NQ + NQ + h0 + gtid];
      // a bad per-row length is reported once, after the prologue cleared the error word
      if (split == 0 && hh == 0 && gtid == 0) query_len(p.seq_lens, b, p.n_new, p.T, p.err, true);
    }
    named_bar(barid, 128);
    bool ok = true;
    // test-only stall: every softmax warp waits on a barrier that nothing
    // completes, so the bounded wait runs out and the failure path runs
    if (p.stall_ns != 0u && !wait_bar(&ms.never, 0, abort, p.stall_ns)) ok = false;
    float *cm = ms.cm[sw];  // -(score offset + running max m), per head (this warp's copy), negated
                            // so that the score FMA adds it
    float lsum[HQ];
    if (lane == 0)
      for (int n = 0; n < HQ; ++n) cm[n] = -ms.corr[h0 + n];  // provisional m = 0; the first tile rescales
    __syncwarp();
#pragma unroll
    for (int n = 0; n < HQ; ++n) lsum[n] = 0.f;
    // this thread's folded sums: slot k (ACC block k / 8, head k % 8), addressed on use
    auto fl_slot = [&](int k) -> float * {
      return reinterpret_cast<float *>(smem + C::SM_FL) + k * C::NSMX * 32 + sw * 32 + lane;
    };
    if constexpr (FOLD) {
#pragma unroll
      for (int k = 0; k < 16; ++k) *fl_slot(k) = 0.f;
    }
    const int r = 32 * q + lane;        // token row within the tile
    const int kap = kappa_of_token(r);  // its K position in the pooling operand
    // tiles i >= ilim hold this row past the split's end; only the last tile
    // can, when the range is not a whole number of tiles (-1: none)
    const int ilim = (int)min((int64_t)n_tiles, (t1 - t0 - r + kTile - 1) / kTile);
    const int last_ragged = ((t1 - t0) % kTile) != 0 ? n_tiles - 1 : -1;
    static_assert(HQ == 8, "softmax warps own eight heads");
    // x <- score - m of one tile from its raw S (a, b terms); rows past the
    // split's end (ragged last tile only) take no weight; returns the row max
    float sgr[HQ];  // the group's per-head scales, held for the whole split
#pragma unroll
    for (int n = 0; n < HQ; ++n) sgr[n] = ms.sig[h0 + n];
    auto scores = [&](int i, const uint32_t (&ra)[HQ], const uint32_t (&rb)[HQ], float (&x)[HQ]) -> float {
      const float4 *cm4 = reinterpret_cast<const float4 *>(cm);
      float lm = -INFINITY;
#pragma unroll
      for (int n4 = 0; n4 < HQ / 4; ++n4) {
        const float4 cc = cm4[n4];
        const float sv[4] = {sgr[4 * n4], sgr[4 * n4 + 1], sgr[4 * n4 + 2], sgr[4 * n4 + 3]};
        const float cv[4] = {cc.x, cc.y, cc.z, cc.w};
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          const int n = 4 * n4 + e;
          const int y0 = (int)ra[n] * 128 + (int)rb[n];  // exact: |y| < 2^27
          const int y1 = (int)ra[n + 1] * 128 + (int)rb[n + 1];
          // two heads per packed FMA (each element rounded once, as fmaf)
          const float2 xv = __ffma2_rn(make_float2((float)y0, (float)y1), make_float2(sv[e], sv[e + 1]),
                                       make_float2(cv[e], cv[e + 1]));
          x[n] = xv.x;
          x[n + 1] = xv.y;
          lm = fmax3f(lm, xv.x, xv.y);
        }
      }
      if (i == last_ragged && i >= ilim) {  // only the last tile of a ragged range has such rows
        lm = -INFINITY;
#pragma unroll
        for (int n = 0; n < HQ; ++n) x[n] = -INFINITY;
      }
      return lm;
    };
    // P row of this token (fp16) for this warp's heads into P buffer i % kPBufs, MN-major
    auto write_p = [&](int i, const float (&x)[HQ]) {
      uint8_t *prow = smem + C::SM_P + (i % kPBufs) * C::P_BYTES + (kap >> 3) * 128 + (kap & 7) * 16 +
                      (h0 / 8) * C::SBO_P;
      uint32_t h2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float p0 = ex2_approx(x[2 * k]), p1 = ex2_approx(x[2 * k + 1]);
        const __half2 hv = __floats2half2_rn(p0, p1);
        const float2 ls = __fadd2_rn(make_float2(lsum[2 * k], lsum[2 * k + 1]), make_float2(p0, p1));
        lsum[2 * k] = ls.x;
        lsum[2 * k + 1] = ls.y;
        h2[k] = *reinterpret_cast<const uint32_t *>(&hv);
      }
      *reinterpret_cast<uint4 *>(prow) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
    };
    // Tiles go in pairs (2j in S buffer 0, 2j+1 in S buffer 1): both tiles'
    // scores are loaded together and share one vote, one fence and one pass
    // through the loop.  P buffers stay per tile (the score MMA of tile i
    // waited for P buffer i % kPBufs to be free).
    // A wait that gives up does not end the loop: the warp records the failure
    // (and the abort flag) and keeps running the same instructions without
    // waiting, its data meaningless, so every warp of the group passes the same
    // named barriers; the group decides together after the loop.
    const int n_pairs = (n_tiles + 1) >> 1;
    for (int j = 0; j < n_pairs; ++j) {
      const int i0 = 2 * j;
      const bool two = i0 + 1 < n_tiles;
      const uint32_t par = (uint32_t)j & 1u;  // use j of each S buffer
      float x0[HQ], x1[HQ];
      float xmax;
      {  // tile 2j from S buffer 0, then tile 2j+1 from S buffer 1 (one buffer's raw terms live at a time)
        uint32_t ra[HQ], rb[HQ];
        if (ok && !wait_bar(&ms.s_full[0], par, abort, p.wait_ns)) {
          ok = false;
          fail();
        }
        tc_fence_after();
        tmem_ld8(tm + lane_base + C::OFF_S + h0, ra);
        tmem_ld8(tm + lane_base + C::OFF_S + NQ + h0, rb);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ms.s_free[0]);  // the next score MMA may overwrite it
        xmax = scores(i0, ra, rb, x0);
        if (two) {
          if (ok && !wait_bar(&ms.s_full[1], par, abort, p.wait_ns)) {
            ok = false;
            fail();
          }
          tc_fence_after();
          tmem_ld8(tm + lane_base + C::OFF_S + C::NS + h0, ra);
          tmem_ld8(tm + lane_base + C::OFF_S + C::NS + NQ + h0, rb);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ms.s_free[1]);
          xmax = fmaxf(xmax, scores(i0 + 1, ra, rb, x1));
        } else {
#pragma unroll
          for (int n = 0; n < HQ; ++n) x1[n] = -INFINITY;
        }
      }
      const bool need = (j == 0) || xmax > kTau;
      // one barrier over the group's four warps that also ORs their votes
      const bool any = named_bar_or(barid, 128, need);
      const bool flush = FOLD && (j > 0) && (i0 % kFlushTiles) == 0;  // the pooling MMAs restart at tile i0
      if (any || flush) {
        float *f = ms.fac[sw];
        if (any) {
          // raise the running max: m <- m + max(0, pair max of x) (the first pair: m <- its max)
#pragma unroll
          for (int n = 0; n < HQ; ++n) {
            float v = fmaxf(x0[n], x1[n]);
#pragma unroll
            for (int off = 16; off; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
            if (lane == 0) ms.red[q][h0 + n] = v;
          }
          named_bar(barid, 128);
#pragma unroll
          for (int n = 0; n < HQ; ++n) {
            const int hn = h0 + n;
            const float d = fmaxf(fmaxf(ms.red[0][hn], ms.red[1][hn]), fmaxf(ms.red[2][hn], ms.red[3][hn]));
            const float sh = (j == 0) ? d : fmaxf(d, 0.f);
            const float fn = (j == 0) ? 0.f : exp2f(-sh);
            x0[n] -= sh;
            x1[n] -= sh;
            lsum[n] *= fn;
            if (lane == 0) {
              f[n] = fn;
              cm[n] -= sh;
            }
          }
        } else if (lane == 0) {
#pragma unroll
          for (int n = 0; n < HQ; ++n) f[n] = 1.f;
        }
        __syncwarp();
        if (j > 0) {
          // ACC must hold every earlier tile before it is rescaled or folded
          const int pi = i0 - 1;
          if (ok && !wait_bar(&ms.p_free[pi % kPBufs], (uint32_t)(pi / kPBufs) & 1u, abort, p.wait_ns)) {
            ok = false;
            fail();
          }
          tc_fence_after();
#pragma unroll 1
          for (int blk = 0; blk < 2; ++blk) {  // both ACC blocks, this warp's head columns
            uint32_t a[HQ];
            const uint32_t ta = tm + lane_base + C::OFF_ACC + blk * NQ + h0;
            tmem_ld_hq<HQ>(ta, a);
            tmem_ld_wait();
            float *fl = fl_slot(blk * 8);
            if (flush) {
              // fold into this thread's fp32 sums (rescaled alike); tile i0's MMAs overwrite ACC
#pragma unroll
              for (int n = 0; n < HQ; ++n) fl[n * C::NSMX * 32] = (fl[n * C::NSMX * 32] + __uint_as_float(a[n])) * f[n];
            } else {
              // rescale: ACC and the sums folded out of earlier runs (relative to the same max)
#pragma unroll
              for (int n = 0; n < HQ; ++n) {
                a[n] = __float_as_uint(__uint_as_float(a[n]) * f[n]);
                if constexpr (FOLD) fl[n * C::NSMX * 32] *= f[n];
              }
              tmem_st_hq<HQ>(ta, a);
            }
          }
          if (!flush) tmem_st_wait();
        }
      }
      write_p(i0, x0);
      if (two) write_p(i0 + 1, x1);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ms.p_full[i0 % kPBufs]);
        if (two) mbar_arrive(&ms.p_full[(i0 + 1) % kPBufs]);
      }
    }
    // ------------------------------------------------------------ epilogue: ACC -> partials
    if (ok) ok = wait_bar(&ms.acc_full, 0, abort, p.wait_ns);
    if (named_bar_or(barid, 128, !ok)) {  // the group leaves together if any of its waits gave up
      if (lane == 0) fail();
    } else {
      tc_fence_after();
      // L = sum over the CTA's tokens of the softmax weights (fp32; the pooled
      // copies are their fp16 roundings, relative difference <= 2^-11 each)
#pragma unroll
      for (int n = 0; n < HQ; ++n) {
        float v = lsum[n];
#pragma unroll
        for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) ms.red[q][h0 + n] = v;
      }
      named_bar(barid, 128);
      if (gtid < HQ) {
        const int hn = h0 + gtid;
        ms.lt[hn] = (ms.red[0][hn] + ms.red[1][hn]) + (ms.red[2][hn] + ms.red[3][hn]);
        ms.m[hn] = -ms.cm[4 * hh][gtid] - ms.corr[hn];
      }
      named_bar(barid, 128);
      const float *Lt = ms.lt;
      float *out = p.part + (((size_t)b * p.S + split) * NQ) * (2 + G);
      if (gtid < HQ) {
        out[(size_t)(h0 + gtid) * (2 + G)] = ms.m[h0 + gtid];
        out[(size_t)(h0 + gtid) * (2 + G) + 1] = Lt[h0 + gtid];
      }
      // TMEM lane L of sub-partition q in half h holds coordinate
      // 128h + 32q + 8((L%8)/2) + 4(L%2) + L/8 (see the pooling dequant); the
      // pooled values are n 2^-24 (L/8 even) or n 2^-20 (L/8 odd), n = level + 8.
      // NH=1 keeps one ACC copy per 64-token chunk: add them.
      const int jn = lane >> 3, sl = lane & 7;
      const float vscale = (jn & 1) ? 1048576.f : 16777216.f;
      uint32_t a0[HQ], a1[HQ];
      tmem_ld_hq<HQ>(tm + lane_base + C::OFF_ACC + h0, a0);
      tmem_ld_hq<HQ>(tm + lane_base + C::OFF_ACC + NQ + h0, a1);
      tmem_ld_wait();
      if constexpr (FOLD) {
#pragma unroll
        for (int n = 0; n < HQ; ++n) {  // plus the sums folded out of earlier accumulation runs
          a0[n] = __float_as_uint(__uint_as_float(a0[n]) + *fl_slot(n));
          a1[n] = __float_as_uint(__uint_as_float(a1[n]) + *fl_slot(8 + n));
        }
      }
      if constexpr (C::NH == 2) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int g = 128 * h + 32 * q + 8 * (sl >> 1) + 4 * (sl & 1) + jn;
          if (g < G) {  // G < 256: the second half is partly padding
#pragma unroll
            for (int n = 0; n < HQ; ++n)
              out[(size_t)(h0 + n) * (2 + G) + 2 + g] =
                  fmaf(__uint_as_float(h ? a1[n] : a0[n]), vscale, -8.f * Lt[h0 + n]);
          }
        }
      } else {
        const int g = 32 * q + 8 * (sl >> 1) + 4 * (sl & 1) + jn;
        if (g < G) {
#pragma unroll
          for (int n = 0; n < HQ; ++n) {
            const float d = __uint_as_float(a0[n]) + __uint_as_float(a1[n]);
            out[(size_t)(h0 + n) * (2 + G) + 2 + g] = fmaf(d, vscale, -8.f * Lt[h0 + n]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- prologue
// Per (b, h): q'_g = c * sum_d W_k[j*d_h + d][g] q[b][h][d] (c = scale*log2 e),
// split into two int8 terms q'_g ~ sigma (128 a_g + b_g) with sigma =
// max_g |q'_g| / (127*128).  Written in the K-major no-swizzle layout of the
// score MMA's B operand: rows h (a terms) and NQ + h (b terms), K position
// kappa = 8w + 4e + i for coordinate 8w + 2i + e (the dequant's byte order).
// corr[b] = [sigma_h] then [sigma_h * 8 * sum_g (128 a_g + b_g)]: the score is
// sigma (128 S_a + S_b) - offset, the offset removing the +8 of the bytes.
// BYTE: the cache holds 256-level codes, one byte per coordinate i, read here
// as two nibbles (G = 2 x the latent width): with n = lo + 16 hi, the level
// n - 128 = (lo - 8) + 16 (hi - 8) + 8, so nibble 2i carries weight q'_i and
// nibble 2i+1 weight 16 q'_i; the constant 8 q'_i shifts every score of a head
// alike (the softmax ignores it) and the merge folds the pooled nibble pairs
// back (merge.cu).  W_k^(j) is then [D][G/2].
// Threads: KPAD coordinates x NDQ slices of the head dimension.  W_k^(j)
// is staged in shared memory by 16-byte asynchronous copies (requested before
// q, so the two latencies overlap); thread (dq, g) sums its slice of the head
// dimension for coordinate g, and after one exchange of the slices' sums
// slice dq finishes heads dq, dq + NDQ, ... (scale, split into two int8 terms).
template <int GRP>
struct AbsorbShape {
  static constexpr int NDQ = GRP <= 4 ? 4 : (GRP == 8 ? 2 : 1);
};
template <int G, int NQ, int GRP, bool BYTE>
struct AbsorbSmem {
  static constexpr int GS = Cfg<G, NQ>::KPAD;
  static constexpr int NDQ = AbsorbShape<GRP>::NDQ;
  static constexpr int GW = BYTE ? G / 2 : G;                    // columns of W_k^(j)
  static constexpr int W_BYTES = FSQ_HEAD_DIM * GW * 2;         // W_k^(j), bf16 [D][GW]
  static constexpr int PART_OFF = (W_BYTES + 15) / 16 * 16;
  static constexpr int BYTES = PART_OFF + NDQ * GRP * GS * 4;  // slice sums, fp32 [NDQ][GRP][GS]
};

__device__ __forceinline__ void cp_async16_g2s(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}

template <int G, int NQ, int GRP, bool BYTE>
__global__ void __launch_bounds__(Cfg<G, NQ>::KPAD * AbsorbShape<GRP>::NDQ)
    absorb_query_tc(const uint16_t *__restrict__ q, const uint16_t *__restrict__ W_kv, float c,
                    uint8_t *__restrict__ qphys, float *__restrict__ corr, uint32_t *err, MergeScratch ms) {
  // one CTA per (kv head j, batch row b): the group's heads share W_k^(j), read once
  using C = Cfg<G, NQ>;
  using SM = AbsorbSmem<G, NQ, GRP, BYTE>;
  constexpr int GW = SM::GW;
  constexpr int D = FSQ_HEAD_DIM;
  constexpr int NDQ = SM::NDQ;
  constexpr int GS = SM::GS;        // threads per slice (one per padded coordinate)
  constexpr int DS = D / NDQ;       // head-dimension rows per thread
  constexpr int NW = GS / 32;       // warps per slice
  constexpr int NT = GS * NDQ;
  extern __shared__ __align__(16) uint8_t asmem[];
  const uint16_t *wks = reinterpret_cast<const uint16_t *>(asmem);
  float *part = reinterpret_cast<float *>(asmem + SM::PART_OFF);
  __shared__ __align__(16) float qs[GRP][D];  // read as float4
  __shared__ float red[GRP][NW];
  __shared__ int ired[GRP][NW];
  __shared__ float sig_s[GRP], inv_s[GRP];
  const int j = blockIdx.x, b = blockIdx.y;
  const int g = threadIdx.x % GS, dq = threadIdx.x / GS;
  const int wis = g >> 5, lane = threadIdx.x & 31;  // warp within the slice
  // Nothing here depends on the kernel before this one (q and W_kv are inputs
  // of the call; no kernel of this library that may still run writes them,
  // and the workspace is no longer read by the previous call's kernels, which
  // have completed), so the whole prologue overlaps with it - with the append
  // of the step's new tokens in a decode step.  It waits for that kernel only
  // at the end, before releasing the split kernel, whose first code loads
  // precede its own wait.
  {
    const uint8_t *src = reinterpret_cast<const uint8_t *>(W_kv + (int64_t)j * D * GW);
    for (int k = threadIdx.x; k < SM::W_BYTES / 16; k += NT) cp_async16_g2s(asmem + 16 * k, src + 16 * k);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  if (j == 0 && b == 0) {
    if (threadIdx.x == 0) *err = 0u;
    for (int i = threadIdx.x; i < ms.ncnt; i += NT) ms.cnt[i] = 0u;  // the merge's arrival counts
  }
  for (int i = threadIdx.x; i < GRP * D; i += NT)
    qs[i / D][i % D] = bf16_to_f32(q[((int64_t)b * NQ + j * GRP) * D + i]);
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  float v[GRP];
#pragma unroll
  for (int hh = 0; hh < GRP; ++hh) v[hh] = 0.f;
  if (g < G) {
    const uint16_t *wk = wks + (dq * DS) * GW + (BYTE ? g >> 1 : g);
#pragma unroll 8
    for (int u = 0; u < DS; u += 4) {
      const float w0 = bf16_to_f32(wk[(u + 0) * GW]), w1 = bf16_to_f32(wk[(u + 1) * GW]);
      const float w2 = bf16_to_f32(wk[(u + 2) * GW]), w3 = bf16_to_f32(wk[(u + 3) * GW]);
#pragma unroll
      for (int hh = 0; hh < GRP; ++hh) {
        const float4 qv = *reinterpret_cast<const float4 *>(&qs[hh][dq * DS + u]);
        v[hh] = fmaf(w0, qv.x, fmaf(w1, qv.y, fmaf(w2, qv.z, fmaf(w3, qv.w, v[hh]))));
      }
    }
  }
#pragma unroll
  for (int hh = 0; hh < GRP; ++hh) part[(dq * GRP + hh) * GS + g] = v[hh];
  __syncthreads();
  // slice dq finishes heads dq, dq + NDQ, ...
  constexpr int HPS = (GRP + NDQ - 1) / NDQ;  // heads per slice
  const float cg = (BYTE && (g & 1)) ? 16.f * c : c;  // the high nibble of a byte code weighs 16
  float vf[HPS];
#pragma unroll
  for (int k = 0; k < HPS; ++k) {
    const int hh = dq + k * NDQ;
    float t = 0.f;
    if (hh < GRP) {
#pragma unroll
      for (int i = 0; i < NDQ; ++i) t += part[(i * GRP + hh) * GS + g];
    }
    vf[k] = t * cg;
    float am = fabsf(vf[k]);
#pragma unroll
    for (int o = 16; o; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    if (lane == 0 && hh < GRP) red[hh][wis] = am;
  }
  __syncthreads();
  if (threadIdx.x < GRP) {
    float am = 0.f;
    for (int i = 0; i < NW; ++i) am = fmaxf(am, red[threadIdx.x][i]);
    const float sg = am > 0.f ? am / (127.f * 128.f) : 1.f;
    sig_s[threadIdx.x] = sg;
    inv_s[threadIdx.x] = 1.f / sg;
  }
  __syncthreads();
  // coordinate g = 8w + 2i + e sits at K position kappa = 8w + 4e + i
  const int kap = (g & ~7) | ((g & 1) << 2) | ((g >> 1) & 3);
  uint8_t *dst = qphys + (size_t)b * C::Q_BYTES;
  const int base = (kap >> 4) * C::LBO_Q + (kap & 15);
#pragma unroll
  for (int k = 0; k < HPS; ++k) {
    const int hh = dq + k * NDQ;
    if (hh >= GRP) break;
    const int h = j * GRP + hh;
    const float t = vf[k] * inv_s[hh];
    const int a = max(-127, min(127, __float2int_rn(t * (1.f / 128.f))));
    const int bt = max(-127, min(127, __float2int_rn(t - 128.f * (float)a)));
    int isum = 128 * a + bt;
    dst[base + (h >> 3) * 128 + (h & 7) * 16] = (uint8_t)(int8_t)a;
    dst[base + ((NQ + h) >> 3) * 128 + ((NQ + h) & 7) * 16] = (uint8_t)(int8_t)bt;
#pragma unroll
    for (int o = 16; o; o >>= 1) isum += __shfl_xor_sync(0xffffffffu, isum, o);
    if (lane == 0) ired[hh][wis] = isum;
  }
  __syncthreads();
  if (threadIdx.x < GRP) {
    long long tot = 0;
    for (int i = 0; i < NW; ++i) tot += ired[threadIdx.x][i];
    const int h = j * GRP + threadIdx.x;
    corr[(size_t)b * 2 * NQ + h] = sig_s[threadIdx.x];
    corr[(size_t)b * 2 * NQ + NQ + h] = (float)((double)sig_s[threadIdx.x] * 8.0 * (double)tot);
  }
  pdl_wait();
  pdl_trigger();  // the split kernel may start its prologue and code loads
}

template <int G, int NQ, int GRP, bool BYTE>
cudaError_t absorb_query_launch(const dim3 &grid, const uint16_t *q, const uint16_t *W_kv, float c, uint8_t *qphys,
                                float *corr, uint32_t *err, MergeScratch ms, cudaStream_t st) {
  using SM = AbsorbSmem<G, NQ, GRP, BYTE>;
  cudaError_t e = ensure_smem_limit((const void *)absorb_query_tc<G, NQ, GRP, BYTE>, (size_t)SM::BYTES);
  if (e != cudaSuccess) return e;
  return launch_pdl(absorb_query_tc<G, NQ, GRP, BYTE>, grid, dim3(Cfg<G, NQ>::KPAD * AbsorbShape<GRP>::NDQ),
                    (size_t)SM::BYTES, st, q, W_kv, c, qphys, corr, err, ms);
}

template <int G, int NQ, bool BYTE>
cudaError_t launch_absorb_query(const uint16_t *q, int64_t B, int n_kv, const uint16_t *W_kv, float c,
                                uint8_t *qphys, float *corr, uint32_t *err, MergeScratch ms, cudaStream_t st) {
  const dim3 grid(n_kv, (unsigned)B);
  switch (NQ / n_kv) {
    case 1: return absorb_query_launch<G, NQ, 1, BYTE>(grid, q, W_kv, c, qphys, corr, err, ms, st);
    case 2: return absorb_query_launch<G, NQ, 2, BYTE>(grid, q, W_kv, c, qphys, corr, err, ms, st);
    case 4: return absorb_query_launch<G, NQ, 4, BYTE>(grid, q, W_kv, c, qphys, corr, err, ms, st);
    case 8: return absorb_query_launch<G, NQ, 8, BYTE>(grid, q, W_kv, c, qphys, corr, err, ms, st);
    case 16: return absorb_query_launch<G, NQ, 16, BYTE>(grid, q, W_kv, c, qphys, corr, err, ms, st);
    default: return cudaErrorInvalidValue;
  }
}

// Tensor map of the code cache as a 3-D byte tensor [B][T][row bytes]: the
// box is one 128-row tile of one batch row, swizzled 128 B.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

cudaError_t make_code_tensor_map(CUtensorMap *map, const uint8_t *codes, int64_t bstride, int64_t T, int64_t B,
                                 int row_bytes) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  if (T > 0x7fffffffLL || B > 0x7fffffffLL) return cudaErrorInvalidValue;
  const cuuint64_t dims[3] = {(cuuint64_t)row_bytes, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)bstride};
  const cuuint32_t box[3] = {(cuuint32_t)row_bytes, (cuuint32_t)kTile, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(codes), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int G, int NQ, bool BYTE>
cudaError_t launch(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int n_new, int64_t T,
                   const int32_t *seq_lens, int n_kv, const uint16_t *W_kv, float scale, int S, int64_t tps,
                   uint8_t *qphys, float *corr, float *part, uint32_t *err, MergeScratch ms, uint32_t stall_ns,
                   void *const *prof, cudaStream_t st) {
  using C = Cfg<G, NQ>;
  cudaError_t e = launch_absorb_query<G, NQ, BYTE>(q, B, n_kv, W_kv, scale * kLog2e, qphys, corr, err, ms, st);
  if (e != cudaSuccess) return e;
  // one CTA per SM: ask for more shared memory than two CTAs could share
  const int smem = C::SM_TOTAL > 120 * 1024 ? C::SM_TOTAL : 120 * 1024;
  const bool fold = tps > kFoldAbove;  // long splits keep their accumulation runs short
  auto kern = fold ? absorbed_split_tc<G, NQ, true> : absorbed_split_tc<G, NQ, false>;
  e = ensure_smem_limit((const void *)kern, (size_t)smem);
  if (e != cudaSuccess) return e;
  Params p{codes, bstride, T, tps, S, qphys, corr, part, err, kWaitLimitNs, seq_lens, stall_ns, n_new};
  CUtensorMap tmap;
  memset(&tmap, 0, sizeof(tmap));
  if constexpr (C::TMA) {
    e = make_code_tensor_map(&tmap, codes, bstride, T, B / n_new, C::HALF);
    if (e != cudaSuccess) return e;
  }
  record_prof_event(prof[0], st);
  e = launch_pdl(kern, dim3(S, (unsigned)B), dim3(C::THREADS), (size_t)smem, st, tmap, p);
  record_prof_event(prof[1], st);
  return e;
}

}  // namespace tc

// Width of the nibble rows the split kernel reads: G at 16 levels; 2G at 256
// levels (each 8-bit code read as two nibbles); 0 when the kernel does not
// cover the shape.
int absorbed_tc_width(int n_q, int n_kv, int G, int levels) {
  const int Gn = levels == 16 ? G : (levels == 256 ? 2 * G : 0);
  const bool ok = (n_q == 16 || n_q == 32) && (Gn == 256 || Gn == 160 || Gn == 84) && n_kv > 0 && n_q % n_kv == 0 &&
                  n_q / n_kv <= 16;
  return ok ? Gn : 0;
}

size_t absorbed_tc_qphys_bytes(int n_q, int G) {
  const int kpad = (G + 31) / 32 * 32;
  return (size_t)2 * n_q * kpad;
}

cudaError_t merge_absorbed_launch(const float *part, int S, int64_t B, int n_q, int n_kv, int d_h, int G,
                                  const uint16_t *W_kv, void *o, int out_fp32, MergeScratch ms, cudaStream_t st,
                                  int fold_bytes);

// G: the latent width of the cache (levels 16 or 256); the partials carry
// absorbed_tc_width(...) nibble coordinates, folded back by the merge.
// B: grid rows (cache rows x n_new queries).
cudaError_t launch_absorbed_tc(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int n_new,
                               int64_t T, const int32_t *seq_lens, int n_q, int n_kv, int d_h, int G, int levels,
                               const uint16_t *W_kv, float scale, int S, int64_t tps, uint8_t *qphys, float *corr,
                               float *part, uint32_t *err, MergeScratch ms, void *o, int out_fp32,
                               uint32_t stall_ns, void *const *prof, cudaStream_t st) {
  const int Gn = absorbed_tc_width(n_q, n_kv, G, levels);
  const bool byte = levels == 256;
  cudaError_t e = cudaErrorInvalidValue;
#define FSQ_TC_LAUNCH(GG, NN, BB)                                                                                  \
  tc::launch<GG, NN, BB>(q, codes, bstride, B, n_new, T, seq_lens, n_kv, W_kv, scale, S, tps, qphys, corr, part, \
                         err, ms, stall_ns, prof, st)
#define FSQ_TC_CASE(GG)                                                       \
  if (Gn == GG && n_q == 32) e = byte ? FSQ_TC_LAUNCH(GG, 32, true) : FSQ_TC_LAUNCH(GG, 32, false); \
  else if (Gn == GG && n_q == 16) e = byte ? FSQ_TC_LAUNCH(GG, 16, true) : FSQ_TC_LAUNCH(GG, 16, false);
  FSQ_TC_CASE(256)
  else FSQ_TC_CASE(160)
  else FSQ_TC_CASE(84)
  else return cudaErrorInvalidValue;
#undef FSQ_TC_CASE
#undef FSQ_TC_LAUNCH
  if (e != cudaSuccess) return e;
  return merge_absorbed_launch(part, S, B, n_q, n_kv, d_h, Gn, W_kv, o, out_fp32, ms, st, byte ? 1 : 0);
}

}  // namespace fsq
