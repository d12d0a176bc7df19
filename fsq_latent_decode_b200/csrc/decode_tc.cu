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
//   -> dequant warps unpack nibbles in registers straight into two TMEM
//      operand layouts: token-major Z (A of the score MMA) and, through 8x8
//      register transposes, coordinate-major Z^T (A of the pooling MMA)
//   -> one thread issues both MMAs (A from TMEM, B from shared memory)
//   -> softmax warps read S from TMEM, keep the running max, write P (fp16)
//      to shared memory, rescale ACC in TMEM when the max grows.
//
// Nibbles are turned into fp16 without a per-value subtract.  Score operand:
// one LOP3 per pair ORs the nibble into the bit pattern of 1024.0, giving
// 1024 + n exactly (ulp 1), or 1024 + 16 n for the high nibble of a byte; the
// constant and the factor 1 or 16 are folded into Q' and a per-head score
// offset.  Pooling operand: a shift and a LOP3 per pair give 16 + n; ACC is
// corrected by 24 l per head at the end (16 for the bias, 8 for the level
// offset), keeping the long fp32 accumulation well conditioned.
//
// Warp roles (12 warps): 0 loads code tiles and owns TMEM, 1 issues MMAs,
// 2-3 stage Q' once, 4-7 dequantise (TMEM sub-partitions 0-3), 8-11 softmax.
// Every wait is bounded; on a timeout the CTA records FSQ_ERR_TIMEOUT in the
// workspace error word and all roles drain and exit.
#include "common.cuh"
#include "tc_ptx.cuh"

namespace fsq {
namespace tc {

using namespace ptx;

constexpr int kTile = 128;
constexpr int kStages = 4;
constexpr float kTau = 8.f;                  // rescale when a score exceeds the running max by 2^8
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait

template <int G, int NQ>
struct Cfg {
  static constexpr int HALF = G / 2;                 // bytes per token row
  static constexpr int KPAD = (G + 15) / 16 * 16;    // K of the score MMA
  static constexpr int KW = KPAD / 8;                // 32-bit code words (8 coordinates) per padded row
  static constexpr int SCOLS = KPAD / 2;             // TMEM columns of token-major Z
  static constexpr int NH = (G + 127) / 128;         // 128-row halves of the pooling MMA
  static constexpr int TILE_BYTES = kTile * HALF;
  static constexpr int STAGE_BYTES = (TILE_BYTES + 16 + 127) / 128 * 128;  // + over-read pad
  static constexpr int Q_BYTES = NQ * KPAD * 2;      // Q' in the K-major no-swizzle layout
  static constexpr int P_BYTES = kTile * NQ * 2;     // P in the MN-major no-swizzle layout
  // TMEM columns
  static constexpr int OFF_CS = 0;
  static constexpr int OFF_CP = (SCOLS + 15) / 16 * 16;
  static constexpr int CP_BUF = NH * 64;
  static constexpr int OFF_S = OFF_CP + 2 * CP_BUF;
  static constexpr int OFF_ACC = OFF_S + 2 * NQ;
  static constexpr int TMEM_USED = OFF_ACC + NH * NQ;
  static constexpr int TMEM_COLS = 512;
  static_assert(TMEM_USED <= 512, "TMEM plan exceeds 512 columns");
  // shared memory
  static constexpr int SM_CODES = 0;
  static constexpr int SM_Q = SM_CODES + kStages * STAGE_BYTES;
  static constexpr int SM_P = SM_Q + Q_BYTES;
  static constexpr int SM_MISC = SM_P + 2 * P_BYTES;
  static constexpr int SM_TOTAL = SM_MISC + 2048;
  static constexpr int LBO_Q = (NQ / 8) * 128;       // K-chunk stride of Q'
  static constexpr int SBO_P = (kTile / 8) * 128;    // N-group stride of P
};

struct Params {
  const uint8_t *codes;
  int64_t bstride;
  int64_t T;
  int64_t tps;
  int S;
  const uint8_t *qphys;  // per batch row: Q' bytes in the shared-memory layout
  const float *corr;     // per batch row: [NQ] score offsets
  float *part;           // [B][S][NQ][2 + G]
  uint32_t *err;
  uint64_t wait_ns;
};

struct Misc {
  uint64_t full[kStages], empty[kStages];
  uint64_t cs_ready, cs_free;
  uint64_t cp_ready[2], cp_free[2];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], p_free[2];
  uint64_t acc_full, q_full, mma_done;
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t vote[4];
  float red[4][64];
  float fac[4][64];
  float corr[64];
};

__device__ __forceinline__ uint32_t lop_lo(uint32_t w) { return (w & 0x000F000Fu) | 0x64006400u; }
__device__ __forceinline__ uint32_t lop_hi(uint32_t w) { return (w & 0x00F000F0u) | 0x64006400u; }
// Nibble j (bits 4j..4j+3) of both half-words moved to mantissa bits 6..9 of
// the pattern of 16.0: the fp16 pair (16 + n_lo, 16 + n_hi), exact.  Used for
// the pooling operand, whose fp32 accumulator runs over a whole split: a bias
// of 16 keeps its cancellation (acc = D - 24 l) small.
template <int J>
__device__ __forceinline__ uint32_t nib16(uint32_t w) {
  const uint32_t x = (J == 0) ? (w << 6) : (J == 1) ? (w << 2) : (J == 2) ? (w >> 2) : (w >> 6);
  return (x & 0x03C003C0u) | 0x4C004C00u;
}

// Physical K position of token r in the pooling operand (see the 16x256b store below).
__device__ __forceinline__ int kappa_of_token(int r) {
  return (r & ~15) | (((r >> 1) & 3) << 2) | (((r >> 3) & 1) << 1) | (r & 1);
}

// 32-bit little-endian load from a 2-byte aligned shared address
__device__ __forceinline__ uint32_t lds_u32_a2(const uint8_t *p) {
  const uint16_t *h = reinterpret_cast<const uint16_t *>(p);
  return (uint32_t)h[0] | ((uint32_t)h[1] << 16);
}

template <int G, int NQ>
__global__ void __launch_bounds__(384, 1) absorbed_split_tc(Params p) {
  using C = Cfg<G, NQ>;
  extern __shared__ __align__(1024) uint8_t smem[];
  Misc &ms = *reinterpret_cast<Misc *>(smem + C::SM_MISC);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, b = blockIdx.y;
  const int64_t t0 = (int64_t)split * p.tps;
  const int64_t t1 = min(p.T, t0 + p.tps);
  const int n_tiles = (int)((t1 - t0 + kTile - 1) / kTile);
  const uint8_t *gcodes = p.codes + (int64_t)b * p.bstride + t0 * C::HALF;
  volatile uint32_t *abort = &ms.abort;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ms.full[s], 1);
      mbar_init(&ms.empty[s], 4);
    }
    mbar_init(&ms.cs_ready, 4);
    mbar_init(&ms.cs_free, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ms.cp_ready[i], 4);
      mbar_init(&ms.cp_free[i], 1);
      mbar_init(&ms.s_full[i], 1);
      mbar_init(&ms.s_free[i], 4);
      mbar_init(&ms.p_full[i], 4);
      mbar_init(&ms.p_free[i], 1);
    }
    mbar_init(&ms.acc_full, 1);
    mbar_init(&ms.q_full, 1);
    mbar_init(&ms.mma_done, 1);
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

  auto fail = [&]() {
    record_error(p.err, FSQ_ERR_TIMEOUT);
    *abort = 1u;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint8_t *ring = smem + C::SM_CODES;
    if (lane == 0) {
      mbar_arrive_expect_tx(&ms.q_full, C::Q_BYTES);
      bulk_g2s(smem + C::SM_Q, p.qphys + (size_t)b * C::Q_BYTES, C::Q_BYTES, &ms.q_full);
    }
    int issued_phase[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) issued_phase[s] = -1;
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int st = i % kStages;
      const uint32_t ph = (uint32_t)(i / kStages) & 1u;
      if (!mbar_wait(&ms.empty[st], ph ^ 1u, abort, p.wait_ns)) {
        if (lane == 0) fail();
        ok = false;
        break;
      }
      const int64_t rows = min((int64_t)kTile, t1 - (t0 + (int64_t)i * kTile));
      uint8_t *dst = ring + st * C::STAGE_BYTES;
      const uint8_t *src = gcodes + (int64_t)i * kTile * C::HALF;
      if (rows == kTile) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&ms.full[st], C::TILE_BYTES);
          bulk_g2s(dst, src, C::TILE_BYTES, &ms.full[st]);
        }
      } else {
        // ragged tail: plain bounded loads, zero fill
        const int nb = (int)rows * C::HALF;
        for (int k = lane; k < C::STAGE_BYTES; k += 32) dst[k] = (k < nb) ? src[k] : (uint8_t)0;
        __syncwarp();
        if (lane == 0) mbar_arrive(&ms.full[st]);
      }
      issued_phase[st] = (int)ph;
    }
    if (!ok) {
      // let copies already in flight land before the CTA exits
      for (int s = 0; s < kStages; ++s)
        if (issued_phase[s] >= 0) mbar_wait(&ms.full[s], (uint32_t)issued_phase[s], abort, p.wait_ns / 4 + 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_f16(128, NQ, 0, 0);
      const uint32_t id_p = idesc_f16(128, NQ, 0, 1);
      const uint32_t qs = smem_u32(smem + C::SM_Q);
      const uint32_t pbase = smem_u32(smem + C::SM_P);
      bool ok = mbar_wait(&ms.q_full, 0, abort, p.wait_ns);
      auto pool = [&](int j) -> bool {
        const int pb = j & 1;
        const uint32_t par = (uint32_t)(j >> 1) & 1u;
        if (!mbar_wait(&ms.p_full[pb], par, abort, p.wait_ns)) return false;
        if (!mbar_wait(&ms.cp_ready[pb], par, abort, p.wait_ns)) return false;
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < C::NH; ++h) {
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint64_t bd = smem_desc(pbase + pb * C::P_BYTES + kk * 256, 128, C::SBO_P);
            mma_ts(tm + C::OFF_ACC + h * NQ, tm + C::OFF_CP + pb * C::CP_BUF + h * 64 + kk * 8, bd, id_p,
                   (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc_commit(&ms.p_free[pb]);
        tc_commit(&ms.cp_free[pb]);
        return true;
      };
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int sb = i & 1;
        ok = mbar_wait(&ms.cs_ready, (uint32_t)i & 1u, abort, p.wait_ns) &&
             mbar_wait(&ms.s_free[sb], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < C::KPAD / 16; ++k) {
          const uint64_t bd = smem_desc(qs + k * 2 * C::LBO_Q, C::LBO_Q, 128);
          mma_ts(tm + C::OFF_S + sb * NQ, tm + C::OFF_CS + k * 8, bd, id_s, k > 0 ? 1u : 0u);
        }
        tc_commit(&ms.s_full[sb]);
        tc_commit(&ms.cs_free);
        if (i > 0) ok = pool(i - 1);
      }
      if (ok && n_tiles > 0) ok = pool(n_tiles - 1);
      if (ok) tc_commit(&ms.acc_full);
      else fail();
      // every MMA issued by this thread has completed once mma_done flips
      tc_commit(&ms.mma_done);
      mbar_wait(&ms.mma_done, 0, abort, p.wait_ns);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ dequant
    const int q = warp - 4;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int st = i % kStages;
      const uint8_t *tile = smem + C::SM_CODES + st * C::STAGE_BYTES;
      if (!mbar_wait(&ms.full[st], (uint32_t)(i / kStages) & 1u, abort, p.wait_ns)) { ok = false; break; }
      // token-major Z: this thread's token row -> TMEM lane (32q + lane)
      if (!mbar_wait(&ms.cs_free, ((uint32_t)i & 1u) ^ 1u, abort, p.wait_ns)) { ok = false; break; }
      tc_fence_after();
      {
        const uint8_t *row = tile + (32 * q + lane) * C::HALF;
        uint32_t w[C::KW];
        if constexpr (G == 256) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            uint4 v = *reinterpret_cast<const uint4 *>(row + 16 * k);
            w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int k = 0; k < C::KW; ++k) {
            if (4 * k + 4 <= C::HALF) w[k] = lds_u32_a2(row + 4 * k);
            else if (4 * k + 2 <= C::HALF) w[k] = *reinterpret_cast<const uint16_t *>(row + 4 * k);
            else w[k] = 0u;
          }
        }
        constexpr int CH = 8;  // words per TMEM store (32 columns)
#pragma unroll
        for (int c0 = 0; c0 < C::KW; c0 += CH) {
          uint32_t r[32];
          const int nw = (C::KW - c0) < CH ? (C::KW - c0) : CH;
#pragma unroll
          for (int k = 0; k < CH; ++k) {
            if (k < nw) {
              const uint32_t x = w[c0 + k], x8 = x >> 8;
              r[4 * k + 0] = lop_lo(x);
              r[4 * k + 1] = lop_hi(x);
              r[4 * k + 2] = lop_lo(x8);
              r[4 * k + 3] = lop_hi(x8);
            }
          }
          const uint32_t ta = tm + lane_base + C::OFF_CS + 4 * c0;
          if (nw == 8) tmem_st32(ta, r);
          else if (nw == 4) tmem_st16(ta, r);
          else if (nw == 2) tmem_st8(ta, r);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.cs_ready);
      // coordinate-major Z^T via 8x8 transposes -> TMEM lanes = coordinates
      const int pb = i & 1;
      if (!mbar_wait(&ms.cp_free[pb], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort, p.wait_ns)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < C::NH; ++h) {
        const int byte0 = 64 * h + 16 * q;  // first byte of this warp's 32 coordinates
        if (byte0 < C::HALF) {
          const uint32_t cbase = tm + lane_base + C::OFF_CP + pb * C::CP_BUF + h * 64;
#pragma unroll 2
          for (int j = 0; j < kTile / 16; ++j) {
            uint32_t t[2][4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int tb = 2 * j + e;
              const uint8_t *src = tile + (8 * tb + (lane >> 2)) * C::HALF + byte0 + 4 * (lane & 3);
              uint32_t x;
              if constexpr (G == 256) x = *reinterpret_cast<const uint32_t *>(src);
              else x = lds_u32_a2(src);
              t[e][0] = movmatrix_trans(nib16<0>(x));
              t[e][1] = movmatrix_trans(nib16<1>(x));
              t[e][2] = movmatrix_trans(nib16<2>(x));
              t[e][3] = movmatrix_trans(nib16<3>(x));
            }
            tmem_st_16x256b(cbase + 8 * j, t[0][0], t[1][0], t[0][1], t[1][1]);
            tmem_st_16x256b(cbase + (16u << 16) + 8 * j, t[0][2], t[1][2], t[0][3], t[1][3]);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ms.cp_ready[pb]);
        mbar_arrive(&ms.empty[st]);
      }
    }
    if (!ok && lane == 0) fail();
  } else if (warp >= 8) {
    // ------------------------------------------------------------ softmax
    const int q = warp - 8;
    const int stid = tid - 256;  // 0..127
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    for (int n = stid; n < NQ; n += 128) ms.corr[n] = p.corr[(size_t)b * NQ + n];
    named_bar(1, 128);
    float m[NQ], lsum[NQ];
#pragma unroll
    for (int n = 0; n < NQ; ++n) {
      m[n] = -INFINITY;
      lsum[n] = 0.f;
    }
    const int r = 32 * q + lane;                  // token row within the tile
    const int kap = kappa_of_token(r);            // its K position in the pooling operand
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int sb = i & 1;
      const uint32_t par = (uint32_t)(i >> 1) & 1u;
      if (!mbar_wait(&ms.s_full[sb], par, abort, p.wait_ns)) { ok = false; break; }
      tc_fence_after();
      uint32_t raw[NQ];
      if constexpr (NQ == 32) tmem_ld32(tm + lane_base + C::OFF_S + sb * NQ, raw);
      else tmem_ld16(tm + lane_base + C::OFF_S + sb * NQ, raw);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.s_free[sb]);
      const bool valid = (t0 + (int64_t)i * kTile + r) < t1;
      float *s = reinterpret_cast<float *>(raw);  // scores in place of the raw MMA values
      bool need = false;
#pragma unroll
      for (int n = 0; n < NQ; ++n) {
        s[n] = valid ? (__uint_as_float(raw[n]) - ms.corr[n]) : -INFINITY;
        need |= s[n] > m[n] + kTau;
      }
      const bool wneed = __any_sync(0xffffffffu, need);
      if (lane == 0) ms.vote[q] = wneed ? 1u : 0u;
      named_bar(1, 128);
      const bool any = (ms.vote[0] | ms.vote[1] | ms.vote[2] | ms.vote[3]) != 0u;
      named_bar(1, 128);
      if (any) {
#pragma unroll
        for (int n = 0; n < NQ; ++n) {
          float v = s[n];
#pragma unroll
          for (int off = 16; off; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
          if (lane == 0) ms.red[q][n] = v;
        }
        named_bar(1, 128);
        float *f = ms.fac[q];  // this warp's copy of the rescale factors
#pragma unroll
        for (int n = 0; n < NQ; ++n) {
          const float mt = fmaxf(fmaxf(ms.red[0][n], ms.red[1][n]), fmaxf(ms.red[2][n], ms.red[3][n]));
          const float mn = fmaxf(m[n], mt);
          const float fn = exp2f(m[n] - mn);  // 0 on the first tile
          m[n] = mn;
          lsum[n] *= fn;
          if (lane == 0) f[n] = fn;
        }
        named_bar(1, 128);
        if (i > 0) {
          // ACC must hold every earlier tile before it is rescaled
          const int pj = (i - 1) & 1;
          if (!mbar_wait(&ms.p_free[pj], (uint32_t)((i - 1) >> 1) & 1u, abort, p.wait_ns)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < C::NH; ++h) {
            uint32_t a[NQ];
            const uint32_t ta = tm + lane_base + C::OFF_ACC + h * NQ;
            if constexpr (NQ == 32) tmem_ld32(ta, a);
            else tmem_ld16(ta, a);
            tmem_ld_wait();
#pragma unroll
            for (int n = 0; n < NQ; ++n) a[n] = __float_as_uint(__uint_as_float(a[n]) * f[n]);
            if constexpr (NQ == 32) tmem_st32(ta, a);
            else tmem_st16(ta, a);
          }
          tmem_st_wait();
        }
      }
      // P row of this token (fp16), MN-major: 4 chunks of 8 heads
      const int pb = i & 1;
      if (!mbar_wait(&ms.p_free[pb], par ^ 1u, abort, p.wait_ns)) { ok = false; break; }
      uint8_t *prow = smem + C::SM_P + pb * C::P_BYTES + (kap >> 3) * 128 + (kap & 7) * 16;
#pragma unroll
      for (int g8 = 0; g8 < NQ / 8; ++g8) {
        uint32_t h2[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float p0 = exp2f(s[8 * g8 + 2 * k] - m[8 * g8 + 2 * k]);
          const float p1 = exp2f(s[8 * g8 + 2 * k + 1] - m[8 * g8 + 2 * k + 1]);
          const __half2 hv = __floats2half2_rn(p0, p1);
          const float2 back = __half22float2(hv);
          lsum[8 * g8 + 2 * k] += back.x;
          lsum[8 * g8 + 2 * k + 1] += back.y;
          h2[k] = *reinterpret_cast<const uint32_t *>(&hv);
        }
        *reinterpret_cast<uint4 *>(prow + g8 * C::SBO_P) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.p_full[pb]);
    }
    // ------------------------------------------------------------ epilogue: ACC -> partials
    if (ok) ok = mbar_wait(&ms.acc_full, 0, abort, p.wait_ns);
    if (!ok) {
      if (lane == 0) fail();
    } else {
      tc_fence_after();
      // L~ = sum over the CTA's tokens of the fp16 weights actually pooled
#pragma unroll
      for (int n = 0; n < NQ; ++n) {
        float v = lsum[n];
#pragma unroll
        for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) ms.red[q][n] = v;
      }
      named_bar(1, 128);
      if (stid < NQ) ms.fac[0][stid] = (ms.red[0][stid] + ms.red[1][stid]) + (ms.red[2][stid] + ms.red[3][stid]);
      named_bar(1, 128);
      const float *Lt = ms.fac[0];
      float *out = p.part + (((size_t)b * p.S + split) * NQ) * (2 + G);
#pragma unroll
      for (int n = 0; n < NQ; ++n)
        if (stid == n) out[(size_t)n * (2 + G)] = m[n];
      if (stid < NQ) out[(size_t)stid * (2 + G) + 1] = Lt[stid];
      // TMEM lane L of sub-partition q in half h holds coordinate
      // 128h + 32q + 8((L%8)/2) + L/8 + 4(L%2); its values were 16 + nibble.
      const int cb = lane >> 3, sl = lane & 7;
#pragma unroll
      for (int h = 0; h < C::NH; ++h) {
        const int g = 128 * h + 32 * q + 8 * (sl >> 1) + cb + 4 * (sl & 1);
        uint32_t a[NQ];
        const uint32_t ta = tm + lane_base + C::OFF_ACC + h * NQ;
        if constexpr (NQ == 32) tmem_ld32(ta, a);
        else tmem_ld16(ta, a);
        tmem_ld_wait();
        if (g < G) {
#pragma unroll
          for (int n = 0; n < NQ; ++n) {
            const float d = __uint_as_float(a[n]);
            out[(size_t)n * (2 + G) + 2 + g] = d - 24.f * Lt[n];
          }
        }
      }
    }
  }
  // warps 2-3 have no role after set-up
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- prologue
// Per (b, h): q'_g = c * sum_d W_k[j*d_h + d][g] q[b][h][d] (c = scale*log2 e), rounded
// to fp16; written at its physical K position kappa, divided by the position's
// nibble factor (1 or 16), in the K-major no-swizzle layout of the score MMA's B
// operand.  corr[b][h] = 1024 * sum_kappa Q'[kappa] + 8 * sum_g q'_g, the part of
// the raw MMA score that the nibble bias and the -8 level offset contribute.
template <int G, int NQ>
__global__ void absorb_query_tc(const uint16_t *__restrict__ q, const uint16_t *__restrict__ W_kv, int n_kv,
                                float c, uint8_t *__restrict__ qphys, float *__restrict__ corr, uint32_t *err) {
  using C = Cfg<G, NQ>;
  constexpr int D = FSQ_HEAD_DIM;
  __shared__ float qs[D];
  __shared__ float red[2][8];
  const int h = blockIdx.x, b = blockIdx.y;
  const int j = h / (NQ / n_kv);
  if (h == 0 && b == 0 && threadIdx.x == 0) *err = 0u;
  for (int d = threadIdx.x; d < D; d += blockDim.x) qs[d] = bf16_to_f32(q[((int64_t)b * NQ + h) * D + d]);
  __syncthreads();
  float sum_q = 0.f, sum_phys = 0.f;
  uint8_t *dst = qphys + (size_t)b * C::Q_BYTES;
  for (int kap = threadIdx.x; kap < C::KPAD; kap += blockDim.x) {
    // kappa = 8w + 2cc + e  <->  coordinate 8w + cc + 4e, nibble factor 16 when cc is odd
    const int w = kap >> 3, cc = (kap >> 1) & 3, e = kap & 1;
    const int g = 8 * w + cc + 4 * e;
    float v = 0.f;
    if (g < G) {
      const uint16_t *wk = W_kv + (int64_t)j * D * G + g;
      for (int d = 0; d < D; ++d) v = fmaf(bf16_to_f32(wk[(int64_t)d * G]), qs[d], v);
      v *= c;
    }
    const __half hq = __float2half_rn(v);
    const float vq = __half2float(hq);          // the value the MMA multiplies (times its factor)
    const float f = (cc & 1) ? 16.f : 1.f;
    const __half hp = __float2half_rn(vq / f);  // exact: division by a power of two
    sum_q += vq;
    sum_phys += __half2float(hp);
    const int off = (kap >> 3) * C::LBO_Q + (h >> 3) * 128 + (h & 7) * 16 + (kap & 7) * 2;
    *reinterpret_cast<__half *>(dst + off) = hp;
  }
  for (int o = 16; o; o >>= 1) {
    sum_q += __shfl_xor_sync(0xffffffffu, sum_q, o);
    sum_phys += __shfl_xor_sync(0xffffffffu, sum_phys, o);
  }
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x >> 5] = sum_q;
    red[1][threadIdx.x >> 5] = sum_phys;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.f, bsum = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
      a += red[0][i];
      bsum += red[1][i];
    }
    corr[(size_t)b * NQ + h] = 1024.f * bsum + 8.f * a;
  }
}

template <int G, int NQ>
cudaError_t launch(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int64_t T, int n_kv,
                   const uint16_t *W_kv, float scale, int S, int64_t tps, uint8_t *qphys, float *corr, float *part,
                   uint32_t *err, void *const *prof, cudaStream_t st) {
  using C = Cfg<G, NQ>;
  absorb_query_tc<G, NQ><<<dim3(NQ, (unsigned)B), 256, 0, st>>>(q, W_kv, n_kv, scale * kLog2e, qphys, corr, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // one CTA per SM: ask for more shared memory than two CTAs could share
  const int smem = C::SM_TOTAL > 120 * 1024 ? C::SM_TOTAL : 120 * 1024;
  e = cudaFuncSetAttribute(absorbed_split_tc<G, NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  Params p{codes, bstride, T, tps, S, qphys, corr, part, err, kWaitLimitNs};
  if (prof[0]) cudaEventRecord((cudaEvent_t)prof[0], st);
  absorbed_split_tc<G, NQ><<<dim3(S, (unsigned)B), 384, smem, st>>>(p);
  e = cudaGetLastError();
  if (prof[1]) cudaEventRecord((cudaEvent_t)prof[1], st);
  return e;
}

}  // namespace tc

bool absorbed_tc_supported(int n_q, int G) { return (n_q == 16 || n_q == 32) && (G == 256 || G == 84); }

size_t absorbed_tc_qphys_bytes(int n_q, int G) {
  const int kpad = (G + 15) / 16 * 16;
  return (size_t)n_q * kpad * 2;
}

cudaError_t merge_absorbed_launch(const float *part, int S, int64_t B, int n_q, int n_kv, int d_h, int G,
                                  const uint16_t *W_kv, void *o, int out_fp32, cudaStream_t st);

cudaError_t launch_absorbed_tc(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int64_t T,
                               int n_q, int n_kv, int d_h, int G, const uint16_t *W_kv, float scale, int S,
                               int64_t tps, uint8_t *qphys, float *corr, float *part, uint32_t *err, void *o,
                               int out_fp32, void *const *prof, cudaStream_t st) {
  cudaError_t e;
  if (G == 256 && n_q == 32) e = tc::launch<256, 32>(q, codes, bstride, B, T, n_kv, W_kv, scale, S, tps, qphys, corr, part, err, prof, st);
  else if (G == 256 && n_q == 16) e = tc::launch<256, 16>(q, codes, bstride, B, T, n_kv, W_kv, scale, S, tps, qphys, corr, part, err, prof, st);
  else if (G == 84 && n_q == 32) e = tc::launch<84, 32>(q, codes, bstride, B, T, n_kv, W_kv, scale, S, tps, qphys, corr, part, err, prof, st);
  else if (G == 84 && n_q == 16) e = tc::launch<84, 16>(q, codes, bstride, B, T, n_kv, W_kv, scale, S, tps, qphys, corr, part, err, prof, st);
  else return cudaErrorInvalidValue;
  if (e != cudaSuccess) return e;
  return merge_absorbed_launch(part, S, B, n_q, n_kv, d_h, G, W_kv, o, out_fp32, st);
}

}  // namespace fsq
