// Decode attention with the keys rebuilt per tile on the 5th-generation tensor
// cores: the pages' own kernel design (slide deck frame "The kernel reads codes
// and never writes reconstructed K/V": unpack codes in registers, reconstruct
// keys with W_k on tensor cores, apply the key norm and RoPE on chip, online
// softmax, accumulate attention-weighted codes, merge partials and apply W_v
// once), and the variant that rebuilds the values per tile as well.
//
// One CTA per (token split, batch row, kv head j); the GRP query heads of kv
// head j share its keys.  Per 128-token tile:
//   Zh  [128 tok x KPAD]  in TMEM: each coordinate's n = level + 8 left in
//                         place as an fp16 subnormal, n 2^-24 or n 2^-20 (one
//                         LOP3 per pair of coordinates)
//   K   [128 tok x 128]   = Zh . Wk'^T on tcgen05 (kind::f16, fp32 in TMEM).
//                         Wk' is W_k^(j) in fp16 with a factor 16 on the
//                         coordinates of the 2^-24 kind, so that every product
//                         carries 2^-20; rows are ordered so that the RoPE pair
//                         (d, d + 64) lands in two adjacent columns.  It is
//                         staged once per call and once per CTA in shared memory.
//   k~  = RoPE_t(g . k), k = 2^20 K - 8 sum_g W_k[d, g], on the CUDA cores in
//         one pass per token ([S] eq. 5: k_t = RoPE_t(N_k(W_k z_t))).  The RMS
//         norm divides k by a per-token scalar that the rotation leaves alone,
//         so that scalar multiplies the scores instead.
//   S   [128 tok x 16]    = k~ . Q'^T on tcgen05 (Q' = q scale log2 e; the GRP
//                         heads zero-padded to N = 16)
//   online softmax (thread = token, lazy rescale at 2^8), P fp16 in shared memory
//   values, HYBRID:  ACC [G x 16] += Zh^T . P on tcgen05: the latent pooling of
//                    the absorbed kernel; the split merge applies W_v once ([S]
//                    eq. 6; deck frame "Attention pools codes before decoding
//                    values")
//           EXPAND:  V [128 tok x 128] = Zh . Wv'^T, then O^T [128 x 16] +=
//                    V^T . P, both on tcgen05 (values rebuilt per tile in
//                    shared memory, the form the absorbed one is measured
//                    against)
//
// Warps: 0 producer (staged decoder slices, queries, code tiles); 1 MMA issuer;
// 4-7 Zh dequant; 8-15 token warps (two per TMEM sub-partition: each rotates
// half the RoPE pairs of its 32 tokens; 8-11 also run the softmax, and all
// eight convert V); 16-23 (HYBRID) Zh^T dequant for the latent pooling.  Every
// wait is bounded; a wait that gives up records FSQ_ERR_TIMEOUT and all roles
// leave their loops, after which the producer and the issuer wait (with their
// own limit) for their copies and MMAs in flight.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc_decode.cuh"
#include "tc_ptx.cuh"

namespace fsq {
namespace tc {

cudaError_t make_code_tensor_map(CUtensorMap *map, const uint8_t *codes, int64_t bstride, int64_t T, int64_t B,
                                 int row_bytes);

namespace x {

constexpr int kT = 128;          // tokens per tile
constexpr int kNP = 16;          // N of the score, pooling and output MMAs: GRP heads, zero padded
constexpr int kPSlots = 4;       // ring of softmax-weight (P) tiles
constexpr float kTau = 8.f;      // rescale when a score exceeds the running max by 2^8
constexpr uint64_t kWaitNs = 1000000000ull;   // 1 s per hand-off wait
constexpr uint64_t kDrainNs = 1000000000ull;  // 1 s for copies and MMAs in flight on the error path
constexpr int kMaxGrp = 8;       // query heads per kv head (softmax registers)
constexpr int kMisc = 8192;
// Every kFlushTiles tiles (HYBRID) the softmax warps fold the latent-pooling
// accumulator into fp32 sums of their own and the pooling MMAs start afresh:
// its products are all non-negative, the tensor core's fp32 accumulation is
// not round-to-nearest, and the epilogue's -8 l correction would magnify the
// drift of one chain over a whole long split.
constexpr int kFlushTiles = 64;

// 16-bit operand layouts in shared memory, no swizzle (8 x 16-byte core matrices):
// K-major [N x K]: 8-row groups 128 bytes apart, 8-element K chunks `lbo` apart
__host__ __device__ constexpr int kmaj(int n, int k, int lbo) {
  return (k >> 3) * lbo + (n >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2;
}
// MN-major [M x K]: 8 consecutive M elements of one K form 16 bytes; 8 K form a
// 128-byte core matrix; K core matrices 128 bytes apart, M groups `sbo` apart
__host__ __device__ constexpr int mnmaj(int m, int k, int sbo) {
  return (k >> 3) * 128 + (k & 7) * 16 + (m >> 3) * sbo + (m & 7) * 2;
}

template <int G, bool VEXP>
struct XC {
  static constexpr int HALF = G / 2;
  static constexpr int KPAD = (G + 15) / 16 * 16;  // K of the key / value MMAs (16 per step)
  static constexpr int KW = KPAD / 8;              // 32-bit code words (8 coordinates) per padded row
  static constexpr int ZCOLS = KPAD / 2;           // TMEM columns of Zh (two fp16 per column)
  static constexpr int NH = (G + 127) / 128;       // 128-row halves of the latent pooling
  static constexpr bool TMA = (HALF == 128);
  static constexpr int TILE_BYTES = kT * HALF;
  static constexpr int STAGE_BYTES = TMA ? TILE_BYTES : (TILE_BYTES + 16 + 127) / 128 * 128;
  static constexpr int W_BYTES = 128 * KPAD * 2;   // one staged decoder slice (fp16)
  static constexpr int W_LBO = (128 / 8) * 128;
  static constexpr int Q_BYTES = kNP * 128 * 2;
  static constexpr int Q_LBO = (kNP / 8) * 128;
  static constexpr int P_BYTES = kT * kNP * 2;
  static constexpr int P_SBO = (kT / 8) * 128;
  static constexpr int VS_BYTES = VEXP ? 128 * kT * 2 : 0;
  static constexpr int VS_SBO = (kT / 8) * 128;
  static constexpr int THREADS = (VEXP ? 16 : 24) * 32;
  // TMEM columns
  static constexpr int A32(int v) { return (v + 31) / 32 * 32; }
  static constexpr int OFF_Z = 0;
  static constexpr int OFF_K = A32(ZCOLS);
  static constexpr int OFF_KR = OFF_K + 128;
  static constexpr int OFF_S = OFF_KR + 64;
  static constexpr int CP_CHUNK = NH * 32;         // one 64-token chunk of Zh^T
  static constexpr int OFF_CP = A32(OFF_S + kNP);
  static constexpr int OFF_ACC = OFF_CP + 2 * CP_CHUNK;
  static constexpr int OFF_V = A32(OFF_S + kNP);
  static constexpr int OFF_O = OFF_V + 128;
  static constexpr int TMEM_USED = VEXP ? OFF_O + kNP : OFF_ACC + NH * kNP;
  static constexpr int TMEM_COLS = TMEM_USED <= 256 ? 256 : 512;
  static_assert(TMEM_USED <= 512, "TMEM plan exceeds 512 columns");
  // shared memory
  static constexpr int FL_BYTES = VEXP ? 0 : 16 * 128 * 4;  // 16 flushed fp32 sums per softmax thread
  static constexpr int FIXED = W_BYTES * (VEXP ? 2 : 1) + Q_BYTES + kPSlots * P_BYTES + VS_BYTES + kMisc + FL_BYTES;
  static constexpr int STAGES_FIT = (226 * 1024 - FIXED) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT < 8 ? STAGES_FIT : 8;
  static_assert(STAGES >= 2, "code-tile ring too shallow");
  static constexpr int SM_CODES = 0;
  static constexpr int SM_WK = STAGES * STAGE_BYTES;
  static constexpr int SM_WV = SM_WK + W_BYTES;
  static constexpr int SM_Q = SM_WV + (VEXP ? W_BYTES : 0);
  static constexpr int SM_P = SM_Q + Q_BYTES;
  static constexpr int SM_VS = SM_P + kPSlots * P_BYTES;
  static constexpr int SM_MISC = SM_VS + VS_BYTES;
  static constexpr int SM_FL = SM_MISC + kMisc;
  static constexpr int SM_TOTAL = SM_FL + FL_BYTES;
};

struct XParams {
  const uint8_t *codes;
  int64_t bstride, T, tps;
  int S, n_q, n_kv, grp;
  const uint8_t *wk, *wv;    // staged decoder slices [n_kv][W_BYTES] (V: EXPAND only)
  const float *ck, *cv;      // [n_kv][128] level-offset terms 8 sum_g W[d, g] (k: pair order)
  const uint8_t *qs;         // [B][n_kv][Q_BYTES] staged queries
  const uint16_t *gain;      // bf16 [128] RMS-norm gain or null (ones)
  float qres;                // scale log2 e / 2^k: the part of the score scale not folded into Q'
  float eps, rope_base;
  int rope;
  float *part;               // HYBRID [B][S][n_q][2 + G]; EXPAND [B][S][n_q][2 + 128]
  uint32_t *err;
  const int32_t *seq_lens;
  uint32_t stall_ns;
  int n_new;                 // queries per cache row: grid row r reads cache row r / n_new (causal)
};

struct XMisc {
  uint64_t full[8], empty[8];
  uint64_t w_full, z_ready, z_free, k_full, k_free, kr_ready, kr_free, s_full, s_free;
  uint64_t p_full[kPSlots], p_free[kPSlots], cp_ready[2], cp_free[2];
  uint64_t v_full, v_free, vs_ready, o_free, acc_full, done, never;
  uint32_t tmem_base, abort;
  double theta_d[64];        // RoPE frequencies base^(-2i/128)
  float theta[64];
  float phib[2][64];         // (tile start * theta_i) mod 2 pi, per tile parity
  float ck[128], cv[128], gp[128];
  float ss[128];             // sum-of-squares exchange between the two halves
  float red[4][kMaxGrp];
  float lt[4][kMaxGrp];
};
static_assert(sizeof(XMisc) <= kMisc, "XMisc exceeds its reservation");

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t *>(&h);
}

template <int G, bool VEXP>
__global__ void __launch_bounds__(XC<G, VEXP>::THREADS, 1)
    expand_split_tc(const __grid_constant__ CUtensorMap tmap, XParams p) {
  using C = XC<G, VEXP>;
  extern __shared__ __align__(1024) uint8_t smem[];
  XMisc &ms = *reinterpret_cast<XMisc *>(smem + C::SM_MISC);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, b = blockIdx.y, j = blockIdx.z;
  const int GRP = p.grp;
  constexpr int REC = 2 + (VEXP ? 128 : G);  // floats per partial record
  const int64_t t0 = (int64_t)split * p.tps;
  const int64_t t1 = min(query_len(p.seq_lens, b, p.n_new, p.T, p.err, false), t0 + p.tps);
  float *prec = p.part + (((size_t)b * p.S + split) * p.n_q + (size_t)j * GRP) * REC;
  if (t1 <= t0) {
    // a split wholly past its row's length (ragged batch, causal query): empty partials
    pdl_wait();
    for (int i = tid; i < GRP * REC; i += C::THREADS) prec[i] = (i % REC) == 0 ? -INFINITY : 0.f;
    return;
  }
  const int n_tiles = (int)((t1 - t0 + kT - 1) / kT);
  const int crow = b / p.n_new;  // cache row
  const uint8_t *gcodes = p.codes + (int64_t)crow * p.bstride + t0 * C::HALF;
  volatile uint32_t *abort = &ms.abort;

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&ms.full[s], 1);
      mbar_init(&ms.empty[s], VEXP ? 4 : 12);
    }
    mbar_init(&ms.w_full, 1);
    mbar_init(&ms.z_ready, 4);
    mbar_init(&ms.z_free, 1);
    mbar_init(&ms.k_full, 1);
    mbar_init(&ms.k_free, 8);
    mbar_init(&ms.kr_ready, 8);
    mbar_init(&ms.kr_free, 1);
    mbar_init(&ms.s_full, 1);
    mbar_init(&ms.s_free, 4);
    for (int i = 0; i < kPSlots; ++i) {
      mbar_init(&ms.p_full[i], 4);
      mbar_init(&ms.p_free[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ms.cp_ready[i], 4);
      mbar_init(&ms.cp_free[i], 1);
    }
    mbar_init(&ms.v_full, 1);
    mbar_init(&ms.v_free, 8);
    mbar_init(&ms.vs_ready, 8);
    mbar_init(&ms.o_free, 1);
    mbar_init(&ms.acc_full, 1);
    mbar_init(&ms.done, 1);
    mbar_init(&ms.never, 1);  // completed by nothing: the test-only stall waits on it
    ms.abort = 0u;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&ms.tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  for (int i = tid; i < kPSlots * C::P_BYTES / 16; i += C::THREADS)  // P ring: padding heads stay zero
    reinterpret_cast<uint4 *>(smem + C::SM_P)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (tid >= 256 && tid < 320) {  // RoPE frequencies and the first tile's base angles
    const int i = tid - 256;
    const double th = pow((double)p.rope_base, -2.0 * (double)i / 128.0);
    ms.theta_d[i] = th;
    ms.theta[i] = (float)th;
    ms.phib[0][i] = (float)fmod((double)t0 * th, 6.283185307179586);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ms.tmem_base;
  pdl_trigger();

  auto fail = [&]() {
    record_error(p.err, FSQ_ERR_TIMEOUT);
    *abort = 1u;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint8_t *ring = smem + C::SM_CODES;
    const uint64_t pol = p.n_new > 1 ? l2_evict_normal() : l2_evict_first();
    int issued = 0;
    bool ok = true, w_loaded = false;
    auto load_w = [&]() {
      // the staged decoder slices and queries come from the prologue kernel
      if (lane == 0) {
        pdl_wait();
        const uint32_t bytes = C::W_BYTES * (VEXP ? 2 : 1) + C::Q_BYTES;
        mbar_arrive_expect_tx(&ms.w_full, bytes);
        bulk_g2s(smem + C::SM_WK, p.wk + (size_t)j * C::W_BYTES, C::W_BYTES, &ms.w_full);
        if constexpr (VEXP) bulk_g2s(smem + C::SM_WV, p.wv + (size_t)j * C::W_BYTES, C::W_BYTES, &ms.w_full);
        bulk_g2s(smem + C::SM_Q, p.qs + ((size_t)b * p.n_kv + j) * C::Q_BYTES, C::Q_BYTES, &ms.w_full);
      }
    };
    for (int i = 0; i < n_tiles; ++i) {
      const int st = i % C::STAGES;
      const uint32_t ph = (uint32_t)(i / C::STAGES) & 1u;
      if (i == C::STAGES) {
        load_w();
        w_loaded = true;
      }
      if (!wait_bar(&ms.empty[st], ph ^ 1u, abort, kWaitNs)) {
        ok = false;
        break;
      }
      const int64_t rows = min((int64_t)kT, t1 - (t0 + (int64_t)i * kT));
      uint8_t *dst = ring + st * C::STAGE_BYTES;
      const uint8_t *src = gcodes + (int64_t)i * kT * C::HALF;
      if constexpr (C::TMA) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&ms.full[st], C::TILE_BYTES);
          tma_load_3d(dst, &tmap, 0, (int)(t0 + (int64_t)i * kT), crow, &ms.full[st], pol);
        }
      } else if (rows == kT) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&ms.full[st], C::TILE_BYTES);
          bulk_g2s_hint(dst, src, C::TILE_BYTES, &ms.full[st], pol);
        }
      } else {
        const int nb = (int)rows * C::HALF;
        for (int k = lane; k < C::STAGE_BYTES; k += 32) dst[k] = (k < nb) ? src[k] : (uint8_t)0;
        __syncwarp();
        if (lane == 0) mbar_arrive(&ms.full[st]);
      }
      issued = i + 1;
    }
    if (!w_loaded) load_w();
    if (!ok) {
      if (lane == 0) fail();
      for (int i = max(0, issued - C::STAGES); i < issued; ++i)
        drain_bar(&ms.full[i % C::STAGES], (uint32_t)(i / C::STAGES) & 1u, kDrainNs);
    }
    drain_bar(&ms.w_full, 0, kDrainNs);  // no copy may land after the CTA exits
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (one elected lane)
    constexpr uint32_t idK = idesc_f16(128, 128, 0, 0);
    constexpr uint32_t idS = idesc_f16(128, kNP, 0, 0);
    constexpr uint32_t idP = idesc_f16(128, kNP, 0, 1);
    constexpr uint32_t idO = idesc_f16(128, kNP, 1, 1);
    const uint64_t wkd = smem_desc(smem_u32(smem + C::SM_WK), C::W_LBO, 128);
    const uint64_t wvd = smem_desc(smem_u32(smem + C::SM_WV), C::W_LBO, 128);
    const uint64_t qd = smem_desc(smem_u32(smem + C::SM_Q), C::Q_LBO, 128);
    const uint64_t pd0 = smem_desc(smem_u32(smem + C::SM_P), 128, C::P_SBO);
    const uint64_t vsd = smem_desc(smem_u32(smem + C::SM_VS), 128, C::VS_SBO);
    bool ok = wait_bar(&ms.w_full, 0, abort, kWaitNs);
    // keys (and values) of tile i: A = Zh, B = the staged decoder slice
    auto issue_kv = [&](int i) -> bool {
      const uint32_t pi = (uint32_t)i & 1u;
      if (!wait_bars(&ms.z_ready, pi, &ms.k_free, pi ^ 1u, abort, kWaitNs)) return false;
      if constexpr (VEXP)
        if (!wait_bar(&ms.v_free, pi ^ 1u, abort, kWaitNs)) return false;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll 4
        for (int k = 0; k < C::KPAD / 16; ++k)
          mma_ts(tm + C::OFF_K, tm + C::OFF_Z + 8 * k, wkd + (uint64_t)((2 * k * C::W_LBO) >> 4), idK, k > 0);
        if constexpr (VEXP) {
#pragma unroll 4
          for (int k = 0; k < C::KPAD / 16; ++k)
            mma_ts(tm + C::OFF_V, tm + C::OFF_Z + 8 * k, wvd + (uint64_t)((2 * k * C::W_LBO) >> 4), idK, k > 0);
          tc_commit(&ms.v_full);
        }
        tc_commit(&ms.k_full);
        tc_commit(&ms.z_free);
      }
      __syncwarp();
      return true;
    };
    if (ok) ok = issue_kv(0);
    for (int i = 0; i < n_tiles && ok; ++i) {
      const uint32_t pi = (uint32_t)i & 1u;
      // scores of tile i: A = the rotated keys, B = the staged queries
      if (!wait_bars(&ms.kr_ready, pi, &ms.s_free, pi ^ 1u, abort, kWaitNs)) { ok = false; break; }
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ts(tm + C::OFF_S, tm + C::OFF_KR + 8 * k, qd + (uint64_t)((2 * k * C::Q_LBO) >> 4), idS, k > 0);
        tc_commit(&ms.s_full);
        tc_commit(&ms.kr_free);
      }
      __syncwarp();
      if (i + 1 < n_tiles && !issue_kv(i + 1)) { ok = false; break; }
      // values of tile i
      const int slot = i % kPSlots;
      const uint64_t pd = pd0 + (uint64_t)((slot * C::P_BYTES) >> 4);
      if constexpr (VEXP) {
        if (!wait_bars(&ms.p_full[slot], (uint32_t)(i / kPSlots) & 1u, &ms.vs_ready, pi, abort, kWaitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ss(tm + C::OFF_O, vsd + (uint64_t)(16 * k), pd + (uint64_t)(16 * k), idO, (i > 0 || k > 0) ? 1u : 0u);
          tc_commit(&ms.o_free);
          tc_commit(&ms.p_free[slot]);
        }
        __syncwarp();
      } else {
        if (!wait_bar(&ms.p_full[slot], (uint32_t)(i / kPSlots) & 1u, abort, kWaitNs)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (!wait_bar(&ms.cp_ready[c], pi, abort, kWaitNs)) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int h = 0; h < C::NH; ++h)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ts(tm + C::OFF_ACC + h * kNP, tm + C::OFF_CP + c * C::CP_CHUNK + h * 32 + kk * 8,
                       pd + (uint64_t)(16 * (4 * c + kk)), idP,
                       (i % kFlushTiles == 0 && c == 0 && kk == 0) ? 0u : 1u);
            tc_commit(&ms.cp_free[c]);
          }
          __syncwarp();
        }
        if (!ok) break;
        tc_commit_elect(&ms.p_free[slot]);
      }
    }
    if (ok) tc_commit_elect(&ms.acc_full);
    else if (lane == 0) fail();
    // every MMA of this warp completes before TMEM is freed, error or not
    tc_commit_elect(&ms.done);
    drain_bar(&ms.done, 0, kDrainNs);
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ Zh dequant: token row -> TMEM lane
    const int q = warp - 4;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const int rr = 32 * q + lane;
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      const int st = i % C::STAGES;
      const uint8_t *tile = smem + C::SM_CODES + st * C::STAGE_BYTES;
      if (!wait_bars(&ms.full[st], (uint32_t)(i / C::STAGES) & 1u, &ms.z_free, ((uint32_t)i & 1u) ^ 1u, abort,
                     kWaitNs)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // code word w (coordinates 8w..8w+7) -> columns 4w..4w+3: (n0,n4) (n1,n5) (n2,n6) (n3,n7)
#pragma unroll
      for (int w0 = 0; w0 < C::KW; w0 += 8) {
        const int nw = (C::KW - w0) < 8 ? (C::KW - w0) : 8;
        uint32_t r[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int kw = w0 + k;
          uint32_t w = 0u;
          if constexpr (C::TMA) {
            w = *reinterpret_cast<const uint32_t *>(tile + swz(rr, kw >> 2) + 4 * (kw & 3));
          } else {
            const uint8_t *row = tile + rr * C::HALF;
            if (4 * kw + 4 <= C::HALF) w = lds_u32_a2(row + 4 * kw);
            else if (4 * kw + 2 <= C::HALF) w = *reinterpret_cast<const uint16_t *>(row + 4 * kw);
          }
          nib_sub4(w, r[4 * k], r[4 * k + 1], r[4 * k + 2], r[4 * k + 3]);
        }
        const uint32_t ta = tm + lane_base + C::OFF_Z + 4 * w0;
        if (nw == 8) {
          tmem_st32(ta, r);
        } else {
          if (nw >= 4) tmem_st16(ta, r);
          if (nw % 4 == 2) tmem_st8(ta + 4 * (nw - 2), r + 4 * (nw - 2));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.empty[st]);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.z_ready);
    }
    if (!ok && lane == 0) fail();
  } else if (warp >= 8 && warp < 16) {
    // ------------------------------------------------------------ token warps: keys, softmax, values
    const int q = warp & 3;
    const int hv = (warp - 8) >> 2;            // which half of the RoPE pairs (and of V's dims)
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const int r = 32 * q + lane;               // token row within the tile
    const float rf = (float)r;
    // threads r < 64 of warps 8-9 carry (tile start * theta_r) mod 2 pi and its per-tile step
    double phd = 0.0, dphi = 0.0;
    if (hv == 0 && r < 64) {
      phd = fmod((double)t0 * ms.theta_d[r], 6.283185307179586);
      dphi = fmod((double)kT * ms.theta_d[r], 6.283185307179586);
    }
    const int gt = tid - 256;                  // 0..255 over the eight token warps
    pdl_wait();                                // the offset terms come from the prologue kernel
    // a bad per-row length is reported once, after the prologue cleared the error word
    if (split == 0 && j == 0 && gt == 0) query_len(p.seq_lens, b, p.n_new, p.T, p.err, true);
    for (int d = gt; d < 128; d += 256) {
      const int dk = (d >> 1) + 64 * (d & 1);  // pair order: column 2i + e is dimension i + 64 e
      ms.ck[d] = p.ck[(size_t)j * 128 + d];
      ms.gp[d] = (p.rope && p.gain) ? bf16_to_f32(p.gain[dk]) : 1.f;
      if constexpr (VEXP) ms.cv[d] = p.cv[(size_t)j * 128 + d];
    }
    named_bar(2, 256);
    // A wait that gives up leaves `good` false; the warps of a group learn of it
    // at their next common barrier (which ORs the flags), so they always pass
    // the same named barriers and leave together.
    bool ok = true;
    if (p.stall_ns != 0u && !wait_bar(&ms.never, 0, abort, p.stall_ns)) ok = false;
    // softmax state (warps 8-11): running max per head (equal in every thread), the thread's weight sums
    float m[kMaxGrp], lsum[kMaxGrp];
#pragma unroll
    for (int h = 0; h < kMaxGrp; ++h) {
      m[h] = 0.f;
      lsum[h] = 0.f;
    }
    const int kap = VEXP ? r : kappa_of_token(r);  // this token's K position in the value MMA's operands
    // this thread's flushed latent sums (HYBRID): slot k (ACC block k / 8, head k % 8) at fl[k * 128]
    float *fl = reinterpret_cast<float *>(smem + C::SM_FL) + (32 * q + lane);
    if (!VEXP && hv == 0) {
#pragma unroll
      for (int k = 0; k < 16; ++k) fl[k * 128] = 0.f;
    }
    for (int i = 0; i < n_tiles; ++i) {
      const uint32_t pi = (uint32_t)i & 1u;
      bool good = ok;
      // ---- keys: one pass over this thread's 32 RoPE pairs
      if (good) good = wait_bars(&ms.k_full, pi, &ms.kr_free, pi ^ 1u, abort, kWaitNs);
      float ss = 0.f;
      if (good) {
        tc_fence_after();
        const float *phb = ms.phib[i & 1];
#pragma unroll 1
        for (int c0 = 32 * hv; c0 < 32 * hv + 32; c0 += 8) {
          uint32_t kv[16], out[8];
          tmem_ld16(tm + lane_base + C::OFF_K + 2 * c0, kv);
          tmem_ld_wait();
#pragma unroll
          for (int pp = 0; pp < 8; ++pp) {
            const int ii = c0 + pp;
            float kx = fmaf(__uint_as_float(kv[2 * pp]), 1048576.f, -ms.ck[2 * ii]);
            float ky = fmaf(__uint_as_float(kv[2 * pp + 1]), 1048576.f, -ms.ck[2 * ii + 1]);
            if (p.rope) {
              ss = fmaf(kx, kx, fmaf(ky, ky, ss));
              kx *= ms.gp[2 * ii];
              ky *= ms.gp[2 * ii + 1];
              float ang = fmaf(rf, ms.theta[ii], phb[ii]);
              ang = fmaf(-6.283185307179586f, rintf(ang * 0.15915494309189535f), ang);
              float sn, cs;
              __sincosf(ang, &sn, &cs);
              const float rx = fmaf(kx, cs, -ky * sn), ry = fmaf(kx, sn, ky * cs);
              kx = rx;
              ky = ry;
            }
            out[pp] = pack_half2(kx, ky);
          }
          tmem_st8(tm + lane_base + C::OFF_KR + c0, out);
        }
        tmem_st_wait();
        tc_fence_before();
      }
      if (hv) ms.ss[r] = ss;
      if (hv == 0 && r < 64) {  // base angles of the next tile: advance by 128 theta_r, mod 2 pi, in fp64
        phd += dphi;
        if (phd >= 6.283185307179586) phd -= 6.283185307179586;
        ms.phib[(i + 1) & 1][r] = (float)phd;
      }
      if (named_bar_or(2, 256, !good)) {
        if (lane == 0) fail();
        ok = false;
        break;
      }
      // 1 / rms(k) of this token, read before the keys' buffer is released
      // the score scale of this token: 1 / rms(k) (key norm) times the part of scale log2 e not in Q'
      const float inv_r = ((hv == 0 && p.rope) ? rsqrtf((ss + ms.ss[r]) * (1.f / 128.f) + p.eps) : 1.f) * p.qres;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ms.k_free);
        mbar_arrive(&ms.kr_ready);
      }
      // ---- softmax (warps 8-11)
      if (hv == 0) {
        bool g2 = wait_bar(&ms.s_full, pi, abort, kWaitNs);
        uint32_t sv[8];
        if (g2) {
          tc_fence_after();
          tmem_ld8(tm + lane_base + C::OFF_S, sv);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ms.s_free);
        }
        if (named_bar_or(1, 128, !g2)) {
          good = false;  // reported at the next common barrier (or the epilogue's)
        } else {
          const bool valid = t0 + (int64_t)i * kT + r < t1;
          float x[kMaxGrp];
          float xm = -INFINITY;
#pragma unroll
          for (int h = 0; h < kMaxGrp; ++h) {
            x[h] = (h < GRP && valid) ? fmaf(__uint_as_float(sv[h]), inv_r, -m[h]) : -INFINITY;
            xm = fmaxf(xm, x[h]);
          }
          const bool need = (i == 0) || xm > kTau;
          const bool any = named_bar_or(1, 128, need);
          const bool flush = !VEXP && i > 0 && (i % kFlushTiles) == 0;  // the pooling MMAs restart at tile i
          if (any || flush) {
            float f[kMaxGrp];
#pragma unroll
            for (int h = 0; h < kMaxGrp; ++h) f[h] = 1.f;
            if (any) {
              // raise the running max to the tile's (m <- m + max(0, tile max of x); first tile: its max)
#pragma unroll
              for (int h = 0; h < kMaxGrp; ++h) {
                float v = x[h];
#pragma unroll
                for (int off = 16; off; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
                if (lane == 0) ms.red[q][h] = v;
              }
              named_bar(1, 128);
#pragma unroll
              for (int h = 0; h < kMaxGrp; ++h) {
                const float dmax = fmaxf(fmaxf(ms.red[0][h], ms.red[1][h]), fmaxf(ms.red[2][h], ms.red[3][h]));
                const float sh = (i == 0) ? dmax : fmaxf(dmax, 0.f);
                f[h] = (i == 0) ? 0.f : exp2f(-sh);
                if (h < GRP) {
                  x[h] -= sh;
                  m[h] += sh;
                  lsum[h] *= f[h];
                }
              }
              named_bar(1, 128);  // ms.red is reused by the next rescale
            }
            if (i > 0) {
              // the accumulator must hold every earlier tile before it is rescaled or folded
              const int pi1 = i - 1;
              good = wait_bar(&ms.p_free[pi1 % kPSlots], (uint32_t)(pi1 / kPSlots) & 1u, abort, kWaitNs);
              if (good) {
                tc_fence_after();
                const int nblk = VEXP ? 1 : C::NH;
                for (int blk = 0; blk < nblk; ++blk) {
                  uint32_t a[8];
                  const uint32_t ta = tm + lane_base + (VEXP ? C::OFF_O : C::OFF_ACC + blk * kNP);
                  tmem_ld8(ta, a);
                  tmem_ld_wait();
                  if (flush) {  // fold into this thread's fp32 sums; tile i's MMAs overwrite ACC
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                      float *slot = fl + (blk * 8 + h) * 128;
                      *slot = (*slot + __uint_as_float(a[h])) * f[h];
                    }
                  } else {
                    // rescale: the accumulator and (HYBRID) the sums folded out of earlier runs
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                      a[h] = __float_as_uint(__uint_as_float(a[h]) * f[h]);
                      if (!VEXP) fl[(blk * 8 + h) * 128] *= f[h];
                    }
                    tmem_st8(ta, a);
                  }
                }
                if (!flush) tmem_st_wait();
                tc_fence_before();
              }
            }
          }
          // weights of this token (heads 0..7; the slot's heads 8..15 stay zero)
          const int slot = i % kPSlots;
          if (good && i >= kPSlots)
            good = wait_bar(&ms.p_free[slot], (uint32_t)((i - kPSlots) / kPSlots) & 1u, abort, kWaitNs);
          if (good) {
            uint32_t h2[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float p0 = ex2_approx(x[2 * k]), p1 = ex2_approx(x[2 * k + 1]);
              lsum[2 * k] += p0;
              lsum[2 * k + 1] += p1;
              h2[k] = pack_half2(p0, p1);
            }
            uint8_t *prow = smem + C::SM_P + slot * C::P_BYTES + mnmaj(0, kap, C::P_SBO);
            *reinterpret_cast<uint4 *>(prow) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ms.p_full[slot]);
          }
        }
      }
      // ---- values (EXPAND): V of this token -> fp16, MN-major in shared memory
      if constexpr (VEXP) {
        if (good) good = wait_bars(&ms.v_full, pi, &ms.o_free, pi ^ 1u, abort, kWaitNs);
        if (good) {
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 64 * hv; c0 < 64 * hv + 64; c0 += 16) {
            uint32_t vv[16];
            tmem_ld16(tm + lane_base + C::OFF_V + c0, vv);
            tmem_ld_wait();
            uint32_t o8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              o8[e] = pack_half2(fmaf(__uint_as_float(vv[2 * e]), 1048576.f, -ms.cv[c0 + 2 * e]),
                                 fmaf(__uint_as_float(vv[2 * e + 1]), 1048576.f, -ms.cv[c0 + 2 * e + 1]));
            uint8_t *vs = smem + C::SM_VS;
            *reinterpret_cast<uint4 *>(vs + mnmaj(c0, r, C::VS_SBO)) = make_uint4(o8[0], o8[1], o8[2], o8[3]);
            *reinterpret_cast<uint4 *>(vs + mnmaj(c0 + 8, r, C::VS_SBO)) = make_uint4(o8[4], o8[5], o8[6], o8[7]);
          }
          tc_fence_before();
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&ms.v_free);
            mbar_arrive(&ms.vs_ready);
          }
        }
      }
      ok = good;
    }
    // ------------------------------------------------------------ epilogue (warps 8-11): accumulator -> partials
    if (hv == 0) {
      bool g3 = ok;
      if (g3) g3 = wait_bar(&ms.acc_full, 0, abort, kWaitNs);
      if (named_bar_or(1, 128, !g3)) {
        if (lane == 0) fail();
      } else {
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < kMaxGrp; ++h) {
          float v = lsum[h];
#pragma unroll
          for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
          if (lane == 0) ms.lt[q][h] = v;
        }
        named_bar(1, 128);
        float L[kMaxGrp];
#pragma unroll
        for (int h = 0; h < kMaxGrp; ++h) L[h] = (ms.lt[0][h] + ms.lt[1][h]) + (ms.lt[2][h] + ms.lt[3][h]);
        if (gt < GRP) {
#pragma unroll
          for (int h = 0; h < kMaxGrp; ++h)
            if (h == gt) {
              prec[(size_t)h * REC] = m[h];
              prec[(size_t)h * REC + 1] = L[h];
            }
        }
        if constexpr (VEXP) {
          uint32_t a[8];
          tmem_ld8(tm + lane_base + C::OFF_O, a);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < kMaxGrp; ++h)
            if (h < GRP) prec[(size_t)h * REC + 2 + r] = __uint_as_float(a[h]);
        } else {
          // TMEM lane L of sub-partition q in half hh holds coordinate
          // 128 hh + 32 q + 8 ((L % 8) / 2) + 4 (L % 2) + L / 8, pooled as n 2^-24
          // (L / 8 even) or n 2^-20 (L / 8 odd), n = level + 8
          const int jn = lane >> 3, sl = lane & 7;
          const float vscale = (jn & 1) ? 1048576.f : 16777216.f;
#pragma unroll
          for (int hh = 0; hh < C::NH; ++hh) {
            uint32_t a[8];
            tmem_ld8(tm + lane_base + C::OFF_ACC + hh * kNP, a);
            tmem_ld_wait();
            const int g = 128 * hh + 32 * q + 8 * (sl >> 1) + 4 * (sl & 1) + jn;
            if (g < G) {
#pragma unroll
              for (int h = 0; h < kMaxGrp; ++h)
                if (h < GRP)
                  prec[(size_t)h * REC + 2 + g] =
                      fmaf(__uint_as_float(a[h]) + fl[(hh * 8 + h) * 128], vscale, -8.f * L[h]);
            }
          }
        }
      }
    } else if (!ok && lane == 0) {
      fail();
    }
  } else if (!VEXP && warp >= 16 && warp < 24) {
    // ------------------------------------------------------------ Zh^T dequant for the latent pooling (HYBRID)
    // the same operand as the absorbed kernel's pooling: chunk c = 64 tokens,
    // coordinates on TMEM lanes, nibbles as fp16 subnormals in place
    const int q = warp & 3;
    const int c = (warp - 16) >> 2;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int st = i % C::STAGES;
      const uint8_t *tile = smem + C::SM_CODES + st * C::STAGE_BYTES;
      if (!wait_bars(&ms.full[st], (uint32_t)(i / C::STAGES) & 1u, &ms.cp_free[c], ((uint32_t)i & 1u) ^ 1u, abort,
                     kWaitNs)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < C::NH; ++h) {
        const int byte0 = 64 * h + 16 * q;
        if (byte0 >= C::HALF) continue;
        uint32_t lo[16], hi[16], y[8];
        if constexpr (C::TMA) {
          const uint32_t t0a = smem_u32(tile);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int rr = 8 * (8 * c + 4 * hf + (lane >> 3)) + (lane & 7);
            uint32_t r4[4];
            ldmatrix_x4_trans(t0a + (uint32_t)swz(rr, byte0 >> 4), r4);
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) y[4 * hf + mm] = r4[mm];
          }
        } else {
#pragma unroll
          for (int mm = 0; mm < 8; ++mm) {
            const int rr = 8 * (8 * c + mm) + (lane >> 2);
            y[mm] = movmatrix_trans(lds_u32_a2(tile + rr * C::HALF + byte0 + 4 * (lane & 3)));
          }
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            nib_sub4(y[2 * jj + e], lo[4 * jj + e], lo[4 * jj + 2 + e], hi[4 * jj + e], hi[4 * jj + 2 + e]);
        const uint32_t cb = tm + lane_base + C::OFF_CP + c * C::CP_CHUNK + h * 32;
        tmem_st_16x256b_x4(cb, lo);
        tmem_st_16x256b_x4(cb + (16u << 16), hi);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.empty[st]);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.cp_ready[c]);
    }
    if (!ok && lane == 0) fail();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- prologue
// Once per call: the decoder slices in the key / value MMAs' operand layout
// (fp16, factor 16 on the 2^-24 coordinates, keys in RoPE pair order), their
// level-offset terms 8 sum_g W[d, g] (from the fp16 values the MMAs use), and
// per (b, j) the queries Q'[h][2i + e] = q_h[i + 64 e] 2^k in the score MMA's
// operand layout: 2^k is the power of two at or below scale log2 e, so that
// Q' holds the bf16 query exactly; the rest of the scale multiplies the fp32
// scores.  Grid (n_kv, B).
template <int G, bool VEXP>
__global__ void __launch_bounds__(256) expand_prep(const uint16_t *__restrict__ q, const uint16_t *__restrict__ W_kv,
                                                   int n_q, int n_kv, int grp, float c, uint8_t *wk, uint8_t *wv,
                                                   float *ck, float *cv, uint8_t *qs, uint32_t *err,
                                                   MergeScratch msc) {
  using C = XC<G, VEXP>;
  constexpr int D = FSQ_HEAD_DIM;
  const int j = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  if (j == 0 && b == 0) {
    if (tid == 0) *err = 0u;
    for (int i = tid; i < msc.ncnt; i += 256) msc.cnt[i] = 0u;
  }
  if (b == 0) {
    // coordinate of K position kappa = 8w + 2c + e: 8w + c + 4e (c odd: the 2^-20 kind)
    for (int mat = 0; mat < (VEXP ? 2 : 1); ++mat) {
      uint8_t *dst = (mat == 0 ? wk : wv) + (size_t)j * C::W_BYTES;
      float *cd = (mat == 0 ? ck : cv) + (size_t)j * D;
      const uint16_t *src = W_kv + ((size_t)(mat == 0 ? j : n_kv + j) * D) * G;
      for (int e = tid; e < D * C::KPAD; e += 256) {
        const int n = e / C::KPAD, kap = e % C::KPAD;
        const int d = mat == 0 ? (n >> 1) + 64 * (n & 1) : n;  // keys: pair order
        const int cc = (kap & 7) >> 1, g = 8 * (kap >> 3) + cc + 4 * (kap & 1);
        const float w = g < G ? bf16_to_f32(src[(size_t)d * G + g]) : 0.f;
        const __half hv = __float2half_rn((cc & 1) ? w : 16.f * w);
        *reinterpret_cast<__half *>(dst + kmaj(n, kap, C::W_LBO)) = hv;
      }
      __syncthreads();
      if (tid < D) {
        // 8 sum_g W[d, g] over the fp16 values the MMA multiplies (factor 16 removed)
        float s = 0.f;
        for (int kap = 0; kap < C::KPAD; ++kap) {
          const int cc = (kap & 7) >> 1;
          const float v = __half2float(*reinterpret_cast<const __half *>(dst + kmaj(tid, kap, C::W_LBO)));
          s += (cc & 1) ? v : v * 0.0625f;
        }
        cd[tid] = 8.f * s;
      }
      __syncthreads();
    }
  }
  uint8_t *qd = qs + ((size_t)b * n_kv + j) * C::Q_BYTES;
  for (int e = tid; e < kNP * D; e += 256) {
    const int h = e / D, kap = e % D;
    const int d = (kap >> 1) + 64 * (kap & 1);
    const float v = h < grp ? bf16_to_f32(q[((size_t)b * n_q + (size_t)j * grp + h) * D + d]) * c : 0.f;
    *reinterpret_cast<__half *>(qd + kmaj(h, kap, C::Q_LBO)) = __float2half_rn(v);
  }
  pdl_wait();
  pdl_trigger();
}

}  // namespace x

template <int G, bool VEXP>
cudaError_t launch_expand_tc_t(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int n_new,
                               int64_t T, const int32_t *seq_lens, int n_q, int n_kv, const uint16_t *W_kv, float scale, int S,
                               int64_t tps, int rope, float rope_base, const uint16_t *gain, float eps, uint8_t *wk,
                               uint8_t *wv, float *ck, float *cv, uint8_t *qs, float *part, uint32_t *err,
                               MergeScratch msc, uint32_t stall_ns, void *const *prof, cudaStream_t st) {
  using C = x::XC<G, VEXP>;
  const int grp = n_q / n_kv;
  const float c = scale * kLog2e;
  const float pow2 = exp2f(floorf(log2f(c)));  // Q' = q 2^k holds the bf16 query exactly
  cudaError_t e = launch_pdl(x::expand_prep<G, VEXP>, dim3(n_kv, (unsigned)B), dim3(256), 0, st, q, W_kv, n_q, n_kv,
                             grp, pow2, wk, wv, ck, cv, qs, err, msc);
  if (e != cudaSuccess) return e;
  e = ensure_smem_limit((const void *)x::expand_split_tc<G, VEXP>, (size_t)C::SM_TOTAL);
  if (e != cudaSuccess) return e;
  x::XParams p{codes, bstride, T, tps, S, n_q, n_kv, grp, wk, wv, ck, cv, qs, gain, c / pow2, eps, rope_base, rope,
               part, err, seq_lens, stall_ns, n_new};
  CUtensorMap tmap;
  memset(&tmap, 0, sizeof(tmap));
  if constexpr (C::TMA) {
    e = make_code_tensor_map(&tmap, codes, bstride, T, B / n_new, C::HALF);
    if (e != cudaSuccess) return e;
  }
  record_prof_event(prof[0], st);
  e = launch_pdl(x::expand_split_tc<G, VEXP>, dim3(S, (unsigned)B, (unsigned)n_kv), dim3(C::THREADS),
                 (size_t)C::SM_TOTAL, st, tmap, p);
  record_prof_event(prof[1], st);
  return e;
}

}  // namespace tc

size_t expand_tc_stage_bytes(int G, int variant_expand) {
  const int kpad = (G + 15) / 16 * 16;
  return (size_t)128 * kpad * 2 * (variant_expand ? 2 : 1);
}

bool expand_tc_supported(int n_q, int n_kv, int G) {
  const int grp = n_kv > 0 ? n_q / n_kv : 0;
  return (G == 256 || G == 84) && n_kv > 0 && n_q % n_kv == 0 && grp >= 1 && grp <= tc::x::kMaxGrp;
}

cudaError_t merge_absorbed_launch(const float *part, int S, int64_t B, int n_q, int n_kv, int d_h, int G,
                                  const uint16_t *W_kv, void *o, int out_fp32, MergeScratch ms, cudaStream_t st,
                                  int fold_bytes);
cudaError_t merge_expand_launch(const float *part, int S, int64_t B, int n_q, int d_h, void *o, int out_fp32,
                                cudaStream_t st);

// Keys rebuilt per tile on the tensor cores; values pooled in latent space
// (hybrid, W_v applied by the merge) or rebuilt per tile as well (expand).
// B: grid rows (cache rows x n_new queries).
cudaError_t launch_expand_tc(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int n_new, int64_t T,
                             const int32_t *seq_lens, int n_q, int n_kv, int d_h, int G, const uint16_t *W_kv,
                             float scale, int S, int64_t tps, int hybrid, int rope, float rope_base,
                             const uint16_t *gain, float eps, uint8_t *wk, uint8_t *wv, float *ck, float *cv,
                             uint8_t *qs, float *part, uint32_t *err, MergeScratch ms, void *o, int out_fp32,
                             uint32_t stall_ns, void *const *prof, cudaStream_t st) {
  cudaError_t e;
#define FSQ_X_LAUNCH(GG, VV)                                                                                         \
  tc::launch_expand_tc_t<GG, VV>(q, codes, bstride, B, n_new, T, seq_lens, n_q, n_kv, W_kv, scale, S, tps, rope,    \
                                 rope_base, gain, eps, wk, wv, ck, cv, qs, part, err, ms, stall_ns, prof, st)
  if (G == 256) e = hybrid ? FSQ_X_LAUNCH(256, false) : FSQ_X_LAUNCH(256, true);
  else if (G == 84) e = hybrid ? FSQ_X_LAUNCH(84, false) : FSQ_X_LAUNCH(84, true);
  else return cudaErrorInvalidValue;
#undef FSQ_X_LAUNCH
  if (e != cudaSuccess) return e;
  if (hybrid) return merge_absorbed_launch(part, S, B, n_q, n_kv, d_h, G, W_kv, o, out_fp32, ms, st, 0);
  return merge_expand_launch(part, S, B, n_q, d_h, o, out_fp32, st);
}

}  // namespace fsq
