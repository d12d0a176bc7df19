// Append path on the 5th-generation tensor cores (prefill-sized token counts):
//   u = x E^T      bf16 operands, fp32 accumulation in TMEM   ([S] eq. 4)
//   level = #{k : u >= theta_k} - L/2, b-bit codes packed    ([S] eq. 2;
//   slide deck frames "A wide product code uses four bits per coordinate" and
//   "the grid size is an allocation choice": L = 4, 16, 256 at b = 2, 4, 8).
//
// Two kernels share the operand pipeline: warp 0 streams 64-wide slices of C
// of x and E into a ring of shared-memory stages by TMA (128-byte swizzle,
// rows past the tensor read as zero); one lane of warp 1 issues tcgen05.mma
// kind::f16 (bf16 x bf16 -> fp32) with both operands K-major in that swizzled
// layout.
//  - encode_pack_ks (G <= 256): a CTA owns 128 tokens x all coordinates of a
//    coordinate tile, over a slice of C; the CTAs of a thread-block cluster
//    add their partial sums through distributed shared memory (below).
//  - encode_pack_tc (wider G): a CTA owns 128 tokens x NC coordinates (NC =
//    64, 48, 32 or 16, whichever divides G rounded up to 16) over all of C;
//    after the last slice its four warps read their token rows of the
//    accumulator from TMEM, count thresholds and store the packed bytes.
// Every wait is bounded; a wait that gives up records FSQ_ERR_TIMEOUT in the
// caller's status word (if any), and the CTA lets its copies and MMAs finish
// (waits with their own fixed limit) and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "encode.cuh"
#include "tc_ptx.cuh"

namespace fsq {
namespace enc {

using namespace ptx;

constexpr int kM = 128;             // tokens per tile: MMA M, TMEM lanes
constexpr int kKc = 64;             // C elements per stage: one 128-byte swizzle row of bf16
constexpr int kStages = 6;
constexpr int kThreads = 128;
constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s per wait
constexpr uint64_t kDrainNs = 1000000000ull; // 1 s for in-flight copies and MMAs on the error path
constexpr int kABytes = kM * kKc * 2;        // x slice per stage

template <int NC>
struct ECfg {
  static constexpr int B_BYTES = NC * kKc * 2;  // E slice per stage
  static constexpr int STAGE = kABytes + B_BYTES;
  static constexpr int TMEM_COLS = NC <= 32 ? 32 : 64;
  static constexpr int SMEM = kStages * STAGE + 1024;  // + barriers; stages 1024-byte aligned
  static_assert(kABytes % 1024 == 0 && B_BYTES % 1024 == 0, "swizzled tiles must stay 1024-byte aligned");
};

struct EncMisc {
  uint64_t full[kStages], empty[kStages], done, never;
  uint32_t tmem_base;
  uint32_t abort;
};

// Shared-memory matrix descriptor, K-major, 128-byte swizzle (8-row atoms of
// 128 bytes, 1024 bytes apart): start address, stride-dimension offset 1024,
// descriptor version 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;             // leading-dimension offset (not used by swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;   // stride-dimension offset: next 8-row atom
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Bounded wait (gives up after kWaitNs or once *abort is set).
__device__ __forceinline__ bool wait_ok(uint64_t *b, uint32_t parity, volatile uint32_t *abort) {
  return mbar_wait(b, parity, abort, kWaitNs);
}

// Code of u against L-1 sorted thresholds held in shared memory: a
// branchless binary search for #{k : u >= th[k]} (NaN counts none), log2(L)
// load-compare-select steps instead of L-1 compares.  The running index is
// kept in bytes so that each step's load takes its offset as an immediate.
template <int L>
__device__ __forceinline__ uint32_t fsq_code_smem(float u, const float *th) {
  const uint8_t *tb = reinterpret_cast<const uint8_t *>(th);
  uint32_t nb = 0;  // 4 x code so far
#pragma unroll
  for (uint32_t step = L / 2; step; step >>= 1)
    nb += (u >= *reinterpret_cast<const float *>(tb + nb + 4 * (step - 1))) ? 4 * step : 0u;  // index <= L - 2
  return nb >> 2;
}

// Codes of 16 consecutive coordinates of one token (fp32 u as bits in v),
// packed b bits each and stored at dst; nvalid of them lie inside G.  The
// thresholds are the kernel parameter (th) or, when ths is given, their copy
// in shared memory.
template <int L>
__device__ __forceinline__ void pack_store16(const uint32_t (&v)[16], const Thresholds<L> &th, uint8_t *dst,
                                             int nvalid, const float *ths = nullptr) {
  constexpr int BITS = bits_of_levels(L);
  constexpr int WORDS = 16 * BITS / 32;  // 32-bit words of packed codes per 16 coordinates
  uint32_t w[WORDS];
#pragma unroll
  for (int k = 0; k < WORDS; ++k) w[k] = 0u;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const uint32_t code =
        ths ? fsq_code_smem<L>(__uint_as_float(v[e]), ths) : fsq_code<L>(__uint_as_float(v[e]), th);
    w[e * BITS / 32] |= code << ((e * BITS) % 32);
  }
  if (nvalid == 16 && ((reinterpret_cast<uintptr_t>(dst) & (4u * WORDS - 1u)) == 0)) {
    if constexpr (WORDS == 1) *reinterpret_cast<uint32_t *>(dst) = w[0];
    else if constexpr (WORDS == 2) *reinterpret_cast<uint2 *>(dst) = make_uint2(w[0], w[1]);
    else *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    // a ragged last group (nvalid a multiple of 8 / BITS) or an unaligned row
    for (int bb = 0; bb < nvalid * BITS / 8; ++bb) dst[bb] = (uint8_t)(w[bb / 4] >> (8 * (bb % 4)));
  }
}

template <int NC, int L>
__global__ void __launch_bounds__(kThreads, 1)
    encode_pack_tc(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap te, int64_t n_tok,
                   int64_t C, int G, const __grid_constant__ Thresholds<L> th, const CodeRows dst,
                   uint32_t *status, uint32_t stall_ns) {
  using EC = ECfg<NC>;
  extern __shared__ __align__(1024) uint8_t esm[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(esm) + 1023) & ~uintptr_t(1023));
  EncMisc &ms = *reinterpret_cast<EncMisc *>(sm + kStages * EC::STAGE);
  volatile uint32_t *abort = &ms.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * NC;                // first coordinate of this tile
  const int64_t m0 = (int64_t)blockIdx.y * kM;   // first token of this tile
  const int nk = (int)(C / kKc);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ms.full[s], 1);
      mbar_init(&ms.empty[s], 1);
    }
    mbar_init(&ms.done, 1);
    mbar_init(&ms.never, 1);  // completed by nothing: the test-only stall waits on it
    ms.abort = 0u;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&ms.tmem_base, EC::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ms.tmem_base;
  auto fail = [&]() {
    if (status) atomicCAS(status, 0u, (uint32_t)(-FSQ_ERR_TIMEOUT));
    *abort = 1u;
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      for (int c = 0; c < nk; ++c) {
        const int s = c % kStages;
        if (!wait_ok(&ms.empty[s], ((uint32_t)(c / kStages) & 1u) ^ 1u, abort)) {
          ok = false;
          break;
        }
        uint8_t *a = sm + s * EC::STAGE;
        mbar_arrive_expect_tx(&ms.full[s], EC::STAGE);
        tma_load_2d(a, &tx, c * kKc, (int)m0, &ms.full[s]);
        tma_load_2d(a + kABytes, &te, c * kKc, n0, &ms.full[s]);
        issued = c + 1;
      }
      if (!ok) {
        fail();
        // let the copies in flight land before the CTA exits
        for (int c = max(0, issued - kStages); c < issued; ++c)
          mbar_wait_fixed(&ms.full[c % kStages], (uint32_t)(c / kStages) & 1u, kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id = idesc_bf16(kM, NC);
      bool ok = true;
      for (int c = 0; c < nk && ok; ++c) {
        const int s = c % kStages;
        if (!wait_ok(&ms.full[s], (uint32_t)(c / kStages) & 1u, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t da = desc_sw128(smem_u32(sm + s * EC::STAGE));
        const uint64_t db = desc_sw128(smem_u32(sm + s * EC::STAGE + kABytes));
#pragma unroll
        for (int k = 0; k < kKc / 16; ++k)  // K = 16 per MMA: 32 bytes along the swizzled row
          mma_ss(tm, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), id, (c > 0 || k > 0) ? 1u : 0u);
        tc_commit(&ms.empty[s]);
      }
      if (!ok) fail();
      tc_commit(&ms.done);
    }
  }
  // ---------------------------------------------------------------- epilogue: all four warps
  __syncwarp();
  // test-only stall: a wait that runs out on purpose (nothing completes `never`)
  if (stall_ns != 0u && !mbar_wait(&ms.never, 0, abort, stall_ns) && lane == 0) fail();
  __syncwarp();
  // the MMAs must be complete before TMEM is read or freed, error or not: this
  // wait ignores the abort flag and keeps its own limit
  const bool ok = mbar_wait_fixed(&ms.done, 0, kDrainNs) && *abort == 0u;
  if (!ok) {
    if (lane == 0) fail();
  } else {
    tc_fence_after();
    const int64_t row = m0 + 32 * warp + lane;  // this thread's token: TMEM lane 32 warp + lane
    const uint32_t tl = tm + ((uint32_t)(32 * warp) << 16);
    constexpr int BITS = bits_of_levels(L);
#pragma unroll
    for (int j0 = 0; j0 < NC; j0 += 16) {
      uint32_t v[16];
      tmem_ld16(tl + j0, v);
      tmem_ld_wait();
      if (row < n_tok) pack_store16<L>(v, th, dst.row(row) + (n0 + j0) * BITS / 8, min(16, G - (n0 + j0)));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, EC::TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
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

// 2-D bf16 tensor [rows][cols] with the given row stride (elements), box
// {kKc, box_rows}, 128-byte swizzle; reads outside the tensor return zero.
cudaError_t make_bf16_map(CUtensorMap *map, const uint16_t *base, int64_t rows, int64_t cols, int64_t ld,
                          int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kKc, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(base), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int NC, int L>
cudaError_t launch_nc(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C, const uint16_t *E, int G,
                      const Thresholds<L> &th, const CodeRows &dst, uint32_t *status, uint32_t stall_ns,
                      cudaStream_t s) {
  using EC = ECfg<NC>;
  CUtensorMap tx, te;
  cudaError_t e = make_bf16_map(&tx, x, n_tok, C, ldx, kM);
  if (e != cudaSuccess) return e;
  e = make_bf16_map(&te, E, G, C, C, NC);
  if (e != cudaSuccess) return e;
  e = ensure_smem_limit((const void *)encode_pack_tc<NC, L>, EC::SMEM);
  if (e != cudaSuccess) return e;
  const int gp = (G + 15) / 16 * 16;
  const dim3 grid((unsigned)(gp / NC), (unsigned)((n_tok + kM - 1) / kM));
  encode_pack_tc<NC, L><<<grid, kThreads, EC::SMEM, s>>>(tx, te, n_tok, C, G, th, dst, status, stall_ns);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// K-split form for G <= 256: one CTA computes every coordinate of a
// coordinate tile for its 128 tokens (MMA N = TN: G rounded up to 16, or half
// of that past 128 coordinates, see tn_of) over a slice of C, and the ks CTAs
// of a thread-block cluster (one per slice of C) add their fp32 partial sums
// through distributed shared memory.  The operand bytes a CTA streams per
// output fall from (1/64 + 1/128) to (1/TN + 1/128) of a C-long row pair,
// while the split of C keeps as many SMs busy as a split into 64-wide
// coordinate tiles would.
//
// CTA rank r owns the 16-column groups g = r, r + ks, ... of the tile.  Once
// every CTA of the cluster has finished its MMAs (cluster barrier A: the
// operand rings are spent), each CTA copies the groups it does not own from
// TMEM into one staging block per peer in its own shared memory, and one
// thread sends each block to its peer with a bulk copy (one transfer per
// peer, rather than a 16-byte store per thread and chunk) that completes on
// the peer's receive mbarrier.  The owner waits for its ks - 1 blocks
// (bounded), adds its groups' ks partials in rank order, its own straight
// from TMEM (a fixed summation order: the result does not depend on timing),
// quantises, packs and stores.  Cluster barrier C keeps every CTA resident
// until all copies have landed, so none reads a staging block of a CTA that
// has left.  Every CTA sends its blocks and passes both cluster barriers
// exactly once, error or not: a CTA whose bounded waits gave up publishes
// that in a flag before barrier A, and no CTA of the cluster then stores
// codes of that tile.  With ks = 1 the accumulator is quantised straight
// from TMEM.

template <int TN>
struct KsCfg {
  static constexpr int B_BYTES = TN * kKc * 2;  // E slice per stage (all TN rows)
  static constexpr int STAGE = kABytes + B_BYTES;
  static constexpr int STAGES = (200 * 1024 / STAGE) < 8 ? (200 * 1024 / STAGE) : 8;
  static constexpr int RING = STAGES * STAGE;
  static constexpr int NG = TN / 16;            // 16-column groups of the tile
  static constexpr int GB = kM * 64;            // one group of the partial: 128 rows x 16 fp32
  // staging (ks - 1 outgoing blocks) + receive area (ks - 1 incoming blocks)
  static constexpr int xch(int ks) { return 2 * (ks - 1) * ((NG + ks - 1) / ks) * GB; }
  static constexpr int XCH = xch(8) > xch(4) ? (xch(8) > xch(2) ? xch(8) : xch(2)) : (xch(4) > xch(2) ? xch(4) : xch(2));
  static constexpr int BODY = RING > XCH ? RING : XCH;
  static constexpr int TMEM_COLS = TN <= 32 ? 32 : TN <= 64 ? 64 : TN <= 128 ? 128 : 256;
  static constexpr int SMEM = BODY + 1024 + 1280;  // + alignment slack, barriers and thresholds
  static_assert(TN % 16 == 0 && TN >= 16 && TN <= 256, "MMA N for M = 128");
  static_assert(STAGES >= 2 && kABytes % 1024 == 0 && B_BYTES % 1024 == 0, "ring of 1024-byte aligned stages");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

constexpr int kKsThreads = 512;  // 16 warps: four per TMEM lane quarter share the epilogue's groups

struct KsMisc {
  uint64_t full[8], empty[8], done, never, rx;
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t ok;  // read by the cluster's other CTAs
  float th[kMaxLevels];  // the thresholds, for the epilogue's binary search
};
static_assert(sizeof(KsMisc) <= 1280, "barriers and thresholds fit their reserve");

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in cluster rank `rank`.
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Bulk copy of `bytes` (a multiple of 16) from this CTA's shared memory to a
// cluster peer's, completing `bytes` transactions on the peer's mbarrier.
__device__ __forceinline__ void bulk_to_peer(uint32_t dst_cluster, uint32_t src_cta, uint32_t bytes,
                                             uint32_t mbar_cluster) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   dst_cluster),
               "r"(src_cta), "r"(bytes), "r"(mbar_cluster)
               : "memory");
}
// Byte offset of 16-byte chunk c (0..3) of row r in a group block: rows of 64
// bytes, chunks XOR-swizzled by row so that the 16-byte accesses of eight
// consecutive rows hit distinct banks.
__device__ __forceinline__ uint32_t gb_off(int r, int c) { return (uint32_t)(64 * r + ((c ^ ((r >> 1) & 3)) << 4)); }
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t caddr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(caddr) : "memory");
  return v;
}
// Whole-cluster barrier: every thread of every CTA arrives (release) and waits (acquire).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int TN, int L>
__global__ void __launch_bounds__(kKsThreads, 1)
    encode_pack_ks(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap te, int64_t n_tok,
                   int64_t C, int G, const __grid_constant__ Thresholds<L> th, const CodeRows dst,
                   uint32_t *status, uint32_t stall_ns) {
  using KC = KsCfg<TN>;
  extern __shared__ __align__(1024) uint8_t esm[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(esm) + 1023) & ~uintptr_t(1023));
  KsMisc &ms = *reinterpret_cast<KsMisc *>(sm + KC::BODY);
  volatile uint32_t *abort = &ms.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();           // slice of C (the cluster spans gridDim.x)
  const uint32_t ks = gridDim.x;
  const int64_t m0 = (int64_t)blockIdx.y * kM;    // first token of this tile
  const int n0 = (int)blockIdx.z * TN;            // first coordinate of this tile
  const int Gt = G - n0;                          // coordinates of G inside this tile (may exceed TN)
  const int nk = (int)(C / kKc);
  const int k0 = (int)((int64_t)rank * nk / ks), k1 = (int)((int64_t)(rank + 1) * nk / ks);  // k1 > k0: ks <= nk

  if (threadIdx.x == 0) {
    for (int st = 0; st < KC::STAGES; ++st) {
      mbar_init(&ms.full[st], 1);
      mbar_init(&ms.empty[st], 1);
    }
    mbar_init(&ms.done, 1);
    mbar_init(&ms.never, 1);  // completed by nothing: the test-only stall waits on it
    mbar_init(&ms.rx, 1);     // the peers' partials landing in this CTA
    ms.abort = 0u;
    ms.ok = 0u;
    fence_mbar_init();
  }
  for (int k = threadIdx.x; k < L - 1; k += kKsThreads) ms.th[k] = th.th[k];
  if (warp == 0) {
    tmem_alloc(&ms.tmem_base, KC::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ms.tmem_base;
  auto fail = [&]() {
    if (status) atomicCAS(status, 0u, (uint32_t)(-FSQ_ERR_TIMEOUT));
    *abort = 1u;
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      for (int c = k0; c < k1; ++c) {
        const int i = c - k0, st = i % KC::STAGES;
        if (!wait_ok(&ms.empty[st], ((uint32_t)(i / KC::STAGES) & 1u) ^ 1u, abort)) {
          ok = false;
          break;
        }
        uint8_t *a = sm + st * KC::STAGE;
        mbar_arrive_expect_tx(&ms.full[st], KC::STAGE);
        tma_load_2d(a, &tx, c * kKc, (int)m0, &ms.full[st]);
        tma_load_2d(a + kABytes, &te, c * kKc, n0, &ms.full[st]);
        issued = i + 1;
      }
      if (!ok) {
        fail();
        // let the copies in flight land before the ring is reused or the CTA exits
        for (int i = max(0, issued - KC::STAGES); i < issued; ++i)
          mbar_wait_fixed(&ms.full[i % KC::STAGES], (uint32_t)(i / KC::STAGES) & 1u, kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id = idesc_bf16(kM, TN);
      bool ok = true;
      for (int c = k0; c < k1 && ok; ++c) {
        const int i = c - k0, st = i % KC::STAGES;
        if (!wait_ok(&ms.full[st], (uint32_t)(i / KC::STAGES) & 1u, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t da = desc_sw128(smem_u32(sm + st * KC::STAGE));
        const uint64_t db = desc_sw128(smem_u32(sm + st * KC::STAGE + kABytes));
#pragma unroll
        for (int k = 0; k < kKc / 16; ++k)  // K = 16 per MMA: 32 bytes along the swizzled row
          mma_ss(tm, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), id, (i > 0 || k > 0) ? 1u : 0u);
        tc_commit(&ms.empty[st]);
      }
      if (!ok) fail();
      tc_commit(&ms.done);
    }
  }
  // ---------------------------------------------------------------- epilogue: all four warps
  __syncwarp();
  // test-only stall: a wait that runs out on purpose (nothing completes `never`)
  if (stall_ns != 0u && !mbar_wait(&ms.never, 0, abort, stall_ns) && lane == 0) fail();
  __syncwarp();
  // the MMAs must be complete before TMEM is read or freed, or the ring is
  // overwritten, error or not: this wait ignores the abort flag and keeps its
  // own limit
  const bool done = mbar_wait_fixed(&ms.done, 0, kDrainNs);
  const bool ok = __syncthreads_and(done && *abort == 0u) != 0;
  if (!ok && threadIdx.x == 0) fail();
  constexpr int BITS = bits_of_levels(L);
  constexpr int NPART = kKsThreads / 128;  // warps that share one TMEM lane quarter
  const int quarter = warp & 3, part = warp >> 2;
  const int r = 32 * quarter + lane;  // this thread's token row: TMEM lane r
  const int64_t row = m0 + r;
  const uint32_t tl = tm + ((uint32_t)(32 * quarter) << 16);
  if (ks == 1) {
    if (ok) {
      tc_fence_after();
      for (int g = part; g < KC::NG && 16 * g < Gt; g += NPART) {
        uint32_t v[16];
        tmem_ld16(tl + 16 * g, v);
        tmem_ld_wait();
        if (row < n_tok)
          pack_store16<L>(v, th, dst.row(row) + (n0 + 16 * g) * BITS / 8, min(16, Gt - 16 * g), ms.th);
      }
    }
  } else {
    const int J = (KC::NG + (int)ks - 1) / (int)ks;  // groups per owner
    const uint32_t blk = (uint32_t)J * KC::GB;      // bytes one CTA sends one peer
    uint8_t *stage = sm;                            // ks - 1 outgoing blocks, by peer
    uint8_t *rbuf = sm + (size_t)(ks - 1) * blk;    // ks - 1 incoming blocks, by source
    if (threadIdx.x == 0) {
      ms.ok = ok ? 1u : 0u;
      mbar_arrive_expect_tx(&ms.rx, (ks - 1) * blk);
    }
    cluster_sync_all();  // A: every CTA's MMAs are done (its ring is free) and its flag is set
    const uint32_t peer_ok = lane < (int)ks ? ld_cluster_u32(map_rank(smem_u32(&ms.ok), (uint32_t)lane)) : 1u;
    if (ok) {
      // this warp's groups g = part + NPART i: all TMEM loads first, one wait,
      // then the groups other ranks own into their staging blocks
      constexpr int GI = (KC::NG + NPART - 1) / NPART;
      uint32_t v[GI][16];
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < GI; ++i)
        if (part + NPART * i < KC::NG) tmem_ld16(tl + 16 * (part + NPART * i), v[i]);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < GI; ++i) {
        const int g = part + NPART * i;
        if (g >= KC::NG || 16 * g >= Gt) break;
        const int own = g % (int)ks;
        if (own == (int)rank) continue;  // kept in TMEM
        const int qi = own < (int)rank ? own : own - 1;
        uint8_t *gb = stage + (size_t)qi * blk + (size_t)(g / (int)ks) * KC::GB;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4 *>(gb + gb_off(r, c)) = make_uint4(v[i][4 * c], v[i][4 * c + 1], v[i][4 * c + 2],
                                                                      v[i][4 * c + 3]);
      }
    }
    fence_proxy_async_smem();  // the staging blocks are read by the bulk copies
    __syncthreads();
    if (threadIdx.x == 0) {
      for (uint32_t q = 0; q < ks; ++q) {
        if (q == rank) continue;
        const uint32_t qi = q < rank ? q : q - 1;         // my block for peer q
        const uint32_t si = rank < q ? rank : rank - 1;   // my slot in peer q's receive area
        bulk_to_peer(map_rank(smem_u32(rbuf + (size_t)si * blk), q), smem_u32(stage + (size_t)qi * blk), blk,
                     map_rank(smem_u32(&ms.rx), q));
      }
    }
    // every block sent to this CTA must land before it reads them or leaves:
    // this wait ignores the abort flag and keeps its own limit
    const bool rx_ok = mbar_wait_fixed(&ms.rx, 0, kDrainNs);
    const bool flags_ok = __all_sync(0xffffffffu, peer_ok != 0u);  // the same in every warp
    const bool all_ok = __syncthreads_and(rx_ok && flags_ok) != 0;
    if (!rx_ok && threadIdx.x == 0) fail();
    if (all_ok) {
      tc_fence_after();
      for (int j = part; j < J; j += NPART) {
        const int g = (int)rank + j * (int)ks;
        if (g >= KC::NG || 16 * g >= Gt) break;
        uint32_t vo[16];
        tmem_ld16(tl + 16 * g, vo);
        tmem_ld_wait();
        float acc[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = 0.f;
        for (int src = 0; src < (int)ks; ++src) {  // rank order: a fixed summation order
          if (src == (int)rank) {
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[e] += __uint_as_float(vo[e]);
          } else {
            const int si = src < (int)rank ? src : src - 1;
            const uint8_t *gb = rbuf + (size_t)si * blk + (size_t)j * KC::GB;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float4 t = *reinterpret_cast<const float4 *>(gb + gb_off(r, c));
              acc[4 * c] += t.x;
              acc[4 * c + 1] += t.y;
              acc[4 * c + 2] += t.z;
              acc[4 * c + 3] += t.w;
            }
          }
        }
        if (row < n_tok) {
          uint32_t v[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(acc[e]);
          pack_store16<L>(v, th, dst.row(row) + (n0 + 16 * g) * BITS / 8, min(16, Gt - 16 * g), ms.th);
        }
      }
    }
    cluster_sync_all();  // C: all copies have landed, so no CTA's staging blocks are still being read
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, KC::TMEM_COLS);
  }
}

// Cluster size: the largest power of two <= 8 (and <= the 64-wide slices of
// C) that keeps the grid (token tiles x coordinate tiles x ks) within one CTA
// per SM of a 148-SM part.
inline int ks_of(int64_t n_tiles, int64_t nk) {
  int ks = 1;
  while (ks < 8 && n_tiles * 2 * ks <= 148 && 2 * ks <= nk) ks *= 2;
  return ks;
}
// Coordinate tiles: a split of C costs distributed-shared-memory traffic
// ((ks - 1) / ks of a 128 x TN fp32 partial per CTA, at a few tens of GB/s
// per SM), a split of G costs a second read of x from DRAM.  At 4096 tokens
// and G = 256 two coordinate tiles with ks = 2 beat one with ks = 4 (22.3
// against 23.7 us), so past 128 coordinates the tile is halved (TN = 16 *
// ceil(GP / 32)) while the doubled grid still fits one wave; beyond that the
// whole width stays in one tile.
inline int tn_of(int gp, int64_t n_tiles) { return gp >= 128 && 2 * n_tiles <= 148 ? 16 * ((gp + 31) / 32) : gp; }

template <int TN, int L>
cudaError_t launch_ks(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C, const uint16_t *E, int G,
                      const Thresholds<L> &th, const CodeRows &dst, uint32_t *status, uint32_t stall_ns,
                      cudaStream_t s) {
  using KC = KsCfg<TN>;
  CUtensorMap tx, te;
  cudaError_t e = make_bf16_map(&tx, x, n_tok, C, ldx, kM);
  if (e != cudaSuccess) return e;
  e = make_bf16_map(&te, E, G, C, C, TN);  // rows past G (last coordinate tile) read as zero
  if (e != cudaSuccess) return e;
  e = ensure_smem_limit((const void *)encode_pack_ks<TN, L>, KC::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t n_tiles = (n_tok + kM - 1) / kM;
  const int nz = (G + TN - 1) / TN;  // coordinate tiles
  const int ks = ks_of(n_tiles * nz, C / kKc);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ks, (unsigned)n_tiles, (unsigned)nz);
  cfg.blockDim = dim3(kKsThreads);
  cfg.dynamicSmemBytes = KC::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)ks;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, encode_pack_ks<TN, L>, tx, te, n_tok, C, G, th, dst, status, stall_ns);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int L>
cudaError_t launch_ks_g(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C, const uint16_t *E, int G,
                        const Thresholds<L> &th, const CodeRows &dst, uint32_t *status, uint32_t stall_ns,
                        cudaStream_t s) {
  switch (tn_of((G + 15) / 16 * 16, (n_tok + kM - 1) / kM) / 16) {
#define FSQ_KS_CASE(n) \
  case n:              \
    return launch_ks<16 * n, L>(x, n_tok, ldx, C, E, G, th, dst, status, stall_ns, s);
    FSQ_KS_CASE(1) FSQ_KS_CASE(2) FSQ_KS_CASE(3) FSQ_KS_CASE(4) FSQ_KS_CASE(5) FSQ_KS_CASE(6) FSQ_KS_CASE(7)
    FSQ_KS_CASE(8) FSQ_KS_CASE(9) FSQ_KS_CASE(10) FSQ_KS_CASE(11) FSQ_KS_CASE(12) FSQ_KS_CASE(13)
    FSQ_KS_CASE(14) FSQ_KS_CASE(15) FSQ_KS_CASE(16)
#undef FSQ_KS_CASE
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace enc

// Tensor-core append for n_tok tokens; C a multiple of 64, G even <= FSQ_MAX_G
// (a multiple of 4 at L = 4).
template <int L>
cudaError_t launch_encode_pack_tc(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C, const uint16_t *E, int G,
                                  const Thresholds<L> &th, const CodeRows &dst, uint32_t *status,
                                  uint32_t stall_ns, cudaStream_t s) {
  if (n_tok > (int64_t)65535 * enc::kM || C > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int gp = (G + 15) / 16 * 16;
  if (gp <= 256) return enc::launch_ks_g<L>(x, n_tok, ldx, C, E, G, th, dst, status, stall_ns, s);
  if (gp % 64 == 0) return enc::launch_nc<64, L>(x, n_tok, ldx, C, E, G, th, dst, status, stall_ns, s);
  if (gp % 48 == 0) return enc::launch_nc<48, L>(x, n_tok, ldx, C, E, G, th, dst, status, stall_ns, s);
  if (gp % 32 == 0) return enc::launch_nc<32, L>(x, n_tok, ldx, C, E, G, th, dst, status, stall_ns, s);
  return enc::launch_nc<16, L>(x, n_tok, ldx, C, E, G, th, dst, status, stall_ns, s);
}
template cudaError_t launch_encode_pack_tc<4>(const uint16_t *, int64_t, int64_t, int64_t, const uint16_t *, int,
                                              const Thresholds<4> &, const CodeRows &, uint32_t *, uint32_t,
                                              cudaStream_t);
template cudaError_t launch_encode_pack_tc<16>(const uint16_t *, int64_t, int64_t, int64_t, const uint16_t *, int,
                                               const Thresholds<16> &, const CodeRows &, uint32_t *, uint32_t,
                                               cudaStream_t);
template cudaError_t launch_encode_pack_tc<256>(const uint16_t *, int64_t, int64_t, int64_t, const uint16_t *, int,
                                                const Thresholds<256> &, const CodeRows &, uint32_t *, uint32_t,
                                                cudaStream_t);

}  // namespace fsq
