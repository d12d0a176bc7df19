// Append path on the 5th-generation tensor cores (prefill-sized token counts):
//   u = x E^T      bf16 operands, fp32 accumulation in TMEM   ([S] eq. 4)
//   level = #{k : u >= theta_k} - L/2, b-bit codes packed    ([S] eq. 2;
//   slide deck frames "A wide product code uses four bits per coordinate" and
//   "the grid size is an allocation choice": L = 4, 16, 256 at b = 2, 4, 8).
//
// One CTA computes a tile of 128 tokens x NC coordinates (NC = 64, 48, 32 or
// 16, whichever divides G rounded up to 16), so that a prefill chunk spreads
// over many SMs.  Warp 0 streams 64-wide slices of C of x and E into a ring of
// shared-memory stages by TMA (128-byte swizzle, rows past the tensor read as
// zero); one lane of warp 1 issues tcgen05.mma kind::f16 (bf16 x bf16 -> fp32)
// with both operands K-major in that swizzled layout; after the last slice
// all four warps read their 32 token rows of the accumulator from TMEM, count
// thresholds and store the packed bytes.  Every wait is bounded; a wait that
// gives up records FSQ_ERR_TIMEOUT in the caller's status word (if any), and
// the CTA lets its copies and MMAs finish (waits with their own fixed limit)
// and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
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

template <int NC, int L>
__global__ void __launch_bounds__(kThreads, 1)
    encode_pack_tc(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap te, int64_t n_tok,
                   int64_t C, int G, const __grid_constant__ Thresholds<L> th, uint8_t *__restrict__ codes,
                   int64_t ldc, uint32_t *status, uint32_t stall_ns) {
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
    constexpr int WORDS = 16 * BITS / 32;  // 32-bit words of packed codes per 16 coordinates
#pragma unroll
    for (int j0 = 0; j0 < NC; j0 += 16) {
      uint32_t v[16];
      tmem_ld16(tl + j0, v);
      tmem_ld_wait();
      if (row < n_tok) {
        uint8_t *dst = codes + row * ldc + (n0 + j0) * BITS / 8;
        uint32_t w[WORDS];
#pragma unroll
        for (int k = 0; k < WORDS; ++k) w[k] = 0u;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const uint32_t code = fsq_code<L>(__uint_as_float(v[e]), th);
          w[e * BITS / 32] |= code << ((e * BITS) % 32);
        }
        const int nvalid = min(16, G - (n0 + j0));  // coordinates of this group inside G
        if (nvalid == 16 && ((reinterpret_cast<uintptr_t>(dst) & (4u * WORDS - 1u)) == 0)) {
          if constexpr (WORDS == 1) *reinterpret_cast<uint32_t *>(dst) = w[0];
          else if constexpr (WORDS == 2) *reinterpret_cast<uint2 *>(dst) = make_uint2(w[0], w[1]);
          else *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
          // a ragged last group (nvalid a multiple of 8 / BITS) or an unaligned row
          for (int bb = 0; bb < nvalid * BITS / 8; ++bb) dst[bb] = (uint8_t)(w[bb / 4] >> (8 * (bb % 4)));
        }
      }
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
                      const Thresholds<L> &th, uint8_t *codes, int64_t ldc, uint32_t *status, uint32_t stall_ns,
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
  encode_pack_tc<NC, L><<<grid, kThreads, EC::SMEM, s>>>(tx, te, n_tok, C, G, th, codes, ldc, status, stall_ns);
  return cudaGetLastError();
}

}  // namespace enc

// Tensor-core append for n_tok tokens; C a multiple of 64, G even <= FSQ_MAX_G
// (a multiple of 4 at L = 4).
template <int L>
cudaError_t launch_encode_pack_tc(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C, const uint16_t *E, int G,
                                  const Thresholds<L> &th, uint8_t *codes, int64_t ldc, uint32_t *status,
                                  uint32_t stall_ns, cudaStream_t s) {
  if (n_tok > (int64_t)65535 * enc::kM || C > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int gp = (G + 15) / 16 * 16;
  if (gp % 64 == 0) return enc::launch_nc<64, L>(x, n_tok, ldx, C, E, G, th, codes, ldc, status, stall_ns, s);
  if (gp % 48 == 0) return enc::launch_nc<48, L>(x, n_tok, ldx, C, E, G, th, codes, ldc, status, stall_ns, s);
  if (gp % 32 == 0) return enc::launch_nc<32, L>(x, n_tok, ldx, C, E, G, th, codes, ldc, status, stall_ns, s);
  return enc::launch_nc<16, L>(x, n_tok, ldx, C, E, G, th, codes, ldc, status, stall_ns, s);
}
template cudaError_t launch_encode_pack_tc<4>(const uint16_t *, int64_t, int64_t, int64_t, const uint16_t *, int,
                                              const Thresholds<4> &, uint8_t *, int64_t, uint32_t *, uint32_t,
                                              cudaStream_t);
template cudaError_t launch_encode_pack_tc<16>(const uint16_t *, int64_t, int64_t, int64_t, const uint16_t *, int,
                                               const Thresholds<16> &, uint8_t *, int64_t, uint32_t *, uint32_t,
                                               cudaStream_t);
template cudaError_t launch_encode_pack_tc<256>(const uint16_t *, int64_t, int64_t, int64_t, const uint16_t *, int,
                                                const Thresholds<256> &, uint8_t *, int64_t, uint32_t *, uint32_t,
                                                cudaStream_t);

}  // namespace fsq
