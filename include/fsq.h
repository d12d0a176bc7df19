/*
 * fsq.h — C ABI of the B200 (sm_100a) library for Transformer-FSQ's decode
 * hot path: appending tokens to a KV cache that holds only bit-packed FSQ
 * latent codes (4-bit nibbles at the default 16 levels; 2- and 8-bit codes at
 * 4 and 256 levels), and single-token grouped-query attention read directly
 * from those codes through the shared decoder W_kv.
 *
 * Sources (page titles):
 *  [S] "Transformer-FSQ: Discrete Latents for Extreme KV-Cache Compression",
 *      picx.dev summary — Theoretical Basis (eq. 2), Methodology/Architecture
 *      (eqs. 4, 5), Key Design Innovation (eq. 6), Closed-Form Conversion
 *      (eq. 8, row order of W_kv), Byte Budgeting.
 *  [D] Transformer-FSQ slide deck — frames "A wide product code uses four
 *      bits per coordinate" (L=16, b=4, h=7.5075, delta=0.5, ceil(G*b/8)
 *      bytes per token), "Attention pools codes before decoding values"
 *      (eqs. 5-6), "The kernel reads codes and never writes reconstructed
 *      K/V" (read codes, unpack in registers, tensor cores, online softmax,
 *      merge partials, apply W_v once).
 *
 * Conventions shared by every call
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates device memory at run time and never synchronises the
 *    host (except the status readers, which say so).  It keeps no state
 *    between calls; its only device memory of its own is the scratch of
 *    fsq_decode_attn_noalloc (a file-scope array of the library).
 *  - bf16 means IEEE bfloat16 stored as uint16; row-major throughout.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default).
 *  - Argument errors are returned synchronously, before anything is
 *    launched.  A failed launch returns FSQ_ERR_CUDA.  A bounded device-side
 *    wait that gives up records FSQ_ERR_TIMEOUT in a caller-owned status word
 *    (decode: the workspace's error word; append: fsq_encode_opts.status_word;
 *    read either with fsq_workspace_status) instead of hanging or trapping.
 *  - The decode kernels use programmatic dependent launch: the first of
 *    them may start before the kernel preceding the call on the stream has
 *    finished, and reads q and W_kv early.  If that kernel is itself a
 *    programmatic-launch primary (it executes griddepcontrol.launch_dependents)
 *    it must not write q or W_kv.  Ordinary kernels are unaffected.
 *
 * Cache format (FSQ_FORMAT_VERSION 1)
 *  - L levels per coordinate (L = 16 by default; 4 and 256 also supported,
 *    [D] backup frame "the grid size is an allocation choice", Table 8), so
 *    b = log2(L) bits per coordinate.  A token's G levels z_i in
 *    {-L/2 .. L/2-1} are stored as codes n_i = z_i + L/2 of b bits.  Byte k
 *    of the token's row holds coordinates k*(8/b) .. k*(8/b) + 8/b - 1, the
 *    first in its lowest b bits.  At L = 16: coordinate 2i in the low nibble
 *    of byte i and coordinate 2i+1 in its high nibble; at L = 256 one byte per
 *    coordinate; at L = 4 four coordinates per byte.
 *  - A row is exactly R = G*b/8 bytes; no scale, zero point or norm is stored
 *    ([S] Summary; [D] product-code frame: ceil(G*b/8) bytes per token).
 *  - A layer's cache is [B, T_max, R] bytes; row t of batch b starts at
 *    codes + b*code_batch_stride_bytes + t*R.
 */
#ifndef FSQ_H_
#define FSQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FSQ_FORMAT_VERSION 1
#define FSQ_LEVELS 16   /* default level count (levels field 0) */
#define FSQ_MAX_G 576   /* widest latent: Table 8's 144 B/token at L = 4 */
#define FSQ_HEAD_DIM 128

#if defined(__GNUC__)
#define FSQ_API __attribute__((visibility("default")))
#else
#define FSQ_API
#endif

typedef struct CUstream_st *fsq_stream_t; /* same type as cudaStream_t */

typedef enum {
  FSQ_OK = 0,
  FSQ_ERR_INVALID_ARG = -1, /* null pointer, bad size, bad parameter */
  FSQ_ERR_UNSUPPORTED = -2, /* valid request outside the supported shapes */
  FSQ_ERR_MISALIGNED = -3,  /* pointer or stride not 16-byte aligned */
  FSQ_ERR_WORKSPACE = -4,   /* workspace missing or too small */
  FSQ_ERR_CUDA = -5,        /* a CUDA launch or runtime call failed */
  FSQ_ERR_TIMEOUT = -6      /* a bounded device wait gave up (device-recorded) */
} fsq_status;

/* eq. (2) of [S]: u~ = h*tanh(u + atanh(delta/h)) - delta, level = round(u~).
 * levels: L in {4, 16, 256}; 0 selects 16.  Requires 0 < delta < h,
 * h - delta <= L/2 - 1/2 and h + delta <= L/2 + 1/2 so that every level lies
 * in {-L/2 .. L/2-1}.  The acceptance default at L = 16 is {7.5, 0.5}; the
 * deck prints h=7.5075 for L=16 ([D] product-code frame); for the other level
 * counts h = (L-1)/2, delta = 0.5 is the same choice. */
typedef struct {
  float h;
  float delta;
  int levels;
} fsq_quant_params;

enum {
  FSQ_VARIANT_AUTO = 0,     /* library picks: ABSORBED when rope_knorm == 0, else
                               HYBRID (EXPAND for shapes HYBRID does not cover) */
  FSQ_VARIANT_ABSORBED = 1, /* score with W_k^T q, pool codes, apply W_v once */
  FSQ_VARIANT_EXPAND = 2,   /* rebuild K and V per tile through W_kv, then GQA */
  FSQ_VARIANT_HYBRID = 3    /* rebuild K per tile through W_k (then N_k and RoPE_t
                               when rope_knorm), pool codes with the weights and
                               apply W_v once ([D] kernel frame, steps 1-4);
                               tensor cores; G in {84, 256}, n_q / n_kv <= 8,
                               16 levels */
};

typedef struct {
  int variant;            /* FSQ_VARIANT_* */
  float scale;            /* softmax scale; <= 0 selects 1/sqrt(d_h) */
  int num_splits;         /* token-range splits per batch row; 0 = automatic */
  int rope_knorm;         /* 1: k_t = RoPE_t(N_k(W_k z_t)) ([S] eq. 5); EXPAND or HYBRID */
  float rope_base;        /* RoPE base (rope_knorm == 1) */
  const uint16_t *knorm_gain; /* device bf16 [d_h] RMS-norm gain, NULL = ones */
  float knorm_eps;        /* RMS-norm epsilon */
  int out_fp32;           /* 0: o is bf16; 1: o is fp32 */
  void *prof_events[2];   /* optional cudaEvent_t pair: recorded on `stream`
                             right before and right after the main attention
                             kernel (for timing it alone); NULL = none */
  const int32_t *seq_lens; /* optional device int32 [B]: batch row b attends to
                             its first seq_lens[b] cached tokens (a ragged
                             batch; 1 <= seq_lens[b] <= T, where T is the call's
                             argument, the longest row).  NULL = T for every
                             row.  A value outside [1, T] is clamped into it and
                             records FSQ_ERR_INVALID_ARG in the workspace's error
                             word.  Read by the kernels like q and codes. */
  uint32_t debug_stall_ns; /* test-only, 0 in normal use.  When > 0, the tensor-
                             core attention kernel first waits, with this limit
                             in nanoseconds, for a barrier that nothing
                             completes, so that its bounded-wait failure path
                             runs: the call records FSQ_ERR_TIMEOUT and its
                             output is undefined.  Only that wait uses the
                             limit; the waits that let in-flight copies and
                             tensor-core operations finish keep their own. */
  int levels;             /* L of the cache's codes: 4, 16 or 256; 0 = 16.  The
                             tensor-core kernels read 16-level codes; at L = 4
                             and L = 256 the library runs its CUDA-core forms
                             (ABSORBED, EXPAND) and AUTO picks among those. */
} fsq_attn_opts;

/* Fills *opts with {AUTO, 1/sqrt(d_h), auto splits, rope off, 1e6, NULL,
 * 1e-6, bf16 output, no profiling events, no per-row lengths, no stall,
 * 16 levels}. */
FSQ_API void fsq_attn_opts_default(fsq_attn_opts *opts);

/* Host-side: the L-1 ascending u-space decision thresholds the kernels
 * compare against (L = qp.levels; theta_out has room for L-1 floats).  A
 * level is -L/2 + #{k : u >= theta_k}.  theta_k is the smallest fp32 value not
 * below the exact preimage of the half-integer boundary m + 1/2
 * (m = -L/2 .. L/2-2) under eq. (2), so for any fp32 u the count equals the
 * exact rounding of eq. (2) except at an exact tie.  Unreachable boundaries
 * are +/-infinity.  Returns FSQ_ERR_INVALID_ARG for bad h or delta and
 * FSQ_ERR_UNSUPPORTED for a level count other than 4, 16 or 256 (the append
 * calls return the same for such parameters). */
FSQ_API fsq_status fsq_thresholds(fsq_quant_params qp, float *theta_out);

/* Options of the append path. */
typedef struct {
  uint32_t *status_word;   /* optional device pointer to a caller-owned 32-bit
                             word.  When the tensor-core append kernel (used for
                             more than 64 tokens) gives up a bounded wait, it
                             records FSQ_ERR_TIMEOUT there and the codes of that
                             call are incomplete.  The library only ever sets
                             the word (the first error stays) and never clears
                             it: zero it before use, read it with
                             fsq_workspace_status(word, 4, stream).  NULL: such
                             a failure is reported nowhere. */
  uint32_t debug_stall_ns; /* test-only, 0 in normal use.  When > 0, the
                             tensor-core append kernel's epilogue first waits,
                             with this limit in nanoseconds, for a barrier that
                             nothing completes, so that its bounded-wait failure
                             path runs (FSQ_ERR_TIMEOUT in status_word). */
  int64_t tokens_per_row;  /* 0: token t's codes go to codes + t*ldc_bytes.  When
                             > 0, the n_tok tokens are groups of tokens_per_row
                             consecutive tokens (the last group may be shorter),
                             one group per cache row: token t goes to codes +
                             (t / tokens_per_row)*row_stride_bytes + (t %
                             tokens_per_row)*ldc_bytes, so one call appends the
                             new tokens of several rows of a [B, T_max, R] cache
                             (codes = &cache[0][T0], row_stride_bytes = T_max*R,
                             ldc_bytes = R).  Destinations must not overlap. */
  int64_t row_stride_bytes; /* bytes between groups (>= 0) when tokens_per_row > 0 */
} fsq_encode_opts;

/* Append path ([S] eq. 4 then packing; [D] product-code frame):
 *   u = E x_t (bf16 operands, fp32 accumulation), level = eq. (2), packed.
 *  x      bf16 [n_tok, ldx], row t = x_t (C used entries)      — read
 *  E      bf16 [G, C] encoder                                    — read
 *  codes  uint8 [n_tok, ldc_bytes]; row t gets R = G*b/8 bytes    — written
 *  opts   may be NULL (no status word, no stall, one stride ldc_bytes)
 * To append at position T of a [T_max, R] cache pass codes + T*R and
 * ldc_bytes = R.  Needs: G even, 2 <= G <= FSQ_MAX_G, G % 4 == 0 at L = 4;
 * C a positive multiple of 64; ldx >= C and ldx % 8 == 0; x and E 16-byte
 * aligned.  n_tok == 0 is a no-op.  Codes are bit-exact with eq. (2) applied
 * to the fp32 u; the fp32 u itself differs from exact arithmetic by the
 * GEMM's rounding. */
FSQ_API fsq_status fsq_encode_pack(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C,
                           const uint16_t *E, int G, fsq_quant_params qp,
                           uint8_t *codes, int64_t ldc_bytes, const fsq_encode_opts *opts,
                           fsq_stream_t stream);

/* Quantiser + packing alone on given fp32 pre-activations u [n_tok, G]
 * (row-major, contiguous; u 16-byte aligned).  Same codes as fsq_encode_pack
 * would write for that u, under the same G rules.  Used to test eq. (2) in
 * isolation. */
FSQ_API fsq_status fsq_quantize_pack_f32(const float *u, int64_t n_tok, int G, fsq_quant_params qp,
                                 uint8_t *codes, int64_t ldc_bytes, fsq_stream_t stream);

/* Bytes of device workspace fsq_decode_attn needs for this shape and
 * options (0 if the arguments are invalid).  Depends only on its
 * arguments. */
FSQ_API size_t fsq_decode_attn_workspace_size(int64_t B, int64_t T, int n_q, int n_kv, int d_h, int G,
                                      const fsq_attn_opts *opts);

/* Single-token GQA decode attention over the packed code cache.
 * For batch row b and query head h, with kv head j = h / (n_q / n_kv):
 *   k_t = W_k^(j) z_t (RoPE_t(N_k(.)) when opts->rope_knorm), v_t = W_v^(j) z_t
 *   o_h = sum_t softmax_t(scale * q_h . k_t) v_t                 ([S] eq. 5)
 * over cached tokens t = 0..T-1, or t = 0..seq_lens[b]-1 for a ragged batch
 * (the caller appends the current token first; cached token t sits at
 * position t).  ABSORBED evaluates the same sum as
 * (W_k^T q_h) . z_t and W_v (sum_t a_t z_t) ([S] eq. 6).
 *  q        bf16 [B, n_q, d_h], already projected/normed/rotated by the caller
 *  codes    uint8 cache, rows as in the format above
 *  W_kv     bf16 [2*n_kv*d_h, G]; rows [W_k; W_v] ([S] eq. 8), head j of W_k
 *           is rows j*d_h..j*d_h+d_h-1, head j of W_v rows (n_kv+j)*d_h..
 *  o        [B, n_q, d_h], bf16 or fp32 (opts->out_fp32)          — written
 *  workspace  >= fsq_decode_attn_workspace_size(...) bytes, 256-byte aligned,
 *             owned by the caller; contents need no initialisation
 * Needs: d_h == 128, n_q % n_kv == 0, G even, 2 <= G <= FSQ_MAX_G (G % 4 == 0
 * at L = 4), T >= 1; codes and code_batch_stride_bytes 16-byte aligned,
 * code_batch_stride_bytes >= T*R (R = G*b/8 bytes per row); q, W_kv, o 16-byte
 * aligned; B <= 65535.  Shapes whose CUDA-core kernels would not fit in shared memory
 * (large n_q * G, or G above 372 for EXPAND) return FSQ_ERR_UNSUPPORTED.
 * B == 0 is a no-op.  opts may be NULL
 * (defaults).  The absorbed form on the tensor cores reads each code tile once
 * with an L2 evict-first hint, so the call's code stream does not displace
 * other data from L2 (the weights, the workspace, the caller's tensors). */
FSQ_API fsq_status fsq_decode_attn(const uint16_t *q, int64_t B, int n_q, int d_h,
                           const uint8_t *codes, int64_t code_batch_stride_bytes, int64_t T, int G,
                           const uint16_t *W_kv, int n_kv, const fsq_attn_opts *opts,
                           void *workspace, size_t workspace_bytes, void *o, fsq_stream_t stream);

/* Multi-query attention over the code cache: n_new query positions per batch
 * row, each attending causally to the cache (chunked prefill, where a chunk's
 * tokens attend to the cache they were just appended to, or speculative
 * decoding, where draft tokens are verified together).  [S] Methodology
 * eq. (4)-(5) applied to several queries; the deck's backup frame "capacity and
 * accuracy are counted by different protocols" counts prefill peak memory,
 * which a code-only cache keeps small.
 *   q   bf16 [B, n_new, n_q, d_h]: query i of row b, projected/normed/rotated
 *   o   [B, n_new, n_q, d_h], bf16 or fp32 (opts->out_fp32)      — written
 * Row b holds L_b cached tokens (T, or opts->seq_lens[b]) whose last n_new are
 * the new tokens, already appended; query i sits at position L_b - n_new + i
 * and attends to tokens 0 .. L_b - n_new + i.  A row shorter than n_new is
 * clamped (its early queries see one token) and records FSQ_ERR_INVALID_ARG in
 * the workspace's error word.  Same forms, options, alignment rules and errors
 * as fsq_decode_attn, which is the case n_new == 1.  Needs n_new >= 1 and
 * B * n_new <= 65535.  The queries of a row run as consecutive rows of the same
 * kernels and share each code tile through L2 (read at normal L2 priority).
 * Workspace: fsq_decode_attn_multi_workspace_size(...). */
FSQ_API size_t fsq_decode_attn_multi_workspace_size(int64_t B, int n_new, int64_t T, int n_q, int n_kv, int d_h,
                                                    int G, const fsq_attn_opts *opts);
FSQ_API fsq_status fsq_decode_attn_multi(const uint16_t *q, int64_t B, int n_new, int n_q, int d_h,
                                         const uint8_t *codes, int64_t code_batch_stride_bytes, int64_t T, int G,
                                         const uint16_t *W_kv, int n_kv, const fsq_attn_opts *opts,
                                         void *workspace, size_t workspace_bytes, void *o, fsq_stream_t stream);

/* Host-side: the name of the attention (split) kernel that
 * fsq_decode_attn_multi would launch for these arguments — one of
 * "absorbed_split_tc" (tensor cores, 16-level rows of 84, 160 or 256 nibbles;
 * 256-level codes read as nibble pairs), "absorbed_split_gen" (tensor cores,
 * codes unpacked to fp16 levels in shared memory), "hybrid_split_tc",
 * "expand_split_tc", "absorbed_split_simt", "expand_split_simt" — or NULL when
 * the arguments are invalid or unsupported.  For logs and benchmarks; the
 * returned string is static. */
FSQ_API const char *fsq_decode_attn_kernel(int64_t B, int n_new, int64_t T, int n_q, int n_kv, int d_h, int G,
                                           const fsq_attn_opts *opts);

/* Allocation-free decode attention.  There is no counterpart in the paper:
 * this entry point exists for callers that cannot allocate device memory at
 * the point where they decode — for example a plugin whose host framework
 * owns every device allocation, or a latency-bound decode loop in which a
 * cudaMalloc (which may synchronise the device) is not acceptable.
 * Same arguments, semantics and result as fsq_decode_attn, minus the
 * workspace: the scratch comes from a file-scope device array of
 * FSQ_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.  Nothing is allocated: no
 * cudaMalloc, cudaFree or allocating library routine is called.
 *  - The first call in a device's CUDA context looks up that array's device
 *    address there (cudaGetSymbolAddress, with the device current) and keeps
 *    it for that context; a reset device gets a new context and a new lookup.
 *    Make the first call before any stream capture.
 *  - Requests whose fsq_decode_attn_workspace_size exceeds
 *    FSQ_NOALLOC_SCRATCH_BYTES return FSQ_ERR_WORKSPACE before any launch
 *    (use fsq_decode_attn with a workspace of your own for those).
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents (every value a call relies on is rewritten by that call).
 *    Calls that can overlap on the GPU (different streams without ordering)
 *    race on it and must be serialised by the caller. */
#define FSQ_NOALLOC_SCRATCH_BYTES (16u << 20)
FSQ_API fsq_status fsq_decode_attn_noalloc(const uint16_t *q, int64_t B, int n_q, int d_h,
                                           const uint8_t *codes, int64_t code_batch_stride_bytes, int64_t T,
                                           int G, const uint16_t *W_kv, int n_kv, const fsq_attn_opts *opts,
                                           void *o, fsq_stream_t stream);

/* The device status of the last fsq_decode_attn_noalloc call on the current
 * device: the error word of the built-in scratch, which each call clears
 * first (the same word fsq_workspace_status reads in a caller's workspace).
 * Returns FSQ_OK or the recorded status, e.g. FSQ_ERR_TIMEOUT when a
 * bounded device wait of that call gave up and its output is undefined.
 * Blocking: synchronises with `stream`.  A device with no call yet reads
 * FSQ_OK. */
FSQ_API fsq_status fsq_decode_attn_noalloc_status(fsq_stream_t stream);

/* Reads a device status word: the error word at the start of a workspace
 * last used by fsq_decode_attn (each decode call clears it first), or an
 * append path's fsq_encode_opts.status_word (workspace_bytes >= 4).  Blocking
 * copy: synchronises with `stream`.  Returns FSQ_OK or the recorded device
 * status (e.g. FSQ_ERR_TIMEOUT); clears nothing. */
FSQ_API fsq_status fsq_workspace_status(const void *workspace, size_t workspace_bytes, fsq_stream_t stream);

FSQ_API const char *fsq_status_string(fsq_status s);
FSQ_API int fsq_format_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FSQ_H_ */
