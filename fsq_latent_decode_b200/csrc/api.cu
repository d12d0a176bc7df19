// C ABI of the library: argument validation, launch planning, dispatch.
// Every check that can fail runs before any CUDA call, so invalid requests
// return synchronously without touching the device.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"

namespace fsq {
cudaError_t launch_encode_pack(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C, const uint16_t *E, int G,
                               int levels, const float *th, uint8_t *codes, int64_t ldc, int64_t per_row,
                               int64_t row_stride, uint32_t *status, uint32_t stall_ns, cudaStream_t s);
cudaError_t launch_quantize_pack_f32(const float *u, int64_t n_tok, int G, int levels, const float *th,
                                     uint8_t *codes, int64_t ldc, cudaStream_t s);
cudaError_t launch_absorbed_simt(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int n_new,
                                 int64_t T, const int32_t *seq_lens, int n_q, int n_kv, int d_h, int G, int bits,
                                 const uint16_t *W_kv, float scale, int S, int64_t tps, float *qa, float *part,
                                 uint32_t *err, MergeScratch ms, void *o, int out_fp32, void *const *prof,
                                 cudaStream_t st);
cudaError_t launch_expand_simt(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int n_new,
                               int64_t T, const int32_t *seq_lens, int n_q, int n_kv, int d_h, int G, int bits,
                               const uint16_t *W_kv, float scale, int S, int64_t tps, int rope_knorm,
                               float rope_base, const uint16_t *gain, float eps, float *part, uint32_t *err, void *o,
                               int out_fp32, void *const *prof, cudaStream_t st);
size_t absorbed_simt_smem(int n_q, int G);
size_t expand_simt_smem(int G);
bool expand_tc_supported(int n_q, int n_kv, int G);
size_t expand_tc_stage_bytes(int G, int variant_expand);
cudaError_t launch_expand_tc(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int n_new,
                             int64_t T, const int32_t *seq_lens, int n_q, int n_kv, int d_h, int G, const uint16_t *W_kv,
                             float scale, int S, int64_t tps, int hybrid, int rope, float rope_base,
                             const uint16_t *gain, float eps, uint8_t *wk, uint8_t *wv, float *ck, float *cv,
                             uint8_t *qs, float *part, uint32_t *err, MergeScratch ms, void *o, int out_fp32,
                             uint32_t stall_ns, void *const *prof, cudaStream_t st);
int simt_max_nq();
int simt_max_grp();
int absorbed_tc_width(int n_q, int n_kv, int G, int levels);
bool absorbed_gen_supported(int n_q, int n_kv, int G, int levels);
size_t absorbed_gen_qbuf_bytes(int n_q, int G);
int absorbed_gen_ctas_per_sm(int n_q, int G, int levels);
cudaError_t launch_absorbed_gen(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t R, int n_new,
                                int64_t T, const int32_t *seq_lens, int n_q, int n_kv, int d_h, int G, int levels,
                                const uint16_t *W_kv, float scale, int S, int64_t tps, uint8_t *qbuf, float *part,
                                uint32_t *err, MergeScratch ms, void *o, int out_fp32, uint32_t stall_ns,
                                void *const *prof, cudaStream_t st);
size_t absorbed_tc_qphys_bytes(int n_q, int G);
cudaError_t launch_absorbed_tc(const uint16_t *q, const uint8_t *codes, int64_t bstride, int64_t B, int n_new,
                               int64_t T, const int32_t *seq_lens, int n_q, int n_kv, int d_h, int G, int levels,
                               const uint16_t *W_kv, float scale, int S, int64_t tps, uint8_t *qphys, float *corr,
                               float *part, uint32_t *err, MergeScratch ms, void *o, int out_fp32,
                               uint32_t stall_ns, void *const *prof, cudaStream_t st);

namespace {

constexpr int kMaxSplits = 1024;
constexpr int64_t kMaxGridRows = 65535;  // grid rows of a call: batch rows x queries per row (grid y)
constexpr bool kEnableTc = true;  // tensor-core absorbed kernel (being validated)

constexpr size_t kMaxDynSmem = 227 * 1024;  // dynamic shared memory a CTA may request

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Level count of a levels field (0 selects 16); 0 when unsupported.
int levels_of(int levels) {
  if (levels == 0) return FSQ_LEVELS;
  return bits_of_levels(levels) ? levels : 0;
}

// Latent widths that pack into whole bytes and whole coordinate pairs.
bool width_ok(int G, int L) { return G >= 2 && G <= FSQ_MAX_G && G % 2 == 0 && (L != 4 || G % 4 == 0); }

// Every level of eq. (2) must lie in {-L/2 .. L/2-1}.
fsq_status check_quant(fsq_quant_params qp) {
  const int L = levels_of(qp.levels);
  if (!L) return FSQ_ERR_UNSUPPORTED;
  const float top = 0.5f * (float)L;
  if (!(qp.delta > 0.f) || !(qp.h > qp.delta)) return FSQ_ERR_INVALID_ARG;
  if (!(qp.h - qp.delta <= top - 0.5f) || !(qp.h + qp.delta <= top + 0.5f)) return FSQ_ERR_INVALID_ARG;
  return FSQ_OK;
}

// Smallest float not below x (x finite).
float ceil_to_float(double x) {
  float f = (float)x;
  if ((double)f < x) f = nextafterf(f, INFINITY);
  return f;
}

// The L-1 thresholds of eq. (2) at L = levels_of(qp.levels).
void make_thresholds(fsq_quant_params qp, float *out) {
  const int L = levels_of(qp.levels);
  const double h = qp.h, dl = qp.delta;
  const double a = atanh(dl / h);
  for (int k = 0; k < L - 1; ++k) {
    const double m = (double)(k - L / 2);     // boundary between levels m and m+1
    const double arg = (m + 0.5 + dl) / h;    // tanh(u + a) at u~ = m + 1/2
    if (arg >= 1.0) out[k] = INFINITY;
    else if (arg <= -1.0) out[k] = -INFINITY;
    else out[k] = ceil_to_float(atanh(arg) - a);
  }
}

struct Plan {
  int variant;
  int levels;     // L of the codes
  bool gen;       // generic tensor-core absorbed kernel
  bool tc;        // tensor-core kernel (absorbed, expand or hybrid form)
  int S;          // splits per batch row
  int64_t tps;    // tokens per split
  MergePlan mp;   // split merge of the absorbed and hybrid forms
  size_t off_qa, off_corr, off_part, off_mslab, off_mcnt, total;
  size_t off_wk, off_wv, off_ck, off_cv;  // staged decoder slices of the tensor-core expand / hybrid forms
};

fsq_status plan_decode(int64_t B, int64_t T, int n_q, int n_kv, int d_h, int G, const fsq_attn_opts &op, Plan *p) {
  if (B < 0 || T < 1 || n_q < 1 || n_kv < 1 || d_h < 1 || G < 2) return FSQ_ERR_INVALID_ARG;
  if (n_q % n_kv) return FSQ_ERR_INVALID_ARG;
  const int L = levels_of(op.levels);
  if (!L || !width_ok(G, L) || d_h != FSQ_HEAD_DIM) return FSQ_ERR_UNSUPPORTED;
  if (op.variant < FSQ_VARIANT_AUTO || op.variant > FSQ_VARIANT_HYBRID) return FSQ_ERR_INVALID_ARG;
  if (op.num_splits < 0) return FSQ_ERR_INVALID_ARG;
  if (op.rope_knorm != 0 && op.rope_knorm != 1) return FSQ_ERR_INVALID_ARG;
  int variant = op.variant;
  // the tensor-core kernels read 16-level codes
  const bool xtc_shape = kEnableTc && L == 16 && expand_tc_supported(n_q, n_kv, G);
  if (variant == FSQ_VARIANT_AUTO)
    variant = !op.rope_knorm ? FSQ_VARIANT_ABSORBED : (xtc_shape ? FSQ_VARIANT_HYBRID : FSQ_VARIANT_EXPAND);
  if (variant == FSQ_VARIANT_ABSORBED && op.rope_knorm) return FSQ_ERR_UNSUPPORTED;
  if (variant == FSQ_VARIANT_ABSORBED && n_q > simt_max_nq()) return FSQ_ERR_UNSUPPORTED;
  if (variant == FSQ_VARIANT_HYBRID && !xtc_shape) return FSQ_ERR_UNSUPPORTED;
  if (variant == FSQ_VARIANT_EXPAND && !xtc_shape && n_q / n_kv > simt_max_grp()) return FSQ_ERR_UNSUPPORTED;
  if (op.rope_knorm && !(op.rope_base > 1.f && op.knorm_eps >= 0.f)) return FSQ_ERR_INVALID_ARG;

  const int64_t Bc = B > 0 ? B : 1;
  const bool xtc = (variant == FSQ_VARIANT_EXPAND || variant == FSQ_VARIANT_HYBRID) && xtc_shape;
  // the absorbed tensor-core kernel reads rows of Gn nibbles: 16-level codes,
  // or 256-level codes read as two nibbles each (Gn = 2G)
  const int Gn = (kEnableTc && variant == FSQ_VARIANT_ABSORBED) ? absorbed_tc_width(n_q, n_kv, G, L) : 0;
  // other absorbed shapes: the generic tensor-core kernel (codes unpacked to fp16 in shared memory)
  const bool gen = !Gn && kEnableTc && variant == FSQ_VARIANT_ABSORBED && absorbed_gen_supported(n_q, n_kv, G, L);
  const bool tc = Gn > 0 || xtc || gen;
  // the CUDA-core kernels hold a tile of latents (and, in the expand form, W_kv^(j)) in shared memory
  if (!tc && variant == FSQ_VARIANT_ABSORBED && absorbed_simt_smem(n_q, G) > kMaxDynSmem) return FSQ_ERR_UNSUPPORTED;
  if (!tc && variant == FSQ_VARIANT_EXPAND && expand_simt_smem(G) > kMaxDynSmem) return FSQ_ERR_UNSUPPORTED;
  const int64_t ctas_per_row = (variant == FSQ_VARIANT_EXPAND || variant == FSQ_VARIANT_HYBRID) ? n_kv : 1;
  int64_t S = op.num_splits;
  if (S == 0) {
    if (tc) {
      // one wave of CTAs: one per SM (each holds all of TMEM), or as many as
      // an SM holds of the generic kernel
      const int per_sm = gen ? absorbed_gen_ctas_per_sm(n_q, G, L) : 1;
      S = (int64_t)kNumSMs * per_sm / (Bc * ctas_per_row);
      if (S < 1) S = 1;
    } else {
      const int64_t target = 2 * kNumSMs;
      S = (target + Bc * ctas_per_row - 1) / (Bc * ctas_per_row);
      const int64_t max_by_len = (T + 255) / 256;
      if (S > max_by_len) S = max_by_len;
    }
  }
  if (S < 1) S = 1;
  if (S > kMaxSplits) S = kMaxSplits;
  if (S > T) S = T;
  int64_t tps = (T + S - 1) / S;
  if (tc) tps = (tps + 127) / 128 * 128;  // whole 128-token tiles, 16-byte aligned split starts
  S = (T + tps - 1) / tps;  // no empty splits
  p->variant = variant;
  p->levels = L;
  p->tc = tc;
  p->gen = gen;
  p->S = (int)S;
  p->tps = tps;
  const int acc_len = variant == FSQ_VARIANT_EXPAND ? d_h : (Gn ? Gn : G);  // floats per partial after (m, l)
  size_t off = kWsHeader;
  p->off_qa = off;
  if (xtc) off = align_up(off + (size_t)Bc * n_kv * 16 * d_h * 2, 256);  // staged queries
  else if (gen) off = align_up(off + absorbed_gen_qbuf_bytes(n_q, G) * (size_t)Bc, 256);
  else if (tc) off = align_up(off + absorbed_tc_qphys_bytes(n_q, Gn) * (size_t)Bc, 256);
  else if (variant == FSQ_VARIANT_ABSORBED) off = align_up(off + sizeof(float) * (size_t)Bc * n_q * G, 256);
  p->off_corr = off;
  if (tc && !xtc && !gen) off = align_up(off + 2 * sizeof(float) * (size_t)Bc * n_q, 256);  // per-head scales / offsets
  p->off_wk = p->off_wv = p->off_ck = p->off_cv = off;
  if (xtc) {
    const size_t slice = expand_tc_stage_bytes(G, 0);
    p->off_wk = off;
    off = align_up(off + slice * n_kv, 256);
    p->off_wv = off;
    if (variant == FSQ_VARIANT_EXPAND) off = align_up(off + slice * n_kv, 256);
    p->off_ck = off;
    off = align_up(off + sizeof(float) * d_h * n_kv, 256);
    p->off_cv = off;
    off = align_up(off + sizeof(float) * d_h * n_kv, 256);
  }
  p->off_part = off;
  off = align_up(off + sizeof(float) * (size_t)Bc * S * n_q * (2 + acc_len), 256);
  if (variant == FSQ_VARIANT_ABSORBED || variant == FSQ_VARIANT_HYBRID) p->mp = merge_plan((int)S, Bc, n_q, n_kv, acc_len);
  p->off_mslab = off;
  off = align_up(off + p->mp.slab_bytes, 256);
  p->off_mcnt = off;
  off = align_up(off + p->mp.cnt_bytes, 256);
  p->total = off;
  return FSQ_OK;
}

fsq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FSQ_OK : FSQ_ERR_CUDA; }

}  // namespace
}  // namespace fsq

using namespace fsq;

extern "C" {

void fsq_attn_opts_default(fsq_attn_opts *opts) {
  if (!opts) return;
  memset(opts, 0, sizeof(*opts));
  opts->variant = FSQ_VARIANT_AUTO;
  opts->scale = 0.f;
  opts->num_splits = 0;
  opts->rope_knorm = 0;
  opts->rope_base = 1.0e6f;
  opts->knorm_gain = nullptr;
  opts->knorm_eps = 1.0e-6f;
  opts->out_fp32 = 0;
  opts->prof_events[0] = opts->prof_events[1] = nullptr;
  opts->seq_lens = nullptr;
  opts->debug_stall_ns = 0;
  opts->levels = FSQ_LEVELS;
}

fsq_status fsq_thresholds(fsq_quant_params qp, float *theta_out) {
  if (!theta_out) return FSQ_ERR_INVALID_ARG;
  fsq_status st = check_quant(qp);
  if (st != FSQ_OK) return st;
  make_thresholds(qp, theta_out);
  return FSQ_OK;
}

fsq_status fsq_encode_pack(const uint16_t *x, int64_t n_tok, int64_t ldx, int64_t C, const uint16_t *E, int G,
                           fsq_quant_params qp, uint8_t *codes, int64_t ldc_bytes, const fsq_encode_opts *opts,
                           fsq_stream_t stream) {
  if (n_tok < 0 || C < 1 || G < 2) return FSQ_ERR_INVALID_ARG;
  fsq_status st = check_quant(qp);
  if (st != FSQ_OK) return st;
  const int L = levels_of(qp.levels);
  if (!width_ok(G, L) || C % 64) return FSQ_ERR_UNSUPPORTED;
  if (ldx < C || ldc_bytes < (int64_t)G * bits_of_levels(L) / 8) return FSQ_ERR_INVALID_ARG;
  if (n_tok == 0) return FSQ_OK;
  if (!x || !E || !codes) return FSQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(E) || ldx % 8) return FSQ_ERR_MISALIGNED;
  uint32_t *status = opts ? opts->status_word : nullptr;
  if ((uintptr_t)status & 3u) return FSQ_ERR_MISALIGNED;
  const int64_t per_row = opts ? opts->tokens_per_row : 0;
  const int64_t row_stride = opts ? opts->row_stride_bytes : 0;
  if (per_row < 0 || (per_row > 0 && row_stride < 0)) return FSQ_ERR_INVALID_ARG;
  float th[kMaxLevels - 1];
  make_thresholds(qp, th);
  return from_cuda(launch_encode_pack(x, n_tok, ldx, C, E, G, L, th, codes, ldc_bytes, per_row, row_stride, status,
                                      opts ? opts->debug_stall_ns : 0u, (cudaStream_t)stream));
}

fsq_status fsq_quantize_pack_f32(const float *u, int64_t n_tok, int G, fsq_quant_params qp, uint8_t *codes,
                                 int64_t ldc_bytes, fsq_stream_t stream) {
  if (n_tok < 0 || G < 2) return FSQ_ERR_INVALID_ARG;
  fsq_status st = check_quant(qp);
  if (st != FSQ_OK) return st;
  const int L = levels_of(qp.levels);
  if (!width_ok(G, L)) return FSQ_ERR_UNSUPPORTED;
  if (ldc_bytes < (int64_t)G * bits_of_levels(L) / 8) return FSQ_ERR_INVALID_ARG;
  if (n_tok == 0) return FSQ_OK;
  if (!u || !codes) return FSQ_ERR_INVALID_ARG;
  if (!aligned16(u)) return FSQ_ERR_MISALIGNED;
  float th[kMaxLevels - 1];
  make_thresholds(qp, th);
  return from_cuda(launch_quantize_pack_f32(u, n_tok, G, L, th, codes, ldc_bytes, (cudaStream_t)stream));
}

size_t fsq_decode_attn_workspace_size(int64_t B, int64_t T, int n_q, int n_kv, int d_h, int G,
                                      const fsq_attn_opts *opts) {
  return fsq_decode_attn_multi_workspace_size(B, 1, T, n_q, n_kv, d_h, G, opts);
}

size_t fsq_decode_attn_multi_workspace_size(int64_t B, int n_new, int64_t T, int n_q, int n_kv, int d_h, int G,
                                            const fsq_attn_opts *opts) {
  fsq_attn_opts op;
  if (opts) op = *opts;
  else fsq_attn_opts_default(&op);
  Plan p;
  if (n_new < 1 || B < 0 || B * n_new > kMaxGridRows) return 0;
  if (plan_decode(B * n_new, T, n_q, n_kv, d_h, G, op, &p) != FSQ_OK) return 0;
  return p.total;
}

const char *fsq_decode_attn_kernel(int64_t B, int n_new, int64_t T, int n_q, int n_kv, int d_h, int G,
                                   const fsq_attn_opts *opts) {
  fsq_attn_opts op;
  if (opts) op = *opts;
  else fsq_attn_opts_default(&op);
  Plan p;
  if (n_new < 1 || B < 0 || B * n_new > kMaxGridRows) return nullptr;
  if (plan_decode(B * n_new, T, n_q, n_kv, d_h, G, op, &p) != FSQ_OK) return nullptr;
  if (p.variant == FSQ_VARIANT_HYBRID) return "hybrid_split_tc";
  if (p.variant == FSQ_VARIANT_EXPAND) return p.tc ? "expand_split_tc" : "expand_split_simt";
  if (p.gen) return "absorbed_split_gen";
  return p.tc ? "absorbed_split_tc" : "absorbed_split_simt";
}

fsq_status fsq_decode_attn(const uint16_t *q, int64_t B, int n_q, int d_h, const uint8_t *codes,
                           int64_t code_batch_stride_bytes, int64_t T, int G, const uint16_t *W_kv, int n_kv,
                           const fsq_attn_opts *opts, void *workspace, size_t workspace_bytes, void *o,
                           fsq_stream_t stream) {
  return fsq_decode_attn_multi(q, B, 1, n_q, d_h, codes, code_batch_stride_bytes, T, G, W_kv, n_kv, opts, workspace,
                               workspace_bytes, o, stream);
}

// The queries of a cache row run as n_new consecutive grid rows of the same
// kernels (R = B * n_new rows); only the split kernels map a grid row to its
// cache row and causal length.
fsq_status fsq_decode_attn_multi(const uint16_t *q, int64_t B, int n_new, int n_q, int d_h, const uint8_t *codes,
                                 int64_t code_batch_stride_bytes, int64_t T, int G, const uint16_t *W_kv, int n_kv,
                                 const fsq_attn_opts *opts, void *workspace, size_t workspace_bytes, void *o,
                                 fsq_stream_t stream) {
  fsq_attn_opts op;
  if (opts) op = *opts;
  else fsq_attn_opts_default(&op);
  if (n_new < 1 || B < 0) return FSQ_ERR_INVALID_ARG;
  if (B * n_new > kMaxGridRows) return FSQ_ERR_UNSUPPORTED;
  const int64_t R = B * n_new;
  Plan p;
  fsq_status st = plan_decode(R, T, n_q, n_kv, d_h, G, op, &p);
  if (st != FSQ_OK) return st;
  if (B == 0) return FSQ_OK;
  if (!q || !codes || !W_kv || !o) return FSQ_ERR_INVALID_ARG;
  const int bits = bits_of_levels(p.levels);
  if (code_batch_stride_bytes < T * ((int64_t)G * bits / 8)) return FSQ_ERR_INVALID_ARG;
  if (!aligned16(codes) || code_batch_stride_bytes % 16) return FSQ_ERR_MISALIGNED;
  if (!aligned16(q) || !aligned16(W_kv) || !aligned16(o)) return FSQ_ERR_MISALIGNED;
  if ((uintptr_t)op.seq_lens & 3u) return FSQ_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < p.total) return FSQ_ERR_WORKSPACE;
  if ((uintptr_t)workspace & 255u) return FSQ_ERR_MISALIGNED;
  const float scale = op.scale > 0.f ? op.scale : 1.f / sqrtf((float)d_h);
  char *ws = (char *)workspace;
  uint32_t *err = (uint32_t *)ws;
  float *part = (float *)(ws + p.off_part);
  cudaStream_t s = (cudaStream_t)stream;
  MergeScratch ms{nullptr, nullptr, 0};
  if (p.mp.cnt_bytes) ms = {(float *)(ws + p.off_mslab), (uint32_t *)(ws + p.off_mcnt), (int)(R * n_kv)};
  cudaError_t e;
  if (p.tc && (p.variant == FSQ_VARIANT_EXPAND || p.variant == FSQ_VARIANT_HYBRID)) {
    e = launch_expand_tc(q, codes, code_batch_stride_bytes, R, n_new, T, op.seq_lens, n_q, n_kv, d_h, G, W_kv, scale,
                         p.S, p.tps, p.variant == FSQ_VARIANT_HYBRID, op.rope_knorm, op.rope_base, op.knorm_gain,
                         op.knorm_eps, (uint8_t *)(ws + p.off_wk), (uint8_t *)(ws + p.off_wv),
                         (float *)(ws + p.off_ck), (float *)(ws + p.off_cv), (uint8_t *)(ws + p.off_qa), part, err,
                         ms, o, op.out_fp32, op.debug_stall_ns, op.prof_events, s);
  } else if (p.gen) {
    e = launch_absorbed_gen(q, codes, code_batch_stride_bytes, R, n_new, T, op.seq_lens, n_q, n_kv, d_h, G, p.levels,
                            W_kv, scale, p.S, p.tps, (uint8_t *)(ws + p.off_qa), part, err, ms, o, op.out_fp32,
                            op.debug_stall_ns, op.prof_events, s);
  } else if (p.tc) {
    e = launch_absorbed_tc(q, codes, code_batch_stride_bytes, R, n_new, T, op.seq_lens, n_q, n_kv, d_h, G, p.levels,
                           W_kv, scale, p.S, p.tps, (uint8_t *)(ws + p.off_qa), (float *)(ws + p.off_corr), part, err,
                           ms, o, op.out_fp32, op.debug_stall_ns, op.prof_events, s);
  } else if (p.variant == FSQ_VARIANT_ABSORBED) {
    e = launch_absorbed_simt(q, codes, code_batch_stride_bytes, R, n_new, T, op.seq_lens, n_q, n_kv, d_h, G, bits,
                             W_kv, scale, p.S, p.tps, (float *)(ws + p.off_qa), part, err, ms, o, op.out_fp32,
                             op.prof_events, s);
  } else {
    e = launch_expand_simt(q, codes, code_batch_stride_bytes, R, n_new, T, op.seq_lens, n_q, n_kv, d_h, G, bits,
                           W_kv, scale, p.S, p.tps, op.rope_knorm, op.rope_base, op.knorm_gain, op.knorm_eps, part,
                           err, o, op.out_fp32, op.prof_events, s);
  }
  return from_cuda(e);
}

fsq_status fsq_workspace_status(const void *workspace, size_t workspace_bytes, fsq_stream_t stream) {
  if (!workspace || workspace_bytes < sizeof(uint32_t)) return FSQ_ERR_INVALID_ARG;
  if ((uintptr_t)workspace & 3u) return FSQ_ERR_MISALIGNED;
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return FSQ_ERR_CUDA;
  return v == 0 ? FSQ_OK : (fsq_status)(-(int)v);
}

const char *fsq_status_string(fsq_status s) {
  switch (s) {
    case FSQ_OK: return "ok";
    case FSQ_ERR_INVALID_ARG: return "invalid argument";
    case FSQ_ERR_UNSUPPORTED: return "unsupported shape or option";
    case FSQ_ERR_MISALIGNED: return "pointer or stride not 16-byte aligned";
    case FSQ_ERR_WORKSPACE: return "workspace missing or too small";
    case FSQ_ERR_CUDA: return "CUDA error";
    case FSQ_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

int fsq_format_version(void) { return FSQ_FORMAT_VERSION; }

}  // extern "C"
