"""ctypes binding of libfsq.so (declared in include/fsq.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  The shared library is loaded on first use (the first call, or the
first access to `lib`), so that importing the package for its seeded input
generators maps no native code.  If the library is missing, that first use
fails loudly; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import math
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libfsq.so")

FSQ_OK = 0
FSQ_ERR_INVALID_ARG = -1
FSQ_ERR_UNSUPPORTED = -2
FSQ_ERR_MISALIGNED = -3
FSQ_ERR_WORKSPACE = -4
FSQ_ERR_CUDA = -5
FSQ_ERR_TIMEOUT = -6

VARIANT_AUTO, VARIANT_ABSORBED, VARIANT_EXPAND, VARIANT_HYBRID = 0, 1, 2, 3
VARIANTS = {"auto": VARIANT_AUTO, "absorbed": VARIANT_ABSORBED, "expand": VARIANT_EXPAND, "hybrid": VARIANT_HYBRID}

# Every symbol include/fsq.h declares.
EXPORTED = ("fsq_attn_opts_default", "fsq_thresholds", "fsq_encode_pack", "fsq_quantize_pack_f32",
            "fsq_decode_attn_workspace_size", "fsq_decode_attn", "fsq_workspace_status",
            "fsq_status_string", "fsq_format_version", "fsq_decode_attn_noalloc",
            "fsq_decode_attn_noalloc_status", "fsq_decode_attn_multi_workspace_size", "fsq_decode_attn_multi",
            "fsq_decode_attn_kernel")
# FSQ_NOALLOC_SCRATCH_BYTES of include/fsq.h (a host test checks the two agree)
NOALLOC_SCRATCH_BYTES = 16 << 20


class QuantParams(C.Structure):
    _fields_ = [("h", C.c_float), ("delta", C.c_float), ("levels", C.c_int)]


class AttnOpts(C.Structure):
    _fields_ = [("variant", C.c_int), ("scale", C.c_float), ("num_splits", C.c_int),
                ("rope_knorm", C.c_int), ("rope_base", C.c_float), ("knorm_gain", C.c_void_p),
                ("knorm_eps", C.c_float), ("out_fp32", C.c_int), ("prof_events", C.c_void_p * 2),
                ("seq_lens", C.c_void_p), ("debug_stall_ns", C.c_uint32), ("levels", C.c_int)]


class EncodeOpts(C.Structure):
    _fields_ = [("status_word", C.c_void_p), ("debug_stall_ns", C.c_uint32), ("tokens_per_row", C.c_int64),
                ("row_stride_bytes", C.c_int64)]


class FsqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python fsq_latent_decode_b200/build.py` "
                          "(the CUDA library is required; there is no CPU fallback)")
    lib = C.CDLL(LIB_PATH)
    i64, i32, vp, f32 = C.c_int64, C.c_int, C.c_void_p, C.c_float
    lib.fsq_attn_opts_default.argtypes = [C.POINTER(AttnOpts)]
    lib.fsq_attn_opts_default.restype = None
    lib.fsq_thresholds.argtypes = [QuantParams, C.POINTER(C.c_float)]
    lib.fsq_thresholds.restype = i32
    lib.fsq_encode_pack.argtypes = [vp, i64, i64, i64, vp, i32, QuantParams, vp, i64, C.POINTER(EncodeOpts), vp]
    lib.fsq_encode_pack.restype = i32
    lib.fsq_quantize_pack_f32.argtypes = [vp, i64, i32, QuantParams, vp, i64, vp]
    lib.fsq_quantize_pack_f32.restype = i32
    lib.fsq_decode_attn_workspace_size.argtypes = [i64, i64, i32, i32, i32, i32, C.POINTER(AttnOpts)]
    lib.fsq_decode_attn_workspace_size.restype = C.c_size_t
    lib.fsq_decode_attn.argtypes = [vp, i64, i32, i32, vp, i64, i64, i32, vp, i32, C.POINTER(AttnOpts),
                                    vp, C.c_size_t, vp, vp]
    lib.fsq_decode_attn.restype = i32
    lib.fsq_decode_attn_multi_workspace_size.argtypes = [i64, i32, i64, i32, i32, i32, i32, C.POINTER(AttnOpts)]
    lib.fsq_decode_attn_multi_workspace_size.restype = C.c_size_t
    lib.fsq_decode_attn_multi.argtypes = [vp, i64, i32, i32, i32, vp, i64, i64, i32, vp, i32, C.POINTER(AttnOpts),
                                          vp, C.c_size_t, vp, vp]
    lib.fsq_decode_attn_multi.restype = i32
    lib.fsq_decode_attn_kernel.argtypes = [i64, i32, i64, i32, i32, i32, i32, C.POINTER(AttnOpts)]
    lib.fsq_decode_attn_kernel.restype = C.c_char_p
    lib.fsq_decode_attn_noalloc.argtypes = [vp, i64, i32, i32, vp, i64, i64, i32, vp, i32, C.POINTER(AttnOpts),
                                            vp, vp]
    lib.fsq_decode_attn_noalloc.restype = i32
    lib.fsq_decode_attn_noalloc_status.argtypes = [vp]
    lib.fsq_decode_attn_noalloc_status.restype = i32
    lib.fsq_workspace_status.argtypes = [vp, C.c_size_t, vp]
    lib.fsq_workspace_status.restype = i32
    lib.fsq_status_string.argtypes = [i32]
    lib.fsq_status_string.restype = C.c_char_p
    lib.fsq_format_version.argtypes = []
    lib.fsq_format_version.restype = i32
    return lib


_LIB = None


def _lib() -> C.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):  # `_abi.lib` loads the library on first access
    if name == "lib":
        return _lib()
    raise AttributeError(name)


def status_string(s: int) -> str:
    return _lib().fsq_status_string(int(s)).decode()


def _check(st: int, what: str):
    if st != FSQ_OK:
        raise FsqError(st, what)


def bits_of_levels(levels: int) -> int:
    """b = log2 L bits per coordinate code (L = 4, 16 or 256)."""
    return {4: 2, 16: 4, 256: 8}[int(levels)]


def row_bytes(G: int, levels: int = 16) -> int:
    """Bytes of one token's packed codes: G * b / 8."""
    return G * bits_of_levels(levels) // 8


def quant_params(h: float | None = None, delta: float = 0.5, levels: int = 16) -> QuantParams:
    """eq. (2) parameters; h defaults to (L-1)/2 (7.5 at 16 levels)."""
    if h is None:
        h = (int(levels) - 1) / 2.0
    return QuantParams(float(h), float(delta), int(levels))


def thresholds(h: float | None = None, delta: float = 0.5, levels: int = 16):
    n = max(int(levels), 16) - 1  # room for the table of a supported level count
    buf = (C.c_float * n)()
    _check(_lib().fsq_thresholds(quant_params(h, delta, levels), buf), "fsq_thresholds")
    return [buf[i] for i in range(int(levels) - 1)]


def attn_opts(variant="auto", scale=0.0, num_splits=0, rope_knorm=False, rope_base=1.0e6,
              knorm_gain=None, knorm_eps=1e-6, out_fp32=False, prof_events=None, seq_lens=None,
              debug_stall_ns=0, levels=16) -> AttnOpts:
    o = AttnOpts()
    _lib().fsq_attn_opts_default(C.byref(o))
    o.variant = VARIANTS[variant] if isinstance(variant, str) else int(variant)
    o.scale = float(scale)
    o.num_splits = int(num_splits)
    o.rope_knorm = int(bool(rope_knorm))
    o.rope_base = float(rope_base)
    o.knorm_gain = None if knorm_gain is None else int(knorm_gain.data_ptr())
    o.knorm_eps = float(knorm_eps)
    o.out_fp32 = int(bool(out_fp32))
    if prof_events is not None:  # a pair of objects exposing a raw cudaEvent_t as .cuda_event
        o.prof_events[0] = int(prof_events[0].cuda_event)
        o.prof_events[1] = int(prof_events[1].cuda_event)
    o.seq_lens = None if seq_lens is None else int(seq_lens.data_ptr())  # device int32 [B]
    o.debug_stall_ns = int(debug_stall_ns)
    o.levels = int(levels)
    # the struct holds raw device pointers: keep their tensors alive as long as it
    # lives, or the allocator may hand their memory to the next buffer
    o._tensors = (knorm_gain, seq_lens)
    return o


def encode_opts(status_word=None, debug_stall_ns=0, tokens_per_row=0, row_stride_bytes=0) -> EncodeOpts:
    """status_word: a device tensor whose first 4 bytes are the caller's status
    word; tokens_per_row / row_stride_bytes: groups of consecutive tokens, each
    group written at its own cache row (0: one stride between tokens)."""
    o = EncodeOpts(None if status_word is None else int(status_word.data_ptr()), int(debug_stall_ns),
                   int(tokens_per_row), int(row_stride_bytes))
    o._tensors = (status_word,)  # keeps the word's memory alive with the struct
    return o


def _stream_ptr(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _ptr(t) -> int:
    return int(t.data_ptr())


# ---------------------------------------------------------------- raw C-ABI calls (pointers in, status out)
def encode_pack_raw(x_ptr, n_tok, ldx, C_, E_ptr, G, qp, codes_ptr, ldc, stream_ptr, opts=None) -> int:
    return _lib().fsq_encode_pack(x_ptr, n_tok, ldx, C_, E_ptr, G, qp, codes_ptr, ldc,
                                  None if opts is None else C.byref(opts), stream_ptr)


def quantize_pack_f32_raw(u_ptr, n_tok, G, qp, codes_ptr, ldc, stream_ptr) -> int:
    return _lib().fsq_quantize_pack_f32(u_ptr, n_tok, G, qp, codes_ptr, ldc, stream_ptr)


def workspace_size(B, T, n_q, n_kv, d_h, G, opts: AttnOpts | None = None) -> int:
    return int(_lib().fsq_decode_attn_workspace_size(B, T, n_q, n_kv, d_h, G,
                                                     None if opts is None else C.byref(opts)))


def decode_attn_raw(q_ptr, B, n_q, d_h, codes_ptr, bstride, T, G, wkv_ptr, n_kv, opts, ws_ptr, ws_bytes,
                    o_ptr, stream_ptr) -> int:
    return _lib().fsq_decode_attn(q_ptr, B, n_q, d_h, codes_ptr, bstride, T, G, wkv_ptr, n_kv,
                                  None if opts is None else C.byref(opts), ws_ptr, ws_bytes, o_ptr, stream_ptr)


def multi_workspace_size(B, n_new, T, n_q, n_kv, d_h, G, opts: AttnOpts | None = None) -> int:
    return int(_lib().fsq_decode_attn_multi_workspace_size(B, n_new, T, n_q, n_kv, d_h, G,
                                                           None if opts is None else C.byref(opts)))


def split_kernel(B, T, n_q, n_kv, d_h, G, opts: AttnOpts | None = None, n_new=1):
    """Name of the attention (split) kernel a call with these arguments launches, or None."""
    r = _lib().fsq_decode_attn_kernel(B, n_new, T, n_q, n_kv, d_h, G, None if opts is None else C.byref(opts))
    return None if r is None else r.decode()


def decode_attn_multi_raw(q_ptr, B, n_new, n_q, d_h, codes_ptr, bstride, T, G, wkv_ptr, n_kv, opts, ws_ptr,
                          ws_bytes, o_ptr, stream_ptr) -> int:
    return _lib().fsq_decode_attn_multi(q_ptr, B, n_new, n_q, d_h, codes_ptr, bstride, T, G, wkv_ptr, n_kv,
                                        None if opts is None else C.byref(opts), ws_ptr, ws_bytes, o_ptr, stream_ptr)


def decode_attn_noalloc_raw(q_ptr, B, n_q, d_h, codes_ptr, bstride, T, G, wkv_ptr, n_kv, opts, o_ptr,
                            stream_ptr) -> int:
    return _lib().fsq_decode_attn_noalloc(q_ptr, B, n_q, d_h, codes_ptr, bstride, T, G, wkv_ptr, n_kv,
                                          None if opts is None else C.byref(opts), o_ptr, stream_ptr)


def decode_attn_noalloc_status(stream=None) -> int:
    """Device status of the last allocation-free decode call on this device (blocking)."""
    return _lib().fsq_decode_attn_noalloc_status(_stream_ptr(stream))


def workspace_status(ws, stream=None) -> int:
    """Reads a device status word: a decode workspace's error word, or an
    append status word (a device tensor of at least 4 bytes).  Blocking."""
    return _lib().fsq_workspace_status(_ptr(ws), ws.numel() * ws.element_size(), _stream_ptr(stream))


# ---------------------------------------------------------------- tensor-level wrappers (torch for memory only)
def encode_pack(x, E, h=None, delta=0.5, out=None, stream=None, status_word=None, levels=16):
    """codes[n_tok, G*b/8] (uint8) for bf16 rows x[n_tok, C] through E[G, C].
    status_word: optional device tensor (>= 4 bytes, zeroed by the caller)
    that receives a device-detected failure (read it with workspace_status)."""
    import torch
    n_tok, C_ = x.shape
    G = E.shape[0]
    rb = row_bytes(G, levels)
    if out is None:
        out = torch.empty((n_tok, rb), dtype=torch.uint8, device=x.device)
    ldc = out.stride(0) if out.dim() == 2 else rb
    st = encode_pack_raw(_ptr(x), n_tok, x.stride(0), C_, _ptr(E), G, quant_params(h, delta, levels), _ptr(out),
                         ldc, _stream_ptr(stream), encode_opts(status_word))
    _check(st, "fsq_encode_pack")
    return out


def append_rows(x, E, cache, t0, h=None, delta=0.5, stream=None, status_word=None, levels=16):
    """One call appends n new tokens to each of the B rows of a [B, T_max, R]
    uint8 code cache: x is [B * n, C] (row b's tokens are x[b*n:(b+1)*n]) and
    they go to cache[b, t0:t0+n] (fsq_encode_opts.tokens_per_row = n)."""
    B, T_max, rb = cache.shape
    n_tok, C_ = x.shape
    G = E.shape[0]
    if B < 1 or n_tok % B or rb != row_bytes(G, levels) or cache.stride(2) != 1 or cache.stride(1) != rb:
        raise ValueError("append_rows: x must hold B * n rows and cache must be [B, T_max, G*b/8], rows contiguous")
    n = n_tok // B
    if not 0 <= t0 <= T_max - n:
        raise ValueError("append_rows: positions t0 .. t0+n-1 must lie inside the cache")
    st = encode_pack_raw(_ptr(x), n_tok, x.stride(0), C_, _ptr(E), G, quant_params(h, delta, levels),
                         int(cache.data_ptr()) + t0 * rb, rb, _stream_ptr(stream),
                         encode_opts(status_word, tokens_per_row=n, row_stride_bytes=cache.stride(0)))
    _check(st, "fsq_encode_pack")
    return cache


def quantize_pack_f32(u, h=None, delta=0.5, out=None, stream=None, levels=16):
    import torch
    n_tok, G = u.shape
    if out is None:
        out = torch.empty((n_tok, row_bytes(G, levels)), dtype=torch.uint8, device=u.device)
    st = quantize_pack_f32_raw(_ptr(u), n_tok, G, quant_params(h, delta, levels), _ptr(out), out.stride(0),
                               _stream_ptr(stream))
    _check(st, "fsq_quantize_pack_f32")
    return out


class Workspace:
    """Caller-owned device workspace, grown on demand (torch allocates it)."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buf = None

    def get(self, nbytes: int):
        import torch
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf


def decode_attn(q, codes, W_kv, T, n_kv, G, code_batch_stride=None, opts=None, workspace=None, out=None,
                stream=None):
    """o[B, n_q, d_h] = GQA decode attention over codes[B, T_max, G*b/8] (first T rows);
    the level count of the codes is opts.levels."""
    import torch
    B, n_q, d_h = q.shape
    if opts is None:
        opts = attn_opts()
    if code_batch_stride is None:
        # a size-1 leading dim may carry any stride (numpy gives 0); use the row extent then
        if codes.dim() == 3 and codes.shape[0] > 1:
            code_batch_stride = codes.stride(0)
        elif codes.dim() == 3:
            code_batch_stride = codes.shape[1] * codes.shape[2]
        else:
            code_batch_stride = T * row_bytes(G, opts.levels or 16)
    nbytes = workspace_size(B, T, n_q, n_kv, d_h, G, opts)
    if nbytes == 0:
        raise FsqError(FSQ_ERR_INVALID_ARG, "fsq_decode_attn_workspace_size")
    ws = (workspace or Workspace(q.device)).get(nbytes)
    if out is None:
        out = torch.empty((B, n_q, d_h), dtype=torch.float32 if opts.out_fp32 else torch.bfloat16, device=q.device)
    st = decode_attn_raw(_ptr(q), B, n_q, d_h, _ptr(codes), code_batch_stride, T, G, _ptr(W_kv), n_kv, opts,
                         _ptr(ws), ws.numel(), _ptr(out), _stream_ptr(stream))
    _check(st, "fsq_decode_attn")
    return out


def decode_attn_multi(q, codes, W_kv, T, n_kv, G, code_batch_stride=None, opts=None, workspace=None, out=None,
                      stream=None):
    """o[B, n_new, n_q, d_h]: query i of row b (q[b, i]) attends causally to the
    first L_b - n_new + i + 1 cached tokens of codes[b] (L_b = T or seq_lens[b])."""
    import torch
    B, n_new, n_q, d_h = q.shape
    if opts is None:
        opts = attn_opts()
    if code_batch_stride is None:
        if codes.dim() == 3 and codes.shape[0] > 1:
            code_batch_stride = codes.stride(0)
        elif codes.dim() == 3:
            code_batch_stride = codes.shape[1] * codes.shape[2]
        else:
            code_batch_stride = T * row_bytes(G, opts.levels or 16)
    nbytes = multi_workspace_size(B, n_new, T, n_q, n_kv, d_h, G, opts)
    if nbytes == 0:
        raise FsqError(FSQ_ERR_INVALID_ARG, "fsq_decode_attn_multi_workspace_size")
    ws = (workspace or Workspace(q.device)).get(nbytes)
    if out is None:
        out = torch.empty((B, n_new, n_q, d_h), dtype=torch.float32 if opts.out_fp32 else torch.bfloat16,
                          device=q.device)
    st = decode_attn_multi_raw(_ptr(q), B, n_new, n_q, d_h, _ptr(codes), code_batch_stride, T, G, _ptr(W_kv), n_kv,
                               opts, _ptr(ws), ws.numel(), _ptr(out), _stream_ptr(stream))
    _check(st, "fsq_decode_attn_multi")
    return out


def default_scale(d_h: int) -> float:
    return 1.0 / math.sqrt(d_h)
