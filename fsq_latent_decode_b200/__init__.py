"""fsq_latent_decode_b200 — B200 (sm_100a) CUDA library for Transformer-FSQ's
decode hot path: append tokens to a bit-packed FSQ code cache (4-bit codes
at the default 16 levels; 2- or 8-bit at 4 or 256) and run single-token GQA
attention directly over the codes.

The compute lives in libfsq.so (C ABI, include/fsq.h); this package is its
ctypes binding plus seeded synthetic inputs.  PyTorch only provides device
memory and streams.  The library is loaded on first use.
"""
from ._abi import (  # noqa: F401
    EXPORTED, FSQ_OK, append_rows, FSQ_ERR_CUDA, FSQ_ERR_INVALID_ARG, FSQ_ERR_MISALIGNED, FSQ_ERR_TIMEOUT,
    FSQ_ERR_UNSUPPORTED, FSQ_ERR_WORKSPACE, AttnOpts, EncodeOpts, FsqError, QuantParams, Workspace, attn_opts,
    decode_attn, decode_attn_multi, decode_attn_multi_raw, decode_attn_noalloc_status, decode_attn_raw,
    multi_workspace_size, split_kernel, encode_opts, encode_pack, encode_pack_raw, quant_params,
    quantize_pack_f32, quantize_pack_f32_raw, row_bytes, bits_of_levels, status_string, thresholds, workspace_size,
    workspace_status,
)


def __getattr__(name):  # `lib` (the loaded libfsq.so) is mapped on first access
    if name == "lib":
        from . import _abi
        return _abi.lib
    raise AttributeError(name)

__all__ = ["encode_pack", "quantize_pack_f32", "decode_attn", "decode_attn_multi", "attn_opts", "thresholds", "workspace_size",
           "Workspace", "FsqError"]
