"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/fsq.h declares, computes its threshold table and
workspace plans, and rejects bad arguments before touching the device."""
import ctypes as C
import math
import os
import re

import numpy as np
import pytest

import fsq_latent_decode_b200 as F
from fsq_latent_decode_b200 import _abi
from oracle import fsq_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "fsq.h")).read()
    return sorted(set(re.findall(r"FSQ_API\s+[^;(]*?\b(fsq_\w+)\s*\(", src)))


def test_header_symbols_are_exported():
    names = declared_symbols()
    assert len(names) >= 9
    assert sorted(_abi.EXPORTED) == names
    for n in names:
        assert hasattr(F.lib, n), n


def test_noalloc_scratch_size_matches_header():
    src = open(os.path.join(ROOT, "include", "fsq.h")).read()
    m = re.search(r"#define\s+FSQ_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", src)
    assert m, "FSQ_NOALLOC_SCRATCH_BYTES not found in include/fsq.h"
    assert _abi.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_struct_layouts_match_header():
    """The ctypes mirrors of fsq_attn_opts and fsq_encode_opts list the header's fields in order."""
    src = open(os.path.join(ROOT, "include", "fsq.h")).read()

    def fields(struct):
        body = re.search(r"typedef struct \{([^{}]*)\}\s*" + struct + ";", src).group(1)
        body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
        return [re.findall(r"(\w+)\s*(?:\[\d+\])?\s*$", d.strip())[0] for d in body.split(";") if d.strip()]

    assert fields("fsq_attn_opts") == [f[0] for f in _abi.AttnOpts._fields_]
    assert fields("fsq_encode_opts") == [f[0] for f in _abi.EncodeOpts._fields_]


def test_format_version_and_status_strings():
    assert F.lib.fsq_format_version() == 1
    for s in range(0, -7, -1):
        assert F.status_string(s) and F.status_string(s) != "unknown status"


@pytest.mark.parametrize("h", [7.5, 7.5075])
def test_threshold_table_agrees_with_oracle(h):
    th = np.array(F.thresholds(h, 0.5), dtype=np.float32)
    assert np.all(np.diff(th) > 0)
    h = float(np.float32(h))  # the library's h is an fp32 parameter; evaluate the oracle there
    for k, t in enumerate(th):
        below = np.nextafter(t, np.float32(-np.inf), dtype=np.float32)
        # the oracle (literal tanh) puts theta_k in level k-7 and the fp32 value
        # just below it in level k-8: theta_k is the first fp32 of the new level
        lv = O.fsq_quantize(np.array([float(t), float(below)], dtype=np.float64), h, 0.5)
        assert lv[0] == k - 7 and lv[1] == k - 8, (k, t)


def test_threshold_param_checks():
    for h, d in [(7.5, 0.0), (0.4, 0.5), (9.0, 0.5), (7.9, 0.7)]:
        with pytest.raises(F.FsqError):
            F.thresholds(h, d)


def _opts(**kw):
    return F.attn_opts(**kw)


def test_workspace_plan_is_deterministic_and_validates():
    ws = F.workspace_size(16, 131072, 32, 8, 128, 256, _opts())
    assert ws > 0 and ws % 256 == 0
    assert ws == F.workspace_size(16, 131072, 32, 8, 128, 256, _opts())
    assert F.workspace_size(1, 1, 16, 8, 128, 84, _opts()) > 0
    assert F.workspace_size(1, 0, 16, 8, 128, 84, _opts()) == 0          # T = 0
    assert F.workspace_size(1, 10, 16, 8, 64, 84, _opts()) == 0          # d_h != 128
    assert F.workspace_size(1, 10, 12, 8, 128, 84, _opts()) == 0         # n_q % n_kv
    assert F.workspace_size(1, 10, 16, 8, 128, 85, _opts()) == 0         # odd G
    assert F.workspace_size(1, 10, 16, 8, 128, 578, _opts()) == 0        # G > FSQ_MAX_G
    assert F.workspace_size(1, 10, 16, 8, 128, 258, _opts()) > 0         # CUDA-core absorbed form
    assert F.workspace_size(1, 10, 16, 8, 128, 84, _opts(variant="absorbed", rope_knorm=True)) == 0
    assert F.workspace_size(1, 10, 16, 8, 128, 84, _opts(rope_knorm=True)) > 0  # auto -> expand


def test_level_count_plans():
    """4 and 256 levels run the CUDA-core forms; shapes whose shared-memory
    tiles would not fit are refused before any launch."""
    def ws(G, L, n_q=32, **kw):
        return F.workspace_size(2, 4096, n_q, 8, 128, G, _opts(levels=L, **kw))
    for L, G in ((4, 320), (4, 576), (16, 160), (16, 288), (256, 80), (256, 144)):
        assert ws(G, L) > 0, (L, G)                    # Table 8 widths at 80 and 144 B/token
    assert ws(86, 4) == 0                               # 2-bit rows need G % 4 == 0
    assert ws(84, 8) == 0 and ws(84, 2) == 0            # unsupported level counts
    assert ws(576, 4, n_q=64) == 0                      # absorbed tile exceeds shared memory
    assert ws(144, 256, variant="hybrid", rope_knorm=True) == 0  # tensor-core forms read 16 levels
    assert ws(320, 4, rope_knorm=True) > 0              # AUTO + rope -> CUDA-core expand form
    assert ws(576, 4, rope_knorm=True) == 0             # W_kv^(j) of G=576 exceeds shared memory
    # levels 0 selects 16: same plan as 16
    assert ws(256, 0) == ws(256, 16)
    # 256-level codes on the tensor-core absorbed kernel read each byte as two
    # nibbles: the plan of G = 80 at 256 levels is that of G = 160 at 16 levels
    assert ws(80, 256) == ws(160, 16)
    assert ws(128, 256) == ws(256, 16)
    assert ws(144, 256) != ws(288, 16)  # 2 x 144 exceeds the kernel's widths: CUDA-core form


@pytest.mark.parametrize("L", [4, 256])
def test_threshold_table_other_levels_agrees_with_oracle(L):
    h = (L - 1) / 2
    th = np.array(F.thresholds(h, 0.5, levels=L), dtype=np.float32)
    assert len(th) == L - 1 and np.all(np.diff(th) > 0)
    for k, t in enumerate(th):
        below = np.nextafter(t, np.float32(-np.inf), dtype=np.float32)
        lv = O.fsq_quantize(np.array([float(t), float(below)]), h, 0.5, L)
        assert lv[0] == k + 1 - L // 2 and lv[1] == k - L // 2, (k, t)


def test_level_param_checks():
    for h, d, L in [(1.5, 0.5, 8), (2.1, 0.5, 4), (127.5, 1.5, 256), (1.0, 1.0, 4)]:
        with pytest.raises(F.FsqError):
            F.thresholds(h, d, levels=L)
    qp = F.quant_params(levels=4)
    assert (qp.h, qp.delta, qp.levels) == (1.5, 0.5, 4)
    # encode: 2-bit rows need G % 4 == 0; the row must hold G*b/8 bytes
    assert F.encode_pack_raw(16, 4, 64, 64, 16, 86, qp, 16, 64, None) == F.FSQ_ERR_UNSUPPORTED
    assert F.encode_pack_raw(16, 4, 64, 64, 16, 88, qp, 16, 21, None) == F.FSQ_ERR_INVALID_ARG
    assert F.encode_pack_raw(16, 4, 64, 64, 16, 578, F.quant_params(levels=256), 16, 578, None) == \
        F.FSQ_ERR_UNSUPPORTED
    assert F.quantize_pack_f32_raw(16, 3, 144, F.quant_params(levels=256), 16, 143, None) == F.FSQ_ERR_INVALID_ARG
    assert F.encode_pack_raw(16, 4, 64, 64, 16, 88, F.quant_params(1.5, 0.5, 8), 16, 64, None) == \
        F.FSQ_ERR_UNSUPPORTED


def test_multi_query_plans_and_checks():
    o = _opts()
    # n_new queries per row plan as B * n_new grid rows
    assert F.multi_workspace_size(4, 8, 4096, 32, 8, 128, 256, o) == F.workspace_size(32, 4096, 32, 8, 128, 256, o)
    assert F.multi_workspace_size(4, 1, 4096, 32, 8, 128, 84, o) == F.workspace_size(4, 4096, 32, 8, 128, 84, o)
    assert F.multi_workspace_size(4, 0, 4096, 32, 8, 128, 84, o) == 0
    assert F.multi_workspace_size(8192, 8, 4096, 32, 8, 128, 84, o) == 0  # 65536 grid rows
    args = (16, 4, 0, 32, 128, 16, 4096 * 128, 4096, 256, 16, 8, o, 256, 1 << 30, 16, None)
    assert F.decode_attn_multi_raw(*args) == F.FSQ_ERR_INVALID_ARG                     # n_new = 0
    assert F.decode_attn_multi_raw(16, 9000, 8, 32, 128, 16, 4096 * 128, 4096, 256, 16, 8, o, 256, 1 << 30, 16,
                                   None) == F.FSQ_ERR_UNSUPPORTED                         # B * n_new > 65535
    assert F.decode_attn_multi_raw(None, 0, 4, 32, 128, None, 4096 * 128, 4096, 256, None, 8, o, None, 0, None,
                                   None) == F.FSQ_OK                                      # empty batch


def test_invalid_arguments_return_before_launch():
    qp = F.quant_params()
    null = None
    # encode: bad shapes / params / nulls
    assert F.encode_pack_raw(null, 4, 64, 64, null, 256, qp, null, 128, null) == F.FSQ_ERR_INVALID_ARG
    assert F.encode_pack_raw(8, 4, 64, 63, 8, 256, qp, 8, 128, null) == F.FSQ_ERR_UNSUPPORTED
    assert F.encode_pack_raw(16, 4, 64, 64, 16, 255, qp, 16, 128, null) == F.FSQ_ERR_UNSUPPORTED
    assert F.encode_pack_raw(16, 4, 32, 64, 16, 256, qp, 16, 128, null) == F.FSQ_ERR_INVALID_ARG
    assert F.encode_pack_raw(16, 4, 64, 64, 16, 256, qp, 16, 64, null) == F.FSQ_ERR_INVALID_ARG
    assert F.encode_pack_raw(17, 4, 64, 64, 16, 256, qp, 16, 128, null) == F.FSQ_ERR_MISALIGNED
    assert F.encode_pack_raw(16, 4, 68, 64, 16, 256, qp, 16, 128, null) == F.FSQ_ERR_MISALIGNED
    assert F.encode_pack_raw(16, 4, 64, 64, 16, 256, F.quant_params(9.0, 0.5), 16, 128, null) == F.FSQ_ERR_INVALID_ARG
    assert F.encode_pack_raw(null, 0, 64, 64, null, 256, qp, null, 128, null) == F.FSQ_OK  # empty: no-op
    bad_word = F.encode_opts()
    bad_word.status_word = 18  # a status word must be 4-byte aligned
    assert F.encode_pack_raw(16, 4, 64, 64, 16, 256, qp, 16, 128, null, bad_word) == F.FSQ_ERR_MISALIGNED
    # grouped destination rows: a negative group size or row stride
    assert F.encode_pack_raw(16, 4, 64, 64, 16, 256, qp, 16, 128, null,
                             F.encode_opts(tokens_per_row=-1)) == F.FSQ_ERR_INVALID_ARG
    assert F.encode_pack_raw(16, 4, 64, 64, 16, 256, qp, 16, 128, null,
                             F.encode_opts(tokens_per_row=2, row_stride_bytes=-128)) == F.FSQ_ERR_INVALID_ARG
    assert F.quantize_pack_f32_raw(null, 3, 256, qp, null, 128, null) == F.FSQ_ERR_INVALID_ARG
    assert F.quantize_pack_f32_raw(8, 3, 256, qp, 16, 128, null) == F.FSQ_ERR_MISALIGNED
    # decode
    o = _opts()
    args = dict(q=16, B=1, n_q=16, d_h=128, codes=16, bs=4096, T=32, G=256, w=16, n_kv=8)

    def call(**kw):
        a = dict(args, **kw)
        ws = kw.get("ws", 256)
        wsb = kw.get("wsb", 1 << 30)
        return F.decode_attn_raw(a["q"], a["B"], a["n_q"], a["d_h"], a["codes"], a["bs"], a["T"], a["G"], a["w"],
                                 a["n_kv"], o, ws, wsb, 16, None)

    assert call(T=0) == F.FSQ_ERR_INVALID_ARG
    assert call(d_h=64) == F.FSQ_ERR_UNSUPPORTED
    assert call(n_q=12) == F.FSQ_ERR_INVALID_ARG
    assert call(G=85) == F.FSQ_ERR_UNSUPPORTED
    assert call(codes=None) == F.FSQ_ERR_INVALID_ARG
    assert call(bs=100) == F.FSQ_ERR_INVALID_ARG          # stride < T*G*b/8
    assert call(bs=4104) == F.FSQ_ERR_MISALIGNED          # stride % 16
    assert call(codes=24) == F.FSQ_ERR_MISALIGNED
    assert call(q=18) == F.FSQ_ERR_MISALIGNED
    assert call(wsb=16) == F.FSQ_ERR_WORKSPACE
    assert call(ws=None) == F.FSQ_ERR_WORKSPACE
    assert call(ws=272) == F.FSQ_ERR_MISALIGNED
    assert call(B=0, q=None, codes=None, w=None) == F.FSQ_OK  # empty batch: no-op
    o.seq_lens = 18  # per-row lengths must be 4-byte aligned int32
    assert call() == F.FSQ_ERR_MISALIGNED
    o.seq_lens = None
    # status words: null and misaligned pointers are refused before any copy
    assert F.lib.fsq_workspace_status(None, 256, None) == F.FSQ_ERR_INVALID_ARG
    assert F.lib.fsq_workspace_status(16, 2, None) == F.FSQ_ERR_INVALID_ARG
    assert F.lib.fsq_workspace_status(18, 4, None) == F.FSQ_ERR_MISALIGNED


def test_append_rows_rejects_bad_shapes_before_any_call():
    """append_rows checks the cache shape, the token count and the positions
    on the host, before it reaches the library."""
    import torch
    x = torch.zeros((10, 64), dtype=torch.bfloat16)
    E = torch.zeros((256, 64), dtype=torch.bfloat16)
    cache = torch.zeros((5, 40, 128), dtype=torch.uint8)
    with pytest.raises(ValueError):
        F.append_rows(x[:9], E, cache, 0)                   # 9 tokens over 5 rows
    with pytest.raises(ValueError):
        F.append_rows(x, E, cache[:, :, :64], 0)            # rows of 64 bytes for G=256 at 4 bits
    with pytest.raises(ValueError):
        F.append_rows(x, E, cache, 39)                      # positions 39, 40 past T_max = 40
    with pytest.raises(ValueError):
        F.append_rows(x, E, cache[:, ::2], 0)               # every other position: token rows 256 bytes apart
