"""fsq_decode_attn_noalloc: the decode entry point for callers that cannot
allocate device memory (its scratch is a fixed device array inside the
library instead of a caller-owned workspace).

Checked through the C ABI against the regular fsq_decode_attn on the same
inputs, on two calls in a row (the shared scratch keeps the previous call's
contents, which must not leak into the next result).  Collected last so a run
that stops at the first failure has already run every other test."""
import numpy as np
import pytest
import torch

import fsq_latent_decode_b200 as F
from fsq_latent_decode_b200 import _abi

from oracle import fsq_oracle as O

from cases import TOL, decoder_weights, oracle_cache, rel_err

pytestmark = pytest.mark.gpu


def _regular(q, codes, W, T, n_kv, G, opts):
    return F.decode_attn(q, codes, W, T, n_kv, G, opts=opts)


def _noalloc(q, codes, W, T, n_kv, G, opts, out):
    B, n_q, d_h = q.shape
    bstride = codes.shape[1] * codes.shape[2]
    st = _abi.decode_attn_noalloc_raw(q.data_ptr(), B, n_q, d_h, codes.data_ptr(), bstride, T, G, W.data_ptr(),
                                      n_kv, opts, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return st


@pytest.mark.parametrize("B,n_q,n_kv,G,T,variant,out_fp32",
                         [(2, 32, 8, 256, 3001, "absorbed", True), (3, 16, 8, 84, 517, "absorbed", True),
                          (2, 32, 8, 84, 1000, "expand", True), (2, 32, 8, 256, 2000, "absorbed", False)])
def test_noalloc_matches_regular_entry_point_twice(B, n_q, n_kv, G, T, variant, out_fp32):
    dev = "cuda"
    opts = F.attn_opts(variant=variant, out_fp32=out_fp32)
    dtype = torch.float32 if out_fp32 else torch.bfloat16
    results = []
    for call in range(2):
        codes_np = oracle_cache(B, T, G, seed=900 + call)
        codes = torch.from_numpy(codes_np).to(dev)
        W, q = decoder_weights(n_q, n_kv, G, B, seed=950 + call)
        Wd, qd = W.to(dev), q.to(dev)
        ref = _regular(qd, codes, Wd, T, n_kv, G, opts).float().cpu().numpy()
        out = torch.full((B, n_q, 128), float("nan"), device=dev, dtype=dtype)
        assert _noalloc(qd, codes, Wd, T, n_kv, G, opts, out) == F.FSQ_OK
        assert _abi.decode_attn_noalloc_status() == F.FSQ_OK  # no bounded device wait gave up
        got = out.float().cpu().numpy()
        assert np.isfinite(got).all()
        assert rel_err(got, ref) <= TOL
        if call == 1:  # also straight against the fp64 oracle
            assert rel_err(got, O.decode_attn(q.float().numpy(), codes_np[:, :T], W.float().numpy(), n_kv, G)) <= TOL
        results.append(got)
    assert not np.array_equal(results[0], results[1])  # the two calls really had different inputs


def test_noalloc_reports_a_bounded_wait_that_gave_up():
    """The allocation-free call keeps its error word in the built-in scratch;
    its status reader must show a device wait that ran out (made to run out by
    the test-only stall), and the next call must clear it."""
    dev = "cuda"
    B, n_q, n_kv, G, T = 2, 32, 8, 84, 3000
    codes = torch.from_numpy(oracle_cache(B, T, G, seed=970)).to(dev)
    W, q = decoder_weights(n_q, n_kv, G, B, seed=971)
    Wd, qd = W.to(dev), q.to(dev)
    out = torch.empty((B, n_q, 128), device=dev)
    stall = F.attn_opts(variant="absorbed", out_fp32=True, debug_stall_ns=2_000_000)
    assert _noalloc(qd, codes, Wd, T, n_kv, G, stall, out) == F.FSQ_OK
    assert _abi.decode_attn_noalloc_status() == F.FSQ_ERR_TIMEOUT
    opts = F.attn_opts(variant="absorbed", out_fp32=True)
    assert _noalloc(qd, codes, Wd, T, n_kv, G, opts, out) == F.FSQ_OK
    assert _abi.decode_attn_noalloc_status() == F.FSQ_OK
    assert rel_err(out.cpu().numpy(), _regular(qd, codes, Wd, T, n_kv, G, opts).cpu().numpy()) <= TOL


def test_noalloc_rejects_requests_beyond_its_scratch():
    # a workspace far above the built-in maximum: refused before any launch
    B, n_q, n_kv, G, T = 1024, 32, 8, 256, 1 << 20
    opts = F.attn_opts(variant="absorbed")
    assert F.workspace_size(B, T, n_q, n_kv, 128, G, opts) > _abi.NOALLOC_SCRATCH_BYTES
    st = _abi.decode_attn_noalloc_raw(16, B, n_q, 128, 16, T * G // 2, T, G, 16, n_kv, opts, 16,
                                      torch.cuda.current_stream().cuda_stream)
    assert st == F.FSQ_ERR_WORKSPACE
    # invalid arguments report the same status as the regular entry point
    assert _abi.decode_attn_noalloc_raw(16, 1, 32, 64, 16, 4096, 32, 256, 16, 8, opts, 16, None) == F.FSQ_ERR_UNSUPPORTED
