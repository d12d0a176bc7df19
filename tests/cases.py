"""Seeded test inputs shared by the parity tests (no method arithmetic here
except through the oracle, which makes every stored code)."""
from __future__ import annotations

import math

import numpy as np
import torch

from fsq_latent_decode_b200 import synth
from oracle import fsq_oracle as O

TOL = 5e-3  # max|delta| / max|ref| for attention outputs (bf16 operands, fp32 accumulation)


def padded_len(T: int, G: int) -> int:
    """Smallest T_max >= T whose batch stride T_max*G/2 is a multiple of 16 bytes."""
    half = G // 2
    t = T
    while (t * half) % 16:
        t += 1
    return max(t, 1)


def oracle_cache(B, T, G, seed, h=7.5, rows=None, T_max=None):
    """Packed cache [B, T_max, G/2] (numpy uint8).

    Rows in `rows` (default: all) hold the oracle's eq.-(2) codes of seeded
    pre-activations u ~ N(0, 4) (the law of E x for the seeded E and x);
    other rows hold uniform random bytes (every byte is a valid code pair)."""
    T_max = padded_len(T, G) if T_max is None else T_max
    rows = range(B) if rows is None else rows
    codes = np.empty((B, T_max, G // 2), dtype=np.uint8)
    gen = synth._gen(synth.workload_seed(seed, 99))
    codes[:] = synth.random_bytes((B, T_max, G // 2), gen).numpy()
    hq = float(np.float32(h))
    for b in rows:
        g = synth._gen(synth.workload_seed(seed, b))
        chunk = 1 << 18
        for t0 in range(0, T, chunk):
            n = min(chunk, T - t0)
            u = synth.preactivations(n, G, g).numpy()
            codes[b, t0:t0 + n] = O.quantize_pack(u, hq)
    return codes


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    m = np.isfinite(ref)
    return float(np.abs(got[m] - ref[m]).max() / np.abs(ref[m]).max())


def decoder_weights(n_q, n_kv, G, B, seed, d_h=128):
    gen = synth._gen(synth.workload_seed(seed, 7))
    W_kv, q = synth.decoder_inputs(B, n_q, n_kv, d_h, G, gen)
    return W_kv, q


def gemm_error_bound(x, E, unit_roundoff=2.0 ** -23):
    """Forward-error bound gamma_C * sum_c |E_ic x_tc| of an fp32 dot product of
    length C, gamma_C = C u / (1 - C u) (the classical bound for summation in any
    order with unit roundoff u; Higham, Accuracy and Stability of Numerical
    Algorithms, section 3.1).  The bf16 x bf16 products are exact in fp32, so
    only the accumulation rounds.  u = 2^-23, one fp32 ulp rather than half of
    one: the tensor core's fp32 accumulation is not specified to round to
    nearest, and this value also covers truncating (round-toward-zero) adds."""
    Cdim = x.shape[1]
    u = unit_roundoff
    gam = Cdim * u / (1 - Cdim * u)
    return gam * (np.abs(np.asarray(x, np.float64)) @ np.abs(np.asarray(E, np.float64)).T)


def record(kind: str, **fields):
    """Appends one JSON line to $FSQ_PARITY_RECORD (if set): counts that a GPU
    run reports, such as code mismatches near a rounding boundary."""
    import json
    import os
    path = os.environ.get("FSQ_PARITY_RECORD")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(dict(kind=kind, **fields)) + "\n")


def fp16_key_floor(q, codes, W_kv, n_kv, G, ref):
    """The error (max|delta|/max|ref| against the oracle's `ref`) of decode
    attention computed exactly except that the rebuilt keys are rounded to fp16
    before the score product: the floor any kernel holding its keys in fp16
    reaches.  Built from the oracle's own functions (reconstruct_kv, softmax);
    used only to bound the key-expanding forms where scores span hundreds of
    log2 units (q x 30), where bf16 keys would be off by ~14 %."""
    import math as _m
    q = np.asarray(q, dtype=np.float64)
    B, n_q, d_h = q.shape
    grp = n_q // n_kv
    out = np.zeros((B, n_q, d_h))
    for b in range(B):
        K, V = O.reconstruct_kv(O.unpack(codes[b], G), W_kv, n_kv, d_h)
        K16 = K.astype(np.float16).astype(np.float64)
        for h in range(n_q):
            j = h // grp
            out[b, h] = O.softmax((K16[j] @ q[b, h]) / _m.sqrt(d_h)) @ V[j]
    return rel_err(out, ref)

