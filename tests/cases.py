"""Seeded test inputs shared by the parity tests (no method arithmetic here
except through the oracle, which makes every stored code)."""
from __future__ import annotations

import math

import numpy as np
import torch

from fsq_latent_decode_b200 import synth
from oracle import fsq_oracle as O

TOL = 5e-3  # max|delta| / max|ref| for attention outputs (bf16 operands, fp32 accumulation)


def row_bytes(G: int, levels: int = 16) -> int:
    """Bytes of a packed row, G * b / 8 (b = 2, 4, 8 at 4, 16, 256 levels)."""
    return G * O.bits_per_coordinate(levels) // 8


def padded_len(T: int, G: int, levels: int = 16) -> int:
    """Smallest T_max >= T whose batch stride T_max*G*b/8 is a multiple of 16 bytes."""
    rb = row_bytes(G, levels)
    t = T
    while (t * rb) % 16:
        t += 1
    return max(t, 1)


def oracle_cache(B, T, G, seed, h=None, rows=None, T_max=None, levels=16):
    """Packed cache [B, T_max, G*b/8] (numpy uint8) of `levels`-level codes.

    Rows in `rows` (default: all) hold the oracle's eq.-(2) codes of seeded
    pre-activations u ~ N(0, 4) (the law of E x for the seeded E and x);
    other rows hold uniform random bytes (every byte is a valid group of codes
    at 4, 16 and 256 levels).  h defaults to (L-1)/2, as the library's."""
    T_max = padded_len(T, G, levels) if T_max is None else T_max
    rows = range(B) if rows is None else rows
    rb = row_bytes(G, levels)
    codes = np.empty((B, T_max, rb), dtype=np.uint8)
    gen = synth._gen(synth.workload_seed(seed, 99))
    codes[:] = synth.random_bytes((B, T_max, rb), gen).numpy()
    hq = float(np.float32(O.default_h(levels) if h is None else h))
    for b in rows:
        g = synth._gen(synth.workload_seed(seed, b))
        chunk = 1 << 18
        for t0 in range(0, T, chunk):
            n = min(chunk, T - t0)
            u = synth.preactivations(n, G, g).numpy()
            codes[b, t0:t0 + n] = O.quantize_pack(u, hq, levels=levels)
    return codes


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    m = np.isfinite(ref)
    return float(np.abs(got[m] - ref[m]).max() / np.abs(ref[m]).max())


def decoder_weights(n_q, n_kv, G, B, seed, d_h=128, levels=16):
    gen = synth._gen(synth.workload_seed(seed, 7))
    W_kv, q = synth.decoder_inputs(B, n_q, n_kv, d_h, G, gen, levels=levels)
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



def query_grid_floor(q, codes, W_kv, n_kv, G, ref, levels=16):
    """The error (max|delta|/max|ref| against the oracle's `ref`) of decode
    attention computed exactly except that each head's absorbed query weights
    are held on a grid of step m / (127 * 128), m the largest of them: the
    precision of the tensor-core absorbed form, which stores q'_h = scale *
    W_k^T q_h as two int8 terms.  At 256 levels that form reads each 8-bit code
    n as its nibbles lo, hi (level = (lo - 8) + 16 (hi - 8) + 8) with weights
    q'_i and 16 q'_i, so m is 16 max|q'| there.  Built from the oracle's own
    functions (split_wkv, unpack, softmax); used only to bound outputs where
    scores span hundreds of log2 units (q x 30), where bf16 query weights would
    be off by 5 to 14 %."""
    q = np.asarray(q, dtype=np.float64)
    B, n_q, d_h = q.shape
    grp = n_q // n_kv
    Wk, Wv = O.split_wkv(W_kv, n_kv, d_h)
    out = np.zeros((B, n_q, d_h))
    for b in range(B):
        lv = O.unpack(codes[b], G, levels)
        z = lv.astype(np.float64)
        if levels == 256:
            n = lv + 128
            lo, hi = (n & 15) - 8.0, (n >> 4) - 8.0
        for h in range(n_q):
            j = h // grp
            qa = (Wk[j].T @ q[b, h]) / math.sqrt(d_h)
            if levels == 256:
                step = 16 * np.abs(qa).max() / (127 * 128)
                s = lo @ (np.round(qa / step) * step) + hi @ (np.round(16 * qa / step) * step)
            else:
                step = np.abs(qa).max() / (127 * 128)
                s = z @ (np.round(qa / step) * step)
            out[b, h] = Wv[j] @ (O.softmax(s) @ z)
    return rel_err(out, ref)
