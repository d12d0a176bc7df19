"""Plain fp64 CPU oracle for Transformer-FSQ's append and decode-attention path.

TEST INFRASTRUCTURE ONLY.  This module is the slow, obviously-correct statement
of what the CUDA library computes.  Only the test suite, the package smoke check
and the benchmark's CPU-baseline / reference leg may import it.  It imports
nothing from the CUDA library and shares no helper, table or constant with it.

Sources (titles of the pages the method is described on):
  [S]  "Transformer-FSQ: Discrete Latents for Extreme KV-Cache Compression",
       picx.dev summary: Theoretical Basis (eq. 2), Methodology / Architecture
       (eqs. 4-5), Key Design Innovation (eq. 6), Closed-Form Conversion
       (eq. 8), Byte Budgeting.
  [D]  Transformer-FSQ slide deck (slides.en.tex): frame "A wide product code
       uses four bits per coordinate" (L=16, b=4, h=7.5075, delta=0.5,
       ceil(G*b/8) bytes per token per layer), frame "Attention pools codes
       before decoding values" (eqs. 5-6), frame "The kernel reads codes and
       never writes reconstructed K/V".

Readings taken where the pages leave a step open (each one is also listed in
the design notes):
  * the FSQ level fed to W_kv is the rounded integer itself (-8..7 for L=16);
  * rounding ties go to even (numpy.rint);
  * coordinate 2i is the low nibble of byte i, rows are G/2 bytes, no padding;
  * W_kv rows are [W_k; W_v] (eq. 8's order), head-major, d_h rows per head;
  * query head h reads kv head h // (n_q / n_kv);
  * the softmax scale defaults to 1/sqrt(d_h);
  * with the optional key-norm/RoPE flag: per-head RMS norm with a gain vector,
    then half-split rotary embedding at position t (the cache index).

Every function is pinned by tests/test_oracle_pins.py against closed forms,
invariants, a library routine (torch SDPA) and hand-worked cases; none of them
is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

# L=16 levels -> b = ceil(log2 L) = 4 bits per coordinate ([D], product-code frame).
# The deck's backup frame "the grid size is an allocation choice" (Table 8) also
# compares L = 4 (2 bits) and L = 256 (8 bits) at fixed byte budgets; every
# function below takes the level count L (default 16).
LEVELS = 16
BITS = 4
SUPPORTED_LEVELS = (4, 16, 256)


def bits_per_coordinate(levels=LEVELS):
    """b = ceil(log2 L) ([D] product-code frame)."""
    return int(math.ceil(math.log2(levels)))


def default_h(levels=LEVELS):
    """Reading for the bound h of eq. (2) at L levels (the deck gives only
    L = 16, h = 7.5075 = 7.5 x 1.001; the acceptance spec uses 7.5): h = (L-1)/2,
    so that with delta = 1/2 the rounded values are exactly -L/2 .. L/2 - 1."""
    return (levels - 1) / 2.0
# The deck prints h=7.5075, delta=0.5 for L=16 ([D]); the acceptance spec of
# this library uses h=7.5.  Both are accepted as parameters.
H_DEFAULT = 7.5
DELTA_DEFAULT = 0.5


# ---------------------------------------------------------------------------
# eq. (2): finite scalar quantisation, literal form
# ---------------------------------------------------------------------------
def fsq_bounded(u, h=H_DEFAULT, delta=DELTA_DEFAULT):
    """u~ = h * tanh(u + atanh(delta/h)) - delta   ([S] eq. 2; [D] product-code frame)."""
    u = np.asarray(u, dtype=np.float64)
    return h * np.tanh(u + math.atanh(delta / h)) - delta


def fsq_quantize(u, h=H_DEFAULT, delta=DELTA_DEFAULT, levels=LEVELS):
    """Forward value of eq. (2): round(u~) as an integer level.

    The straight-through term sg(round(u~) - u~) only changes gradients; its
    forward value is the rounded u~ ([D]: "the forward pass still uses rounded
    codes").  Ties round to even.  Levels outside the L-level grid are an error,
    never clamped.
    """
    ut = fsq_bounded(u, h, delta)
    c = np.rint(ut)
    lo, hi = -(levels // 2), levels // 2 - 1
    if c.size and (c.min() < lo or c.max() > hi):
        raise AssertionError(f"FSQ level outside the {levels}-level grid")
    return c.astype(np.int64)


def fsq_boundary_distance(u, h=H_DEFAULT, delta=DELTA_DEFAULT, levels=LEVELS):
    """Distance in u-space from u to the nearest rounding boundary of eq. (2).

    A boundary is a u whose u~ is a half-integer m + 1/2.  Inverting eq. (2)
    gives u = atanh((m + 1/2 + delta)/h) - atanh(delta/h).  Used only to
    excuse code mismatches of inputs that sit within a stated band of one.
    """
    u = np.asarray(u, dtype=np.float64)
    a = math.atanh(delta / h)
    halves = np.arange(-(levels // 2), levels // 2 - 1) + 0.5  # -7.5 .. 6.5 at L = 16
    arg = (halves + delta) / h
    ok = np.abs(arg) < 1.0
    bounds = np.arctanh(arg[ok]) - a
    d = np.abs(u[..., None] - bounds)
    return d.min(axis=-1)


# ---------------------------------------------------------------------------
# eq. (4): linear encoder followed by FSQ; nibble packing
# ---------------------------------------------------------------------------
def encode(x, E, h=H_DEFAULT, delta=DELTA_DEFAULT, levels=LEVELS):
    """z_t = Q_FSQ(E x_t) for every row x_t of x  ([S] Architecture, eq. 4).

    x: [N, C], E: [G, C] (any real dtype; converted exactly to fp64).
    Returns (levels int64 [N, G], u fp64 [N, G]).
    """
    x64 = np.asarray(x, dtype=np.float64)
    E64 = np.asarray(E, dtype=np.float64)
    u = x64 @ E64.T
    return fsq_quantize(u, h, delta, levels), u


def pack(levels, L=LEVELS):
    """Pack integer levels [..., G] into bytes [..., G*b/8], b = log2 L.

    Stored code n = level + L/2 (0..L-1, b bits).  Byte k holds coordinates
    k*(8/b) .. k*(8/b) + 8/b - 1, the first in its lowest b bits (at L = 16:
    coordinate 2i in the low nibble of byte i, 2i+1 in the high nibble).  No
    scale, zero point or norm is stored ([S] Summary: "no per-token
    quantisation metadata"; [D] product-code frame: ceil(G*b/8) bytes per
    token).
    """
    lv = np.asarray(levels, dtype=np.int64)
    G = lv.shape[-1]
    b = bits_per_coordinate(L)
    per = 8 // b
    if G % per:
        raise ValueError(f"G must be a multiple of {per} at {L} levels")
    n = lv + L // 2
    if n.size and (n.min() < 0 or n.max() > L - 1):
        raise ValueError(f"level outside the {L}-level grid")
    out = np.zeros(lv.shape[:-1] + (G // per,), dtype=np.int64)
    for i in range(per):
        out |= n[..., i::per] << (b * i)
    return out.astype(np.uint8)


def unpack(codes, G, L=LEVELS):
    """Inverse of pack: bytes [..., G*b/8] -> integer levels [..., G] (code - L/2)."""
    b = bits_per_coordinate(L)
    per = 8 // b
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    if c.shape[-1] != G // per:
        raise ValueError("codes row length must be G*b/8")
    out = np.empty(c.shape[:-1] + (G,), dtype=np.int64)
    for i in range(per):
        out[..., i::per] = (c >> (b * i)) & (L - 1)
    return out - L // 2


def encode_pack(x, E, h=H_DEFAULT, delta=DELTA_DEFAULT, levels=LEVELS):
    """Append path: packed codes [N, G*b/8] for rows of x (eq. 4 then packing)."""
    lv, _ = encode(x, E, h, delta, levels)
    return pack(lv, levels)


def quantize_pack(u, h=H_DEFAULT, delta=DELTA_DEFAULT, levels=LEVELS):
    """Quantiser + packing alone, on given pre-activations u [N, G]."""
    return pack(fsq_quantize(u, h, delta, levels), levels)


# ---------------------------------------------------------------------------
# eq. (5): shared decoder; optional key norm + RoPE
# ---------------------------------------------------------------------------
def split_wkv(W_kv, n_kv, d_h):
    """W_kv = [W_k; W_v] ([S] eq. 8 row order).  Returns W_k, W_v as [n_kv, d_h, G]."""
    W = np.asarray(W_kv, dtype=np.float64)
    if W.shape[0] != 2 * n_kv * d_h:
        raise ValueError("W_kv must have 2*n_kv*d_h rows")
    G = W.shape[1]
    Wk = W[: n_kv * d_h].reshape(n_kv, d_h, G)
    Wv = W[n_kv * d_h:].reshape(n_kv, d_h, G)
    return Wk, Wv


def rms_norm(k, gain, eps):
    """N_k: k * gain / sqrt(mean(k^2) + eps) over the last axis (reading of [S] eq. 5)."""
    k = np.asarray(k, dtype=np.float64)
    r = np.sqrt(np.mean(k * k, axis=-1, keepdims=True) + eps)
    return k / r * np.asarray(gain, dtype=np.float64)


def rope(k, positions, base):
    """RoPE_t with half-split pairing: (k_i, k_{i+d/2}) rotated by t * base^(-2i/d)."""
    k = np.asarray(k, dtype=np.float64)
    d = k.shape[-1]
    half = d // 2
    inv = base ** (-(np.arange(half, dtype=np.float64) * 2.0) / d)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]
    cos, sin = np.cos(ang), np.sin(ang)
    a, b = k[..., :half], k[..., half:]
    return np.concatenate([a * cos - b * sin, a * sin + b * cos], axis=-1)


def reconstruct_kv(levels, W_kv, n_kv, d_h, rope_knorm=None):
    """k_t = RoPE_t(N_k(W_k z_t)), v_t = W_v z_t per kv head ([S] eq. 5).

    levels: [T, G] integers.  Returns K, V as [n_kv, T, d_h] fp64.
    rope_knorm: None (keys used as W_k z_t) or dict(gain=[d_h], eps=, base=).
    """
    z = np.asarray(levels, dtype=np.float64)
    Wk, Wv = split_wkv(W_kv, n_kv, d_h)
    K = np.einsum("tg,jdg->jtd", z, Wk)
    V = np.einsum("tg,jdg->jtd", z, Wv)
    if rope_knorm is not None:
        T = z.shape[0]
        pos = np.arange(T, dtype=np.float64)
        K = np.stack([rope(rms_norm(K[j], rope_knorm["gain"], rope_knorm["eps"]),
                           pos, rope_knorm["base"]) for j in range(n_kv)])
    return K, V


def softmax(s):
    """Numerically plain softmax with max subtraction, fp64."""
    s = np.asarray(s, dtype=np.float64)
    m = np.max(s)
    e = np.exp(s - m)
    return e / e.sum()


# ---------------------------------------------------------------------------
# Decode attention: expanded K/V, then standard GQA softmax attention
# ---------------------------------------------------------------------------
def decode_attn(q, codes, W_kv, n_kv, G, scale=None, rope_knorm=None, rows=None, heads=None, lengths=None,
                levels=LEVELS):
    """Single-token GQA decode attention over a packed FSQ code cache.

    q: [B, n_q, d_h]; codes: [B, T, G/2] uint8; W_kv: [2*n_kv*d_h, G].
    For each batch row b and query head h with kv head j = h // (n_q/n_kv):
        k_t, v_t from eq. (5); s_t = scale * q_h . k_t; a = softmax(s);
        o_h = sum_t a_t v_t.
    rows / heads optionally restrict the computation to a sample (others are
    left as NaN) so large caches can be checked one output at a time.
    lengths: optional per-row token counts (a ragged batch): row b attends to
    its first lengths[b] cached tokens only.  levels: L of the code grid.
    Returns o [B, n_q, d_h] fp64.
    """
    q = np.asarray(q, dtype=np.float64)
    B, n_q, d_h = q.shape
    if n_q % n_kv:
        raise ValueError("n_q must be a multiple of n_kv")
    grp = n_q // n_kv
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    rows = range(B) if rows is None else rows
    heads = range(n_q) if heads is None else heads
    o = np.full((B, n_q, d_h), np.nan)
    for b in rows:
        lv = unpack(codes[b] if lengths is None else codes[b][: int(lengths[b])], G, levels)
        need_j = sorted({h // grp for h in heads})
        Wk, Wv = split_wkv(W_kv, n_kv, d_h)
        for j in need_j:
            # expand only kv head j (same arithmetic as reconstruct_kv for one head)
            z = lv.astype(np.float64)
            Kj = z @ Wk[j].T
            Vj = z @ Wv[j].T
            if rope_knorm is not None:
                pos = np.arange(z.shape[0], dtype=np.float64)
                Kj = rope(rms_norm(Kj, rope_knorm["gain"], rope_knorm["eps"]), pos, rope_knorm["base"])
            for h in heads:
                if h // grp != j:
                    continue
                a = softmax(scale * (Kj @ q[b, h]))
                o[b, h] = a @ Vj
    return o


def decode_attn_multi(q, codes, W_kv, n_kv, G, scale=None, rope_knorm=None, lengths=None, levels=LEVELS,
                      rows=None, heads=None):
    """Several new queries per batch row attending to the code cache, causally
    (chunked prefill or speculative decoding: [S] Methodology eqs. 4-5 for more
    than one query).

    q: [B, n_new, n_q, d_h].  Row b holds L_b cached tokens (lengths[b], else
    all T rows of codes), the last n_new of them the new tokens; query i sits
    at position L_b - n_new + i and attends to tokens 0 .. L_b - n_new + i.
    Each query is therefore a single-token decode over its own prefix of the
    cache.  rows / heads optionally restrict the computation (others left NaN).
    Returns o [B, n_new, n_q, d_h] fp64.
    """
    q = np.asarray(q, dtype=np.float64)
    B, n_new, n_q, d_h = q.shape
    T = codes.shape[1]
    o = np.full(q.shape, np.nan)
    for b in (range(B) if rows is None else rows):
        L = T if lengths is None else int(lengths[b])
        if L < n_new:
            raise ValueError("a row must hold at least its n_new new tokens")
        for i in range(n_new):
            n = L - n_new + i + 1
            o[b, i] = decode_attn(q[b, i][None], codes[b:b + 1, :n], W_kv, n_kv, G, scale=scale,
                                  rope_knorm=rope_knorm, levels=levels, heads=heads)[0]
    return o


def decode_attn_pooled(q, codes, W_kv, n_kv, G, scale=None):
    """eq. (6) form, for cross-checks only: pool codes with the attention
    weights, then apply W_v once; keys scored as (W_k^T q) . z_t.

    Equal to decode_attn when the key norm/RoPE flag is off
    ([S] Key Design Innovation, eq. 6; [D] "Attention pools codes before
    decoding values").
    """
    q = np.asarray(q, dtype=np.float64)
    B, n_q, d_h = q.shape
    grp = n_q // n_kv
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    Wk, Wv = split_wkv(W_kv, n_kv, d_h)
    o = np.empty((B, n_q, d_h))
    for b in range(B):
        z = unpack(codes[b], G).astype(np.float64)
        for h in range(n_q):
            j = h // grp
            qa = Wk[j].T @ q[b, h]              # W_k^T q   [G]
            a = softmax(scale * (z @ qa))
            zbar = a @ z                         # sum_t a_t z_t   [G]
            o[b, h] = Wv[j] @ zbar
    return o


def lse_merge(parts):
    """Merge (m, l, acc) partials of disjoint token ranges by log-sum-exp.

    Each part is (m, l, acc) with m = max score, l = sum exp(s - m),
    acc = sum exp(s - m) * value.  Returns acc_total / l_total.
    ([D] kernel frame: "merge partials").
    """
    M = max(p[0] for p in parts)
    L = sum(p[1] * math.exp(p[0] - M) for p in parts)
    A = sum(p[2] * math.exp(p[0] - M) for p in parts)
    return A / L


def partial_attn(s, V):
    """(m, l, acc) of one token range with scores s [T'] and values V [T', d]."""
    s = np.asarray(s, dtype=np.float64)
    m = float(np.max(s))
    e = np.exp(s - m)
    return m, float(e.sum()), e @ np.asarray(V, dtype=np.float64)


# ---------------------------------------------------------------------------
# Byte budgeting ([S] Byte Budgeting; [D] kernel frame)
# ---------------------------------------------------------------------------
def code_bytes_per_token(G, bits=BITS):
    """ceil(G*b/8) bytes per token per layer ([D] product-code frame)."""
    return -(-G * bits // 8)


def full_cache_bytes_per_token(n_kv, d_h, elem_bytes=2):
    """c_full = 2 * n_kv * d_h * sizeof(float16) ([S] Byte Budgeting)."""
    return 2 * n_kv * d_h * elem_bytes
