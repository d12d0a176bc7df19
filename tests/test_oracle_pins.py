"""Pins for the fp64 CPU oracle: checks it against what the pages and the
mathematics fix, never against itself.

Pages: "Transformer-FSQ: Discrete Latents for Extreme KV-Cache Compression"
(picx.dev summary, eqs. 2, 4, 5, 6, 8 and Byte Budgeting) and the Transformer-FSQ
slide deck (frames "A wide product code uses four bits per coordinate",
"Attention pools codes before decoding values", "The kernel reads codes and
never writes reconstructed K/V").
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.stats import norm

from oracle import fsq_oracle as O


# ---------------------------------------------------------------- eq. (2)
@pytest.mark.parametrize("h", [7.5, 7.5075])
def test_zero_maps_to_level_zero(h):
    # h * tanh(atanh(delta/h)) - delta = delta - delta = 0 for any h.
    assert O.fsq_quantize(np.array([0.0]), h, 0.5)[0] == 0
    assert abs(O.fsq_bounded(0.0, h, 0.5)) < 1e-15


@pytest.mark.parametrize("h", [7.5, 7.5075])
def test_saturation_and_sixteen_levels(h):
    u = np.linspace(-40, 40, 200001)
    c = O.fsq_quantize(u, h, 0.5)
    assert c[0] == -8 and c[-1] == 7
    assert np.all(np.diff(c) >= 0), "eq. 2 must be monotone in u"
    assert sorted(set(c.tolist())) == list(range(-8, 8))
    # u~ lies in [-h - delta, h - delta] (open interval; fp64 tanh saturates)
    ut = O.fsq_bounded(u, h, 0.5)
    assert ut.min() >= -h - 0.5 and ut.max() <= h - 0.5


def _closed_form_thresholds(h, delta):
    # Hand inversion of eq. (2): the level steps from m to m+1 where
    # u~ = m + 1/2, i.e. tanh(u + a) = (m + 1/2 + delta)/h, a = atanh(delta/h).
    a = math.atanh(delta / h)
    out = []
    for m in range(-8, 7):
        out.append(math.atanh((m + 0.5 + delta) / h) - a)
    return np.array(out)


@pytest.mark.parametrize("h", [7.5, 7.5075])
def test_codes_equal_threshold_count_off_band(h):
    th = _closed_form_thresholds(h, 0.5)
    u = np.linspace(-12.0, 12.0, 2_000_001)
    c = O.fsq_quantize(u, h, 0.5)
    n = (u[:, None] >= th[None, :]).sum(axis=1) - 8
    d = np.abs(u[:, None] - th[None, :]).min(axis=1)
    far = d > 1e-9
    assert np.array_equal(c[far], n[far])
    # the oracle's boundary distance agrees with the hand inversion
    assert np.allclose(O.fsq_boundary_distance(u[::997], h, 0.5), d[::997], atol=1e-12)


def test_threshold_values_at_h7p5():
    # Hand-evaluated atanh values (m+1)/7.5 - atanh(0.5/7.5), m = -8..6, to 5 places.
    printed = [-1.75041, -1.16538, -0.87148, -0.66156, -0.49041, -0.34004, -0.20090,
               -0.06677, 0.06737, 0.20651, 0.35688, 0.52803, 0.73795, 1.03185, 1.61688]
    th = _closed_form_thresholds(7.5, 0.5)
    assert np.allclose(th, printed, atol=6e-6)
    for t in th:  # the oracle steps exactly across each threshold
        lo, hi = O.fsq_quantize(np.array([t - 1e-7, t + 1e-7]), 7.5, 0.5)
        assert hi == lo + 1


def test_threshold_endpoints_at_deck_h():
    # The slide deck's h = 7.5075 (four-bit product-code frame): the first and
    # last boundaries, atanh(-7/h) - atanh(0.5/h) and atanh(7/h) - atanh(0.5/h),
    # hand-evaluated to 5 places; the oracle steps across both.
    th = _closed_form_thresholds(7.5075, 0.5)
    assert abs(th[0] - (-1.74316)) < 6e-6 and abs(th[-1] - 1.60976) < 6e-6
    for t in (th[0], th[-1]):
        lo, hi = O.fsq_quantize(np.array([t - 1e-7, t + 1e-7]), 7.5075, 0.5)
        assert hi == lo + 1


@pytest.mark.parametrize("h", [7.5, 7.5075])
def test_odd_symmetry_about_minus_a(h):
    # u~(u) + delta = h tanh(u + a) is odd about u = -a, so
    # round(u~(-2a - u)) = -1 - round(u~(u)) away from ties.  Pins the
    # atanh(delta/h) shift and the -delta offset.
    a = math.atanh(0.5 / h)
    rng = np.random.default_rng(1)
    u = rng.normal(0, 2, 100000)
    u = u[O.fsq_boundary_distance(u, h) > 1e-9]
    assert np.array_equal(O.fsq_quantize(-2 * a - u, h), -1 - O.fsq_quantize(u, h))


def test_code_distribution_matches_normal_law():
    # u ~ N(0, 4) (the law of E x for E ~ N(0, 4/C), x ~ N(0, 1)):
    # P(level k) = Phi(theta_{k}/2) - Phi(theta_{k-1}/2).
    th = _closed_form_thresholds(7.5, 0.5)
    edges = np.concatenate([[-np.inf], th, [np.inf]])
    p = norm.cdf(edges[1:] / 2) - norm.cdf(edges[:-1] / 2)
    assert abs(p[0] - 0.191) < 2e-3 and abs(p[8] - 0.027) < 2e-3 and abs(p[15] - 0.209) < 2e-3
    lv = np.arange(-8, 8)
    assert abs((p * lv * lv).sum() - 36.4) < 0.1
    rng = np.random.default_rng(7)
    n = 400000
    c = O.fsq_quantize(rng.normal(0, 2, n))
    f = np.bincount(c + 8, minlength=16)
    chi2 = ((f - n * p) ** 2 / (n * p)).sum()
    assert chi2 < 50.0  # 15 dof; p-value ~1e-5 at 50


def test_encode_is_gemm_then_eq2():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(17, 40))
    E = rng.normal(size=(6, 40)) * (4 / 40) ** 0.5
    lv, u = O.encode(x, E)
    # u_t,i = sum_c E_ic x_tc, checked element by element
    for t in (0, 5, 16):
        for i in (0, 3, 5):
            assert abs(u[t, i] - sum(E[i, c] * x[t, c] for c in range(40))) < 1e-12
    assert np.array_equal(lv, O.fsq_quantize(u))


# ---------------------------------------------------------------- packing
def test_pack_unpack_roundtrip_and_layout():
    rng = np.random.default_rng(0)
    for G in (2, 84, 256):
        lv = rng.integers(-8, 8, size=(33, G))
        b = O.pack(lv)
        assert b.dtype == np.uint8 and b.shape == (33, G // 2)
        assert np.array_equal(O.unpack(b, G), lv)
    # coordinate 2i in the low nibble, 2i+1 in the high nibble, nibble = level + 8
    assert O.pack(np.array([[-8, 7]]))[0, 0] == 0xF0
    assert O.pack(np.array([[7, -8]]))[0, 0] == 0x0F
    assert O.pack(np.array([[0, 0]]))[0, 0] == 0x88
    with pytest.raises(ValueError):
        O.pack(np.array([[8, 0]]))


def test_byte_budget_matches_pages(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "paper_constants.json")))
    L, b = g["levels_L"]["value"], g["bits_b"]["value"]
    assert b == math.ceil(math.log2(L)) == O.BITS and L == O.LEVELS
    full = O.full_cache_bytes_per_token(g["qwen3_n_kv"]["value"], g["qwen3_d_h"]["value"])
    assert full == g["c_full_bytes_qwen3"]["value"] == 4096
    assert O.code_bytes_per_token(256) == g["bytes_at_32x"]["value"] == 128
    assert full / O.code_bytes_per_token(256) == g["ratio_32x"]["value"]
    G97 = g["g_at_97_5x"]["value"]
    assert O.code_bytes_per_token(G97) == 42
    assert abs(full / O.code_bytes_per_token(G97) - g["ratio_97_5x"]["value"]) < 0.03
    assert full * g["qwen3_8b_layers"]["value"] == g["qwen3_8b_kib_per_token_all_layers"]["value"] * 1024
    # packed rows really are G/2 bytes
    assert O.pack(np.zeros((1, 256), dtype=np.int64)).nbytes == 128
    assert O.pack(np.zeros((1, 84), dtype=np.int64)).nbytes == 42


# ---------------------------------------------------------------- attention
def _load_case(golden_dir, name):
    cases = json.load(open(os.path.join(golden_dir, "tiny_attention_cases.json")))["cases"]
    c = [c for c in cases if c["name"] == name][0]
    codes = np.array([[int(h, 16) for h in row] for row in c["codes_hex"]], dtype=np.uint8)[None]
    return c, codes


@pytest.mark.parametrize("name", ["mha_G4_dh2_T3", "gqa_G2_dh1_T2"])
def test_hand_worked_cases(golden_dir, name):
    c, codes = _load_case(golden_dir, name)
    assert np.array_equal(O.unpack(codes[0], c["G"]), np.array(c["levels"]))
    o = O.decode_attn(np.array(c["q"], float), codes, np.array(c["W_kv"], float),
                      c["n_kv"], c["G"], scale=math.log(2))
    exp = np.array([[[n / d for n, d in hd] for hd in row] for row in c["o_rational"]])
    assert np.allclose(o, exp, atol=1e-14, rtol=0)
    op = O.decode_attn_pooled(np.array(c["q"], float), codes, np.array(c["W_kv"], float),
                              c["n_kv"], c["G"], scale=math.log(2))
    assert np.allclose(op, exp, atol=1e-14, rtol=0)


def _rand_case(seed, B=2, n_q=8, n_kv=2, d_h=16, G=12, T=37):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, size=(B, T, G // 2), dtype=np.uint8)
    W = rng.normal(size=(2 * n_kv * d_h, G)) / math.sqrt(G)
    q = rng.normal(size=(B, n_q, d_h))
    return q, codes, W, n_kv, G


def test_single_token_returns_its_value():
    q, codes, W, n_kv, G = _rand_case(1, T=1)
    o = O.decode_attn(q, codes, W, n_kv, G)
    d_h = q.shape[-1]
    Wv = W[n_kv * d_h:]
    for b in range(q.shape[0]):
        z = O.unpack(codes[b], G)[0]
        for h in range(q.shape[1]):
            j = h // (q.shape[1] // n_kv)
            v = Wv[j * d_h:(j + 1) * d_h] @ z
            assert np.array_equal(o[b, h], v)


def test_equal_scores_give_mean_value():
    q, codes, W, n_kv, G = _rand_case(2)
    o = O.decode_attn(np.zeros_like(q), codes, W, n_kv, G)
    d_h = q.shape[-1]
    for b in range(q.shape[0]):
        zbar = O.unpack(codes[b], G).mean(axis=0)
        for h in range(q.shape[1]):
            j = h // (q.shape[1] // n_kv)
            assert np.allclose(o[b, h], W[n_kv * d_h + j * d_h: n_kv * d_h + (j + 1) * d_h] @ zbar, atol=1e-12)


def test_token_permutation_invariance():
    q, codes, W, n_kv, G = _rand_case(3)
    perm = np.random.default_rng(0).permutation(codes.shape[1])
    a = O.decode_attn(q, codes, W, n_kv, G)
    b = O.decode_attn(q, codes[:, perm], W, n_kv, G)
    assert np.allclose(a, b, atol=1e-12)


@pytest.mark.parametrize("shape", [(2, 8, 2, 16, 12, 37), (1, 32, 8, 128, 84, 300), (1, 16, 8, 128, 256, 129)])
def test_reduces_to_torch_sdpa(shape):
    B, n_q, n_kv, d_h, G, T = shape
    q, codes, W, n_kv, G = _rand_case(4, B, n_q, n_kv, d_h, G, T)
    o = O.decode_attn(q, codes, W, n_kv, G)
    K = np.stack([O.reconstruct_kv(O.unpack(codes[b], G), W, n_kv, d_h)[0] for b in range(B)])
    V = np.stack([O.reconstruct_kv(O.unpack(codes[b], G), W, n_kv, d_h)[1] for b in range(B)])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[:, :, None, :], torch.from_numpy(K), torch.from_numpy(V),
        enable_gqa=True)[:, :, 0, :].numpy()
    assert np.abs(o - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_ragged_lengths_reduce_to_masked_sdpa():
    """Per-row lengths (a ragged batch) equal torch SDPA with a key mask that
    hides each row's tokens past its length; a row of length 1 returns that
    token's value."""
    B, n_q, n_kv, d_h, G, T = 3, 8, 2, 16, 12, 41
    q, codes, W, n_kv, G = _rand_case(8, B, n_q, n_kv, d_h, G, T)
    lengths = [1, 17, 41]
    o = O.decode_attn(q, codes, W, n_kv, G, lengths=lengths)
    K = np.stack([O.reconstruct_kv(O.unpack(codes[b], G), W, n_kv, d_h)[0] for b in range(B)])
    V = np.stack([O.reconstruct_kv(O.unpack(codes[b], G), W, n_kv, d_h)[1] for b in range(B)])
    keep = torch.arange(T)[None, :] < torch.tensor(lengths)[:, None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[:, :, None, :], torch.from_numpy(K), torch.from_numpy(V),
        attn_mask=keep[:, None, None, :], enable_gqa=True)[:, :, 0, :].numpy()
    assert np.abs(o - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    grp = n_q // n_kv
    for h in range(n_q):
        assert np.allclose(o[0, h], V[0, h // grp, 0], atol=1e-12)
    assert np.array_equal(O.decode_attn(q, codes, W, n_kv, G, lengths=[T] * B), O.decode_attn(q, codes, W, n_kv, G))


def test_value_pooling_identity_eq6():
    for seed in range(3):
        q, codes, W, n_kv, G = _rand_case(10 + seed, B=2, n_q=32, n_kv=8, d_h=128, G=84, T=200)
        a = O.decode_attn(q, codes, W, n_kv, G)
        b = O.decode_attn_pooled(q, codes, W, n_kv, G)
        assert np.abs(a - b).max() <= 1e-12 * np.abs(a).max()


def test_split_merge_equals_one_pass():
    rng = np.random.default_rng(5)
    s = rng.normal(0, 6, 1000)
    V = rng.normal(size=(1000, 5))
    a = O.softmax(s) @ V
    for cuts in ([0, 1000], [0, 1, 1000], [0, 333, 334, 999, 1000], list(range(0, 1001, 7)) + [1000]):
        cuts = sorted(set(cuts))
        parts = [O.partial_attn(s[i:j], V[i:j]) for i, j in zip(cuts[:-1], cuts[1:]) if j > i]
        assert np.allclose(O.lse_merge(parts), a, atol=1e-12)


def test_sampled_rows_match_full():
    q, codes, W, n_kv, G = _rand_case(6, B=3)
    full = O.decode_attn(q, codes, W, n_kv, G)
    part = O.decode_attn(q, codes, W, n_kv, G, rows=[2], heads=[1, 6])
    assert np.array_equal(part[2, [1, 6]], full[2, [1, 6]])
    assert np.isnan(part[0]).all()


# ---------------------------------------------------------------- key norm + RoPE flag
def test_rope_identity_at_zero_and_norm_preserving():
    rng = np.random.default_rng(8)
    k = rng.normal(size=(5, 16))
    assert np.allclose(O.rope(k[:1], [0.0], 10000.0), k[:1], atol=0)
    r = O.rope(k, np.arange(5.0) * 13, 10000.0)
    assert np.allclose(np.linalg.norm(r, axis=1), np.linalg.norm(k, axis=1), atol=1e-12)


def test_rope_scores_depend_on_relative_position():
    rng = np.random.default_rng(9)
    q, k = rng.normal(size=(1, 16)), rng.normal(size=(1, 16))
    s1 = (O.rope(q, [10.0], 1e4) * O.rope(k, [3.0], 1e4)).sum()
    s2 = (O.rope(q, [107.0], 1e4) * O.rope(k, [100.0], 1e4)).sum()
    assert abs(s1 - s2) < 1e-10
    # half-split pairing: the first frequency rotates coordinates 0 and d/2
    e0 = np.zeros((1, 16)); e0[0, 0] = 1.0
    r = O.rope(e0, [math.pi / 2], 1e4)
    assert abs(r[0, 8] - 1.0) < 1e-12 and abs(r[0, 0]) < 1e-12


def test_rms_norm_unit_rms():
    k = np.random.default_rng(2).normal(size=(7, 32)) * 5
    n = O.rms_norm(k, np.ones(32), 0.0)
    assert np.allclose(np.sqrt((n * n).mean(axis=1)), 1.0, atol=1e-12)


def test_rope_flag_breaks_pooled_keys():
    # With RoPE on, keys depend on t, so scoring (W_k^T q) . z_t no longer equals
    # the expanded path (the reason the pages expand keys per position).
    q, codes, W, n_kv, G = _rand_case(11, B=1, n_q=4, n_kv=2, d_h=16, G=12, T=40)
    rk = dict(gain=np.ones(16), eps=1e-6, base=10000.0)
    a = O.decode_attn(q, codes, W, n_kv, G, rope_knorm=rk)
    b = O.decode_attn_pooled(q, codes, W, n_kv, G)
    assert np.abs(a - b).max() > 1e-3
    # and at T=1 (position 0) RoPE is the identity, leaving only the key norm,
    # which cannot change a single-token softmax
    q1, c1, W1, _, _ = _rand_case(12, B=1, n_q=4, n_kv=2, d_h=16, G=12, T=1)
    assert np.allclose(O.decode_attn(q1, c1, W1, 2, 12, rope_knorm=rk), O.decode_attn(q1, c1, W1, 2, 12), atol=1e-12)


# ---------------------------------------------------------------- level-count variants (L = 4, 256)
def _closed_form_thresholds_L(L, h, delta):
    # Hand inversion of eq. (2) at L levels: the level steps from m to m+1 where
    # u~ = m + 1/2, m = -L/2 .. L/2 - 2; a boundary past the tanh range is never reached.
    a = math.atanh(delta / h)
    out = []
    for m in range(-(L // 2), L // 2 - 1):
        arg = (m + 0.5 + delta) / h
        out.append(math.atanh(arg) - a if abs(arg) < 1 else (math.inf if arg > 0 else -math.inf))
    return np.array(out)


@pytest.mark.parametrize("L", [4, 256])
def test_level_variants_zero_saturation_and_grid(L):
    h = O.default_h(L)
    assert h == (L - 1) / 2
    assert O.fsq_quantize(np.array([0.0]), h, 0.5, L)[0] == 0  # h tanh(atanh(delta/h)) - delta = 0
    u = np.linspace(-200, 200, 400001)
    c = O.fsq_quantize(u, h, 0.5, L)
    assert c[0] == -(L // 2) and c[-1] == L // 2 - 1
    assert np.all(np.diff(c) >= 0)
    assert sorted(set(c.tolist())) == list(range(-(L // 2), L // 2))  # exactly L levels are reached


@pytest.mark.parametrize("L", [4, 256])
def test_level_variants_equal_threshold_count(L):
    h = O.default_h(L)
    th = _closed_form_thresholds_L(L, h, 0.5)
    assert len(th) == L - 1 and np.all(np.diff(th) > 0)
    u = np.linspace(-8.0, 8.0, 400_001)
    c = O.fsq_quantize(u, h, 0.5, L)
    n = (u[:, None] >= th[None, :]).sum(axis=1) - L // 2
    d = np.abs(u[:, None] - th[None, :]).min(axis=1)
    far = d > 1e-9
    assert np.array_equal(c[far], n[far])
    assert np.allclose(O.fsq_boundary_distance(u[::991], h, 0.5, L), d[::991], atol=1e-12)


def test_level_variant_thresholds_hand_values():
    # L = 4, h = 1.5, delta = 0.5: boundaries at u~ = -1.5, -0.5, 0.5 solve
    # tanh(u + atanh(1/3)) = -2/3, 0, 2/3.  With atanh(x) = ln((1+x)/(1-x))/2,
    # atanh(1/3) = ln(2)/2 and atanh(2/3) = ln(5)/2, so the three boundaries are
    # -ln(10)/2, -ln(2)/2 and ln(5/2)/2.
    hand = [-math.log(10) / 2, -math.log(2) / 2, math.log(2.5) / 2]
    assert np.allclose(_closed_form_thresholds_L(4, 1.5, 0.5), hand, atol=1e-15)
    assert O.fsq_quantize(np.array([hand[0] - 1e-6, hand[0] + 1e-6]), 1.5, 0.5, 4).tolist() == [-2, -1]


def test_level_variant_packing_layout_and_budgets(golden_dir):
    rng = np.random.default_rng(3)
    for L, G in ((4, 320), (4, 576), (256, 80), (256, 144), (16, 160)):
        lv = rng.integers(-(L // 2), L // 2, size=(9, G))
        b = O.pack(lv, L)
        assert b.shape == (9, G * O.bits_per_coordinate(L) // 8)
        assert np.array_equal(O.unpack(b, G, L), lv)
    # L = 4: byte k holds coordinates 4k .. 4k+3, the first in bits 0-1; code = level + 2
    assert O.pack(np.array([[-2, -1, 0, 1]]), 4)[0, 0] == 0b11100100
    assert O.pack(np.array([[1, 0, 0, 0]]), 4)[0, 0] == 0b00000011 | (0b10 << 2) | (0b10 << 4) | (0b10 << 6)
    # L = 256: one byte per coordinate, code = level + 128
    assert O.pack(np.array([[-128, 127, 0]]), 256).tolist() == [[0, 255, 128]]
    with pytest.raises(ValueError):
        O.pack(np.array([[2, 0, 0, 0]]), 4)
    # Table 8: a fixed budget B bytes/token holds 8B/b coordinates at b bits
    g = json.load(open(os.path.join(golden_dir, "paper_constants.json")))["level_grid_table8"]["value"]
    for L, bits in zip(g["levels"], g["bits"]):
        assert O.bits_per_coordinate(L) == bits
        for budget in g["budgets_bytes_per_token"]:
            G = 8 * budget // bits
            assert O.code_bytes_per_token(G, bits) == budget
    assert [8 * 80 // bb for bb in g["bits"]] == [320, 160, 80]
    assert [8 * 144 // bb for bb in g["bits"]] == [576, 288, 144]


def test_level_variant_attention_matches_sdpa():
    # decode over L = 4 and L = 256 codes reduces to torch SDPA on the expanded K, V
    for L, G in ((4, 32), (256, 12)):
        rng = np.random.default_rng(L)
        B, n_q, n_kv, d_h, T = 2, 8, 2, 16, 37
        lv = rng.integers(-(L // 2), L // 2, size=(B, T, G))
        codes = O.pack(lv, L)
        W = rng.normal(size=(2 * n_kv * d_h, G)) / math.sqrt(G)
        q = rng.normal(size=(B, n_q, d_h))
        o = O.decode_attn(q, codes, W, n_kv, G, levels=L)
        K = np.stack([O.reconstruct_kv(lv[b], W, n_kv, d_h)[0] for b in range(B)])
        V = np.stack([O.reconstruct_kv(lv[b], W, n_kv, d_h)[1] for b in range(B)])
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[:, :, None, :], torch.from_numpy(K), torch.from_numpy(V),
            enable_gqa=True)[:, :, 0, :].numpy()
        assert np.abs(o - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_byte_code_equals_its_nibble_pair():
    """An 8-bit code n (256 levels, level n - 128) read as the nibbles lo = n % 16
    and hi = n // 16 (each a 16-level code, level nibble - 8) has level
    (lo - 8) + 16 (hi - 8) + 8: a 256-level row of G coordinates is a 16-level
    row of 2G nibbles with weights 1 and 16 and a constant offset."""
    n = np.arange(256)
    lv = O.unpack(n[:, None].astype(np.uint8), 1, 256)[:, 0]
    lo = O.unpack(n[:, None].astype(np.uint8), 2, 16)[:, 0]
    hi = O.unpack(n[:, None].astype(np.uint8), 2, 16)[:, 1]
    assert np.array_equal(lv, n - 128)
    assert np.array_equal(lo + 16 * hi + 8, lv)


# ---------------------------------------------------------------- multi-query (causal) attention
def _multi_inputs(B=2, n_new=5, n_q=4, n_kv=2, d_h=8, G=6, T=23, seed=0):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, size=(B, T, G // 2), dtype=np.uint8)
    W = rng.normal(size=(2 * n_kv * d_h, G)) / math.sqrt(G)
    q = rng.normal(size=(B, n_new, n_q, d_h))
    return q, codes, W, n_kv, G


def test_multi_query_single_query_is_decode():
    q, codes, W, n_kv, G = _multi_inputs(n_new=1)
    o = O.decode_attn_multi(q, codes, W, n_kv, G)
    assert np.array_equal(o[:, 0], O.decode_attn(q[:, 0], codes, W, n_kv, G))


def test_multi_query_matches_masked_sdpa():
    """Against torch SDPA in fp64 on the expanded K, V with an explicit causal
    mask: query i of a row of T tokens sees tokens t <= T - n_new + i."""
    q, codes, W, n_kv, G = _multi_inputs()
    B, n_new, n_q, d_h = q.shape
    T = codes.shape[1]
    o = O.decode_attn_multi(q, codes, W, n_kv, G)
    K = np.stack([O.reconstruct_kv(O.unpack(codes[b], G), W, n_kv, d_h)[0] for b in range(B)])
    V = np.stack([O.reconstruct_kv(O.unpack(codes[b], G), W, n_kv, d_h)[1] for b in range(B)])
    mask = torch.tensor([[t <= T - n_new + i for t in range(T)] for i in range(n_new)])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).permute(0, 2, 1, 3), torch.from_numpy(K), torch.from_numpy(V), attn_mask=mask,
        enable_gqa=True).permute(0, 2, 1, 3).numpy()
    assert np.abs(o - ref).max() <= 1e-12 * np.abs(ref).max()


def test_multi_query_is_causal_and_honours_lengths():
    q, codes, W, n_kv, G = _multi_inputs(B=1, n_new=4, T=30)
    lengths = [26]
    o = O.decode_attn_multi(q, codes, W, n_kv, G, lengths=lengths)
    # query i sits at position 26 - 4 + i: tokens after it (and past the row's length) do not matter
    c2 = codes.copy()
    c2[0, 23:] ^= 0x5A  # changes tokens 23.. : seen by queries 1..3 only (positions 23, 24, 25)
    o2 = O.decode_attn_multi(q, c2, W, n_kv, G, lengths=lengths)
    assert np.array_equal(o[0, 0], o2[0, 0])
    assert not np.allclose(o[0, 1:], o2[0, 1:])
    c3 = codes.copy()
    c3[0, 26:] ^= 0x5A  # past the row's length: nothing changes
    assert np.array_equal(O.decode_attn_multi(q, c3, W, n_kv, G, lengths=lengths), o)
    with pytest.raises(ValueError):
        O.decode_attn_multi(q, codes, W, n_kv, G, lengths=[3])
