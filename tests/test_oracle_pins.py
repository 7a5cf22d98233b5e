"""Pins of the fp64 oracle to facts outside itself (closed forms, the pages'
printed numbers, textbook special cases, invariants, hand-worked cases)."""
import math
import os

import numpy as np
import pytest

from oracle import kv_budget as kb
from oracle import mla_oracle as om

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ---------------------------------------------------------------- mscale / scale

def test_mscale_closed_form():
    # ln 64 = 6 ln 2, so 0.1 ln 64 + 1 = 1.41588830833597 (YaRN section 3.4 with s = 64).
    assert om.yarn_get_mscale(64.0, 1.0) == pytest.approx(1.4158883083359671, abs=1e-15)
    assert om.yarn_get_mscale(1.0, 1.0) == 1.0          # no extension, no correction
    assert om.yarn_get_mscale(0.5, 1.0) == 1.0
    assert om.yarn_get_mscale(64.0, 0.0) == 1.0         # mscale 0 switches the log term off


def test_softmax_scale_closed_form():
    cfg = om.YarnConfig()
    # (1 + 0.6 ln 2)^2 / sqrt(192), evaluated with 40-digit decimal arithmetic
    assert om.softmax_scale(cfg) == pytest.approx(0.14467962580268923172, rel=1e-14)
    assert om.cos_sin_factor(cfg) == 1.0                # mscale == mscale_all_dim
    plain = om.YarnConfig(factor=1.0)
    assert om.softmax_scale(plain) == pytest.approx(1.0 / math.sqrt(192.0), rel=1e-15)


# ---------------------------------------------------------------- YaRN table

def test_factor_one_is_textbook_rope():
    for theta in (1e4, 1e7):
        f = om.yarn_inv_freq(om.YarnConfig(rope_theta=theta, factor=1.0))
        # textbook RoPE: a geometric progression starting at 1 with ratio theta^(-2/64)
        assert f[0] == 1.0
        ratios = f[1:] / f[:-1]
        assert np.allclose(ratios, theta ** (-1.0 / 32.0), rtol=1e-13, atol=0)


def _rotations_over_original_context(cfg):
    i = np.arange(cfg.rotary_dim // 2)
    base = 1.0 / np.power(cfg.rope_theta, i / (cfg.rotary_dim / 2.0))
    return base, cfg.original_max_position_embeddings * base / (2.0 * math.pi)


@pytest.mark.parametrize("theta", [1e4, 1e7])
def test_yarn_by_parts_behaviour(theta):
    """YaRN section 3.2: pairs that turn more than beta_fast times over the original
    context keep their frequency; pairs that turn fewer than beta_slow times are
    divided by the scale factor; the band between is blended (strictly between)."""
    cfg = om.YarnConfig(rope_theta=theta)
    f = om.yarn_inv_freq(cfg)
    base, rot = _rotations_over_original_context(cfg)
    keep = rot > cfg.beta_fast
    interp = rot < cfg.beta_slow
    assert keep.any() and interp.any()
    assert np.allclose(f[keep], base[keep], rtol=1e-15, atol=0)
    assert np.allclose(f[interp], base[interp] / cfg.factor, rtol=1e-15, atol=0)
    # rounding the band edges outward may keep/interpolate one extra pair at each edge,
    # but every pair lies within [base/factor, base] and frequencies stay decreasing
    assert np.all(f <= base * (1 + 1e-15)) and np.all(f >= base / cfg.factor * (1 - 1e-15))
    assert np.all(np.diff(f) < 0)


def test_yarn_band_edges_at_theta_1e4():
    # Pair 10 turns 36.7 times (> 32) over 4096 positions and pair 11 27.5 times;
    # pair 22 turns 1.16 times (> 1) and pair 23 0.87 times: the band is pairs 11..22.
    cfg = om.YarnConfig()
    base, rot = _rotations_over_original_context(cfg)
    assert rot[10] > 32 > rot[11] and rot[22] > 1 > rot[23]
    f = om.yarn_inv_freq(cfg)
    assert f[10] == pytest.approx(base[10], rel=1e-15)
    assert f[23] == pytest.approx(base[23] / 64, rel=1e-15)
    assert base[11] / 64 < f[11] < base[11]
    assert base[22] / 64 < f[22] < base[22]


def test_yarn_ramp_interior_values_by_hand():
    """Inside the band the blend is linear in the pair index: at theta = 1e4 the
    band edges are 10 and 23 (above), so pair i takes the fraction
    r = (i - 10) / 13 of the divided frequency and 1 - r of the kept one:
        f_i = base_i * (1 - r * (1 - 1/64)).
    Worked out by hand as exact fractions (base_i = 10^(-i/8)):
      pair 12: r = 2/13,  1 - (2/13)(63/64)  = 706/832 = 353/416
      pair 16: r = 6/13,  1 - (6/13)(63/64)  = 454/832 = 227/416, base 1/100
      pair 20: r = 10/13, 1 - (10/13)(63/64) = 202/832 = 101/416
      pair 22: r = 12/13, 1 - (12/13)(63/64) = 76/832  = 19/208"""
    f = om.yarn_inv_freq(om.YarnConfig())
    assert f[16] == pytest.approx(227.0 / 41600.0, rel=1e-14)          # 0.00545673076923...
    assert f[12] == pytest.approx(10.0 ** -1.5 * 353.0 / 416.0, rel=1e-14)
    assert f[20] == pytest.approx(10.0 ** -2.5 * 101.0 / 416.0, rel=1e-14)
    assert f[22] == pytest.approx(10.0 ** -2.75 * 19.0 / 208.0, rel=1e-14)
    # an off-by-one band (edges 11 and 24) or a ramp that is not linear in i would
    # move pair 16 away from 227/41600
    assert abs(f[16] - 0.01 * (1 - 5 / 13 * 63 / 64)) > 1e-4


def test_cos_sin_factor_with_unequal_mscales():
    """cos/sin carry mscale(s, mscale) / mscale(s, mscale_all_dim); with
    mscale = 0.707 and mscale_all_dim = 1 at s = 64 that is
    (0.1 * 0.707 * ln 64 + 1) / (0.1 * ln 64 + 1) = 1.29403303399... / 1.41588830833...
    = 0.91393723..., and the logit scale keeps mscale_all_dim only."""
    ln64 = 6.0 * math.log(2.0)
    cfg = om.YarnConfig(mscale=0.707, mscale_all_dim=1.0)
    want = (0.1 * 0.707 * ln64 + 1.0) / (0.1 * ln64 + 1.0)
    assert want == pytest.approx(0.9139372, abs=1e-7)
    assert om.cos_sin_factor(cfg) == pytest.approx(want, rel=1e-15)
    # swapped numerator and denominator would give 1/want = 1.0941...
    assert abs(om.cos_sin_factor(cfg) - 1.0 / want) > 0.1
    # the factor scales the rotated vector's length, at every position
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 64))
    y = om.rope(x, np.array([0, 7, 4096, 300000]), cfg)
    assert np.allclose(np.linalg.norm(y, axis=1), want * np.linalg.norm(x, axis=1), rtol=1e-13)
    # position 0: a pure scaling by the factor
    assert np.allclose(y[0], want * x[0], rtol=1e-14, atol=0)
    # the logit scale uses mscale_all_dim alone: unchanged from the default config
    assert om.softmax_scale(cfg) == pytest.approx(0.14467962580268923172, rel=1e-14)
    half = om.YarnConfig(mscale=1.0, mscale_all_dim=0.5)
    assert om.softmax_scale(half) == pytest.approx((0.05 * ln64 + 1.0) ** 2 / math.sqrt(192.0),
                                                   rel=1e-14)
    assert om.cos_sin_factor(half) == pytest.approx((0.1 * ln64 + 1.0) / (0.05 * ln64 + 1.0),
                                                    rel=1e-15)


# ---------------------------------------------------------------- RoPE

def test_rope_matches_complex_rotation():
    """Rotate-half RoPE is multiplication of z_i = x_i + i x_{i+32} by exp(i p f_i)."""
    rng = np.random.default_rng(0)
    cfg = om.YarnConfig()
    x = rng.standard_normal((5, 64))
    pos = np.array([0, 1, 4095, 262143, 524287])
    y = om.rope(x, pos, cfg)
    z = (x[:, :32] + 1j * x[:, 32:]) * np.exp(1j * pos[:, None] * om.yarn_inv_freq(cfg)[None, :])
    assert np.allclose(y[:, :32], z.real, atol=1e-12)
    assert np.allclose(y[:, 32:], z.imag, atol=1e-12)
    assert np.array_equal(om.rope(x[:1], np.array([0]), cfg), x[:1])   # position 0 is identity


def test_rope_preserves_norm_and_is_relative():
    rng = np.random.default_rng(1)
    cfg = om.YarnConfig()
    q = rng.standard_normal(64)
    k = rng.standard_normal(64)
    for m, n in [(5, 3), (4095, 17), (262143, 262000), (524287, 1)]:
        qm = om.rope(q, np.array(m), cfg)
        kn = om.rope(k, np.array(n), cfg)
        assert np.linalg.norm(qm) == pytest.approx(np.linalg.norm(q), rel=1e-13)
        shift = 1000
        d0 = qm @ kn
        d1 = om.rope(q, np.array(m - shift), cfg) @ om.rope(k, np.array(n - shift), cfg)
        assert d0 == pytest.approx(d1, abs=1e-9)


# ---------------------------------------------------------------- attention

def _rand_case(rng, N, q_len, H, scale_w=512 ** -0.5):
    q = rng.standard_normal((q_len, H, 192))
    c = rng.standard_normal((N, 512))
    kp = rng.standard_normal((N, 64))
    wk = rng.standard_normal((H, 128, 512)) * scale_w
    wv = rng.standard_normal((H, 512, 128)) * scale_w
    return q, c, kp, wk, wv


@pytest.mark.parametrize("N,q_len,H", [(1, 1, 2), (7, 1, 2), (64, 1, 32), (129, 4, 4), (300, 3, 32)])
def test_absorbed_equals_expanded(N, q_len, H):
    rng = np.random.default_rng(N * 10 + q_len)
    cfg = om.YarnConfig()
    q, c, kp, wk, wv = _rand_case(rng, N, q_len, H)
    ref = om.mla_attention_expanded(q, c, kp, wk, wv, cfg)
    kp_rot = om.rope(kp, np.arange(N), cfg)
    got = om.mla_attention_absorbed(q, c, kp_rot, wk, wv, cfg)
    assert np.max(np.abs(got - ref)) <= 1e-10 * max(1.0, np.max(np.abs(ref)))


def test_absorbed_equals_expanded_4k_context():
    """The 4K-context decode shape (32 heads, 4096 tokens) in both forms."""
    rng = np.random.default_rng(4096)
    cfg = om.YarnConfig()
    q, c, kp, wk, wv = _rand_case(rng, 4096, 1, 32)
    ref = om.mla_attention_expanded(q, c, kp, wk, wv, cfg)
    got = om.mla_attention_absorbed(q, c, om.rope(kp, np.arange(4096), cfg), wk, wv, cfg)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel <= 1e-10


def test_probabilities_sum_to_one_and_respect_causality():
    rng = np.random.default_rng(2)
    cfg = om.YarnConfig()
    q, c, kp, wk, _ = _rand_case(rng, 40, 4, 3)
    P = om.mla_attention_probs(q, c, kp, wk, cfg)
    assert np.allclose(P.sum(axis=-1), 1.0, atol=1e-13)
    for j in range(4):                       # query j sits at position 36 + j
        assert np.all(P[j, :, 36 + j + 1:] == 0.0)
        assert np.all(P[j, :, :36 + j + 1] > 0.0)


def _zeros(N, H):
    return (np.zeros((1, H, 192)), np.zeros((N, 512)), np.zeros((N, 64)),
            np.zeros((H, 128, 512)), np.zeros((H, 512, 128)))


def test_hand_single_token_returns_its_value():
    # N = 1: softmax over one token is 1, so out[h] = W_UV[h]^T c.
    q, c, kp, wk, wv = _zeros(1, 2)
    q[0, 0, 0] = 3.0
    kp[0, 5] = 1.0
    c[0, 3] = 2.0
    wv[0, 3, 5] = 0.5      # head 0: out[5] = 2.0 * 0.5 = 1.0
    wv[1, 3, 7] = -1.5     # head 1: out[7] = 2.0 * -1.5 = -3.0
    out = om.mla_attention_expanded(q, c, kp, wk, wv, om.YarnConfig())
    want = np.zeros((1, 2, 128))
    want[0, 0, 5] = 1.0
    want[0, 1, 7] = -3.0
    assert np.array_equal(out, want)


def test_hand_designed_scores():
    # One head, two tokens.  W_UK maps latent dim 0 onto nope dim 0 and q_nope[0] = a, so the
    # logits are scale*a*c[t,0] = (ln 3, 0): P = (3/4, 1/4).  V reads latent dim 1 = (4, 8):
    # out = 0.75*4 + 0.25*8 = 5.
    cfg = om.YarnConfig()
    q, c, kp, wk, wv = _zeros(2, 1)
    wk[0, 0, 0] = 1.0
    q[0, 0, 0] = math.log(3.0) / om.softmax_scale(cfg)
    c[0, 0], c[1, 0] = 1.0, 0.0
    c[0, 1], c[1, 1] = 4.0, 8.0
    wv[0, 1, 0] = 1.0
    P = om.mla_attention_probs(q, c, kp, wk, cfg)
    assert np.allclose(P[0, 0], [0.75, 0.25], atol=1e-15)
    out = om.mla_attention_expanded(q, c, kp, wk, wv, cfg)
    assert out[0, 0, 0] == pytest.approx(5.0, abs=1e-14)
    assert np.count_nonzero(out) == 1


def test_hand_rope_term():
    # Plain RoPE (factor 1).  The query (position 1) has q_pe = e_0; token 0 has k_pe = 2 e_32 and
    # token 1 has k_pe = 3 e_0.  Pair 0 turns 1 rad per position, so the rope dot products are
    # (cos 1, sin 1).(0, 2) = 2 sin 1 for token 0 and 3 (cos^2 1 + sin^2 1) = 3 for token 1.
    cfg = om.YarnConfig(factor=1.0)
    s = om.softmax_scale(cfg)
    q, c, kp, wk, wv = _zeros(2, 1)
    q[0, 0, 128] = 1.0
    kp[0, 32] = 2.0
    kp[1, 0] = 3.0
    c[0, 0], c[1, 0] = 1.0, 0.0
    wv[0, 0, 0] = 1.0                       # V_t[0] = c[t, 0] = (1, 0): out = P_0
    z0, z1 = s * 2.0 * math.sin(1.0), s * 3.0
    p0 = math.exp(z0) / (math.exp(z0) + math.exp(z1))
    out = om.mla_attention_expanded(q, c, kp, wk, wv, cfg)
    assert out[0, 0, 0] == pytest.approx(p0, abs=1e-14)


def test_hand_causal_two_queries():
    # q_len = 2 over N = 3 with all logits 0: query 0 (position 1) averages tokens 0, 1 and
    # query 1 (position 2) averages tokens 0, 1, 2.  V_t[0] = c[t, 0] = (3, 6, 30).
    q, c, kp, wk, wv = _zeros(3, 1)
    q = np.zeros((2, 1, 192))
    c[:, 0] = [3.0, 6.0, 30.0]
    wv[0, 0, 0] = 1.0
    out = om.mla_attention_expanded(q, c, kp, wk, wv, om.YarnConfig())
    assert out[0, 0, 0] == pytest.approx(4.5, abs=1e-14)
    assert out[1, 0, 0] == pytest.approx(13.0, abs=1e-14)


def test_constant_latent_returns_constant_value():
    rng = np.random.default_rng(3)
    cfg = om.YarnConfig()
    q, _, kp, wk, wv = _rand_case(rng, 50, 2, 4)
    cvec = rng.standard_normal(512)
    c = np.tile(cvec, (50, 1))
    out = om.mla_attention_expanded(q, c, kp, wk, wv, cfg)
    want = np.einsum("c,hcv->hv", cvec, wv)
    assert np.allclose(out, np.broadcast_to(want, out.shape), atol=1e-12)


def _build_pool(rng, seqlens, perm_seed, pad_value=None):
    cfg = om.YarnConfig()
    nblk = sum((n + 63) // 64 for n in seqlens)
    perm = np.random.default_rng(perm_seed).permutation(nblk)
    mb = max((n + 63) // 64 for n in seqlens)
    bt = np.full((len(seqlens), mb), -1, dtype=np.int64)
    pool = np.full((nblk, 64, 576), np.nan if pad_value is None else pad_value)
    rows = []
    k = 0
    for s, n in enumerate(seqlens):
        nb = (n + 63) // 64
        bt[s, :nb] = perm[k:k + nb]
        k += nb
        c = rng.standard_normal((n, 512))
        kp = om.rope(rng.standard_normal((n, 64)), np.arange(n), cfg)
        rows.append(np.concatenate([c, kp], axis=1))
        for t in range(n):
            pool[bt[s, t // 64], t % 64] = rows[-1][t]
    return pool, bt, rows


def test_page_permutation_and_padding_leave_output_unchanged():
    cfg = om.YarnConfig()
    seqlens = [130, 64, 1]
    rng_a = np.random.default_rng(11)
    rng_b = np.random.default_rng(11)
    pool_a, bt_a, rows_a = _build_pool(rng_a, seqlens, perm_seed=1, pad_value=0.0)
    pool_b, bt_b, rows_b = _build_pool(rng_b, seqlens, perm_seed=2, pad_value=1e30)
    assert not np.array_equal(bt_a, bt_b)
    rng = np.random.default_rng(12)
    q = rng.standard_normal((3, 1, 4, 192))
    wk = rng.standard_normal((4, 128, 512)) * 512 ** -0.5
    wv = rng.standard_normal((4, 512, 128)) * 512 ** -0.5
    out_a = om.mla_decode_from_pool(q, pool_a, bt_a, np.array(seqlens), wk, wv, cfg)
    out_b = om.mla_decode_from_pool(q, pool_b, bt_b, np.array(seqlens), wk, wv, cfg)
    assert np.array_equal(out_a, out_b)
    # and the pooled absorbed form agrees with the per-sequence expanded definition
    for s, n in enumerate(seqlens):
        c = rows_a[s][:, :512]
        ref = om.mla_attention_absorbed(q[s], c, rows_a[s][:, 512:], wk, wv, cfg)
        assert np.array_equal(out_a[s], ref)


def test_oracle_cache_append_roundtrip():
    rng = np.random.default_rng(5)
    seqlens = [70, 3]
    nblk = 3
    bt = np.array([[2, 0], [1, -1]])
    pool = np.zeros((nblk, 64, 576), dtype=np.uint16)
    T = sum(seqlens)
    c = rng.integers(0, 65536, size=(T, 512), dtype=np.uint16)
    k = rng.integers(0, 65536, size=(T, 64), dtype=np.uint16)
    sid = np.array([0] * 70 + [1] * 3)
    pos = np.concatenate([np.arange(70), np.arange(3)])
    om.cache_append(pool, bt, sid, pos, c, k)
    g0 = om.gather_sequence(pool, bt[0], 70)
    g1 = om.gather_sequence(pool, bt[1], 3)
    assert np.array_equal(g0, np.concatenate([c[:70], k[:70]], axis=1))
    assert np.array_equal(g1, np.concatenate([c[70:], k[70:]], axis=1))
    assert np.array_equal(pool[2, 5, :512], c[5])      # token 5 of seq 0 -> block 2 row 5
    assert np.array_equal(pool[0, 69 - 64, 512:], k[69])


# ---------------------------------------------------------------- cache ledger

def test_page1_per_token_scalars():
    want = {r[0]: float(r[1]) for r in _read_table("p1_scalars.txt")}
    per_layer = kb.kv_bytes_per_token(kb.mla_elems_page_estimate(), 1)
    per_token = kb.kv_bytes_per_token(kb.mla_elems_page_estimate(), 40)
    assert per_layer == want["mla_bytes_per_token_layer"]
    assert per_token == want["mla_bytes_per_token_40l"]
    mha = kb.kv_bytes_per_token(kb.mha_elems(), 40)
    assert round(mha / per_token) == want["mha_over_mla_ratio"]
    toks = kb.tokens_fitting(want["kv_budget_gb"] * kb.GB, per_token)
    assert round(toks / 1000) == want["kv_budget_tokens_k"]
    full = kb.as_units(kb.cache_bytes(262144, per_token), kb.GiB, 1)
    assert kb.round_half_up(full / 2, 1) == want["q8_cache_256k_gb"]


def test_page1_ledger_table():
    mla = kb.kv_bytes_per_token(kb.mla_elems_page_estimate(), 40)
    mha = kb.kv_bytes_per_token(kb.mha_elems(), 40)
    for label, mla_gb, mha_gb in _read_table("p1_kv_ledger.txt"):
        k = int(label[:-1])
        got_mla = kb.as_units(kb.cache_bytes(k * 1024, mla), kb.GiB, 1)
        assert got_mla == float(mla_gb), label
        mha_tokens = k * 1000 if k <= 128 else k * 1024
        digits = 1 if "." in mha_gb else 0
        got_mha = kb.as_units(kb.cache_bytes(mha_tokens, mha), kb.GiB, digits)
        assert got_mha == float(mha_gb), label


def test_other_pages_ledgers():
    p2 = kb.kv_bytes_per_token(kb.gqa_elems(4, 256), 16)
    p3 = kb.kv_bytes_per_token(kb.gqa_elems(4, 256), 18)
    assert p2 == 64 * 1024 and p3 == 72 * 1024
    for page, tokens, printed in _read_table("p2_p3_kv_ledgers.txt"):
        n = int(tokens)
        if page == "P2":
            assert kb.as_units(n * p2, kb.GiB, 1) == float(printed)
        else:
            gb = n * p3 / kb.GB
            digits = 1 if "." in printed else 0
            assert math.floor(gb * 10 ** digits) / 10 ** digits == float(printed)


def test_repository_cache_row_is_576_elements():
    # [c_kv 512 | k_pe 64] bf16 = 1152 B per token and layer; 45 KiB over 40 layers.
    per_token = kb.kv_bytes_per_token(kb.mla_elems_latent_rope(), 40)
    assert kb.kv_bytes_per_token(kb.mla_elems_latent_rope(), 1) == 1152
    assert per_token == 45 * 1024
    assert kb.cache_bytes(262144, per_token) / kb.GiB == 11.25


# ------------------------------------------------------------------ kv_a_proj_with_mqa

def test_kv_projection_selection_weights_copy_hidden_dims():
    """A weight whose rows are unit vectors selects hidden dims: the first 512
    selected dims land in c_kv and the last 64 in the rope key, in row order."""
    rng = np.random.default_rng(31)
    hidden = rng.standard_normal((5, om.HIDDEN))
    pick = rng.permutation(om.HIDDEN)[:576]
    W = np.zeros((576, om.HIDDEN))
    W[np.arange(576), pick] = 1.0
    c, k = om.kv_a_projection(hidden, W)
    assert np.array_equal(c, hidden[:, pick[:512]])
    assert np.array_equal(k, hidden[:, pick[512:]])


def test_kv_projection_zero_weight_gives_the_bias():
    rng = np.random.default_rng(32)
    bias = rng.standard_normal(576)
    c, k = om.kv_a_projection(rng.standard_normal((3, om.HIDDEN)), np.zeros((576, om.HIDDEN)), bias)
    assert np.array_equal(c, np.broadcast_to(bias[:512], (3, 512)))
    assert np.array_equal(k, np.broadcast_to(bias[512:], (3, 64)))


def test_kv_projection_differences_of_hidden_pairs():
    """Row j = e_{2j} - e_{2j+1}: output j is hidden[2j] - hidden[2j+1]."""
    rng = np.random.default_rng(33)
    hidden = rng.integers(-1000, 1000, (4, om.HIDDEN)).astype(np.float64)
    W = np.zeros((576, om.HIDDEN))
    j = np.arange(576)
    W[j, 2 * j] = 1.0
    W[j, 2 * j + 1] = -1.0
    c, k = om.kv_a_projection(hidden, W)
    want = hidden[:, 0:1152:2] - hidden[:, 1:1152:2]
    assert np.array_equal(np.concatenate([c, k], axis=1), want)


def test_kv_projection_is_linear_in_the_hidden_state():
    rng = np.random.default_rng(34)
    W = rng.standard_normal((576, om.HIDDEN)) / 60.0
    h1, h2 = rng.standard_normal((2, 3, om.HIDDEN))
    c1, k1 = om.kv_a_projection(h1, W)
    c2, k2 = om.kv_a_projection(h2, W)
    c3, k3 = om.kv_a_projection(2.5 * h1 - h2, W)
    assert np.allclose(c3, 2.5 * c1 - c2, rtol=0, atol=1e-10)
    assert np.allclose(k3, 2.5 * k1 - k2, rtol=0, atol=1e-10)


# ---------------------------------------------------------------- partials of a split sequence

def _partial_case(seed=5, N=150, q_len=3):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((q_len, om.N_HEADS, om.D_NOPE + om.D_ROPE))
    c = rng.standard_normal((N, om.D_LATENT))
    k = rng.standard_normal((N, om.D_ROPE))
    W_UK = rng.standard_normal((om.N_HEADS, om.D_NOPE, om.D_LATENT)) / math.sqrt(om.D_LATENT)
    W_UV = rng.standard_normal((om.N_HEADS, om.D_LATENT, om.D_V)) / math.sqrt(om.D_LATENT)
    return q, c, k, W_UK, W_UV


def test_partial_of_one_token_is_that_token():
    # one visible token: l = exp(0) = 1 and O is its latent row; the difference of
    # two tokens' m is their log-probability ratio under the expanded definition
    q, c, k, W_UK, _ = _partial_case(q_len=1)
    cfg = om.YarnConfig()
    N = c.shape[0]
    k_rot = om.rope(k, np.arange(N), cfg)
    t = 41
    m, l, O = om.attention_partial(q, c[t:t + 1], k_rot[t:t + 1], W_UK, cfg, N, t, t + 1)
    assert np.all(l == 1.0)
    assert np.array_equal(O, np.broadcast_to(c[t], O.shape))
    m_u, _, _ = om.attention_partial(q, c[t + 1:t + 2], k_rot[t + 1:t + 2], W_UK, cfg, N,
                                     t + 1, t + 2)
    P = om.mla_attention_probs(q, c, k, W_UK, cfg)
    assert np.abs(np.log(P[0, :, t] / P[0, :, t + 1]) - (m[0] - m_u[0])).max() < 1e-9


def test_empty_and_fully_masked_partials_see_nothing():
    q, c, k, W_UK, _ = _partial_case()
    cfg = om.YarnConfig()
    N = c.shape[0]
    for lo, hi in [(10, 10), (N, N)]:
        m, l, O = om.attention_partial(q, c[lo:hi], k[lo:hi], W_UK, cfg, N, lo, hi)
        assert np.all(m == -np.inf) and np.all(l == 0) and np.all(O == 0)
    # the last token is visible only to the last query (q_len = 3)
    m, l, O = om.attention_partial(q, c[N - 1:], k[N - 1:], W_UK, cfg, N, N - 1, N)
    assert np.all(l[:-1] == 0) and np.all(m[:-1] == -np.inf) and np.all(O[:-1] == 0)
    assert np.all(l[-1] == 1)


@pytest.mark.parametrize("cuts", [[70], [1, 2, 149], [64, 128], [30, 60, 90, 120]])
def test_merged_partials_equal_the_expanded_definition(cuts):
    # the partials of any partition of the tokens merge to the attention of the
    # expanded (non-absorbed) definition, in either order of the parts
    q, c, k, W_UK, W_UV = _partial_case()
    cfg = om.YarnConfig()
    N = c.shape[0]
    k_rot = om.rope(k, np.arange(N), cfg)
    edges = [0] + cuts + [N]
    parts = [om.attention_partial(q, c[a:b], k_rot[a:b], W_UK, cfg, N, a, b)
             for a, b in zip(edges[:-1], edges[1:])]
    want = om.mla_attention_expanded(q, c, k, W_UK, W_UV, cfg)
    for order in (parts, parts[::-1]):
        got = om.finish_partial(*om.merge_partials(order), W_UV)
        assert np.abs(got - want).max() < 1e-12


def test_merge_is_associative_and_has_the_empty_part_as_identity():
    q, c, k, W_UK, _ = _partial_case(seed=9)
    cfg = om.YarnConfig()
    N = c.shape[0]
    a = om.attention_partial(q, c[:50], k[:50], W_UK, cfg, N, 0, 50)
    b = om.attention_partial(q, c[50:90], k[50:90], W_UK, cfg, N, 50, 90)
    d = om.attention_partial(q, c[90:], k[90:], W_UK, cfg, N, 90, N)
    e = om.attention_partial(q, c[:0], k[:0], W_UK, cfg, N, 0, 0)
    flat = om.merge_partials([a, b, d])
    for x in (om.merge_partials([om.merge_partials([a, b]), d]),
              om.merge_partials([a, om.merge_partials([b, d])])):
        assert np.array_equal(x[0], flat[0])                 # the maximum is exact
        assert np.allclose(x[1], flat[1], rtol=1e-14, atol=0)
        assert np.allclose(x[2], flat[2], rtol=1e-13, atol=1e-13)
    with_e = om.merge_partials([a, e])
    assert np.array_equal(with_e[0], a[0]) and np.array_equal(with_e[1], a[1])
    assert np.array_equal(with_e[2], a[2])


# ---------------------------------------------------------------- 8-bit latent cache

def _brute_exponent(amax: float) -> int:
    # smallest e in range with 127 * 2^e >= amax, by search in exact rationals
    from fractions import Fraction
    a = Fraction(amax)
    for e in range(om.Q8_EMIN, om.Q8_EMAX + 1):
        if 127 * Fraction(2) ** e >= a:
            return e
    return om.Q8_EMAX


def test_q8_exponent_matches_a_brute_force_search():
    rng = np.random.default_rng(11)
    amax = np.concatenate([
        np.abs(rng.standard_normal(400)) * np.exp2(rng.integers(-20, 12, 400)),
        # the boundaries: exactly 127 * 2^e, one ulp either side, powers of two
        [127.0 * 2.0 ** e for e in range(-14, 9)],
        [np.nextafter(127.0 * 2.0 ** e, np.inf) for e in range(-14, 9)],
        [np.nextafter(127.0 * 2.0 ** e, 0.0) for e in range(-14, 9)],
        [2.0 ** k for k in range(-20, 16)], [0.0, 1e-30, 1e6]])
    got = om.q8_block_exponent(amax)
    want = np.array([_brute_exponent(float(a)) for a in amax])
    assert np.array_equal(got, want)


def test_q8_round_trip_is_exact_on_representable_rows():
    # a block of integers times 2^e whose largest magnitude lies in (63.5, 127]
    # keeps exactly that exponent and comes back unchanged
    rng = np.random.default_rng(12)
    codes = rng.integers(-127, 128, (5, 576))
    codes[:, ::32] = 127 * np.where(rng.random((5, 18)) < 0.5, 1, -1)
    e = rng.integers(om.Q8_EMIN, om.Q8_EMAX + 1, (5, 18))
    x = (codes.reshape(5, 18, 32) * np.exp2(e)[..., None]).reshape(5, 576)
    c, ex = om.q8_quantize(x)
    assert np.array_equal(ex, e) and np.array_equal(c, codes)
    assert np.array_equal(om.q8_dequantize(c, ex), x)


def test_q8_error_is_at_most_half_a_step():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((64, 576)) * np.exp2(rng.integers(-6, 6, (64, 1)))
    c, e = om.q8_quantize(x)
    d = om.q8_dequantize(c, e)
    step = np.repeat(np.exp2(e.astype(np.float64)), 32, axis=-1)
    assert np.all(np.abs(d - x) <= 0.5 * step)
    assert np.all(np.abs(c) <= 127)
    # the exponent is the smallest that fits: one less would need a code > 127
    amax = np.abs(x.reshape(64, 18, 32)).max(-1)
    assert np.all(amax > 127 * np.exp2(e.astype(np.float64) - 1))


def test_q8_ties_round_to_even_and_special_blocks():
    x = np.zeros((1, 576))
    x[0, 0] = 127.0          # block 0: e = 0
    x[0, 1:5] = [2.5, 3.5, -2.5, -0.5]
    x[0, 32] = 1e-9          # block 1: tiny, clamped to the smallest exponent
    x[0, 64] = 1e9           # block 2: beyond the range, saturates
    x[0, 65] = -1e9
    c, e = om.q8_quantize(x)
    assert e[0, 0] == 0 and list(c[0, 1:5]) == [2, 4, -2, 0]
    assert e[0, 1] == om.Q8_EMIN and c[0, 32] == 0
    assert e[0, 2] == om.Q8_EMAX and c[0, 64] == 127 and c[0, 65] == -127
    assert e[0, 3] == om.Q8_EMIN and not c[0, 96:128].any()   # an all-zero block


def test_q8_row_halves_the_cache_as_the_page_says():
    # [P1] section 三, 方案 A: the q8_0 cache halves the bf16 one (12.5 GB -> ~6.3 GB).
    # 576 one-byte codes + 18 exponent bytes against 576 bf16 values:
    assert (576 + om.Q8_BLOCKS) / (576 * 2) == pytest.approx(6.3 / 12.5, rel=0.05)


def test_chunk_of_queries_equals_one_query_at_a_time():
    # a prompt chunk: query j at position N - q_len + j sees tokens 0..that position,
    # which is the one-query call over the first position + 1 tokens (both forms)
    rng = np.random.default_rng(21)
    cfg = om.YarnConfig()
    N, q_len, H = 40, 24, 2
    q = rng.standard_normal((q_len, H, om.D_NOPE + om.D_ROPE))
    c = rng.standard_normal((N, om.D_LATENT))
    kp = rng.standard_normal((N, om.D_ROPE))
    wk = rng.standard_normal((H, om.D_NOPE, om.D_LATENT)) / 512 ** 0.5
    wv = rng.standard_normal((H, om.D_LATENT, om.D_V)) / 512 ** 0.5
    kr = om.rope(kp, np.arange(N), cfg)
    full = om.mla_attention_absorbed(q, c, kr, wk, wv, cfg)
    full_x = om.mla_attention_expanded(q, c, kp, wk, wv, cfg)
    for j in range(q_len):
        t = N - q_len + j + 1
        one = om.mla_attention_absorbed(q[j:j + 1], c[:t], kr[:t], wk, wv, cfg)[0]
        np.testing.assert_allclose(full[j], one, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(full_x[j], one, rtol=1e-9, atol=1e-11)


def test_attention_over_dequantised_rows_is_the_attention_of_those_values():
    # the 8-bit path's reference is the plain attention over code * 2^e; rows that
    # are exactly representable quantise to themselves, so both give the same output
    rng = np.random.default_rng(22)
    cfg = om.YarnConfig()
    N, H = 70, 2
    codes = rng.integers(-127, 128, (N, 576))
    codes[:, ::32] = 127
    e = rng.integers(-8, -4, (N, 18))
    rows = (codes.reshape(N, 18, 32) * np.exp2(e)[..., None]).reshape(N, 576)
    c8, e8 = om.q8_quantize(rows)
    deq = om.q8_dequantize(c8, e8)
    assert np.array_equal(deq, rows)
    q = rng.standard_normal((1, H, 192))
    wk = rng.standard_normal((H, 128, 512)) / 512 ** 0.5
    wv = rng.standard_normal((H, 512, 128)) / 512 ** 0.5
    a = om.mla_attention_absorbed(q, deq[:, :512], deq[:, 512:], wk, wv, cfg)
    b = om.mla_attention_absorbed(q, rows[:, :512], rows[:, 512:], wk, wv, cfg)
    assert np.array_equal(a, b)
