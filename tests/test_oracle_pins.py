"""Pins of the CPU oracle against facts fixed by the mathematics and the
storage format, not by the oracle's own code.

Each test is chosen so that a plausible slip in the oracle (a dropped term,
a wrong sign, a swapped index, a transposed operand, a wrong scale) fails at
least one of them.  No GPU is needed.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
from persistent_decode_megakernel_02_b200 import workloads as wl

RNG = np.random.default_rng(2024)


def bf16_bits(a) -> np.ndarray:
    t = torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def widen(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ---- bf16 storage format ---------------------------------------------------

def test_bf16_known_encodings():
    # bf16 = top 16 bits of binary32: sign, 8 exponent bits, 7 fraction bits
    assert orc.bf16_to_double(0x3F80) == 1.0
    assert orc.bf16_to_double(0xC000) == -2.0
    assert orc.bf16_to_double(0x4049) == 3.140625
    assert orc.bf16_to_double(0x0001) == 2.0 ** -133          # smallest subnormal
    assert orc.bf16_to_double(0x7F7F) == (2 - 2 ** -7) * 2.0 ** 127
    assert orc.double_to_bf16(1.0) == 0x3F80
    assert orc.double_to_bf16(-2.0) == 0xC000


def test_bf16_round_to_nearest_even():
    # 1 + 2^-8 is halfway between 1 (even mantissa) and 1 + 2^-7: ties to even
    assert orc.double_to_bf16(1 + 2 ** -8) == 0x3F80
    # 1 + 3*2^-8 is halfway between 1+2^-7 (odd) and 1+2^-6 (even)
    assert orc.double_to_bf16(1 + 3 * 2 ** -8) == 0x3F82
    # just above a tie rounds up (a value float32 could not hold)
    assert orc.double_to_bf16(1 + 2 ** -8 + 2 ** -40) == 0x3F81
    assert orc.double_to_bf16(-(1 + 2 ** -8 + 2 ** -40)) == 0xBF81
    # overflow past the largest finite value + half an ulp goes to inf
    assert orc.double_to_bf16(2.0 ** 128) == 0x7F80
    assert orc.double_to_bf16(float("nan")) == 0x7FC0
    assert orc.double_to_bf16(2.0 ** -134 * 3) == 0x0002      # subnormal rounding


def test_bf16_matches_library_on_float32_values():
    # for values float32 holds exactly, direct rounding equals torch's fp32->bf16 (RNE)
    x = RNG.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** RNG.integers(-30, 30, 20000).astype(np.float32)
    x = x[np.isfinite(x)]
    ref = bf16_bits(x)
    got = np.array([orc.double_to_bf16(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(got, ref)
    assert np.array_equal(widen(ref), np.array([orc.bf16_to_double(int(b)) for b in ref]))


# ---- RMSNorm -----------------------------------------------------------------

def test_rmsnorm_unit_rms_and_eps_closed_form():
    n = 257
    x = RNG.standard_normal(n) * 3.0
    ones = bf16_bits(np.ones(n))
    y0 = orc.rmsnorm(x, ones, 0.0)
    assert abs(np.sqrt(np.mean(y0 ** 2)) - 1.0) < 1e-12          # output RMS is 1
    ms = np.mean(x ** 2)
    eps = 0.37
    y = orc.rmsnorm(x, ones, eps)
    assert abs(np.mean(y ** 2) - ms / (ms + eps)) < 1e-12        # eps inside the root
    # direction preserved, scale invariant
    assert np.allclose(y0 / x, (y0 / x)[0], rtol=1e-13)
    assert np.allclose(orc.rmsnorm(5.5 * x, ones, 0.0), y0, rtol=1e-13)


def test_rmsnorm_gain_is_elementwise():
    n = 64
    x = RNG.standard_normal(n)
    g = bf16_bits(RNG.uniform(0.5, 2.0, n))
    y1 = orc.rmsnorm(x, bf16_bits(np.ones(n)), 1e-5)
    yg = orc.rmsnorm(x, g, 1e-5)
    assert np.allclose(yg, y1 * widen(g), rtol=1e-14, atol=0)


# ---- GEMV ----------------------------------------------------------------------

def test_gemv_matches_library_matmul_nonsquare():
    W = bf16_bits(RNG.standard_normal((37, 53)))
    x = RNG.standard_normal(53)
    y = orc.gemv(W, x)
    ref = widen(W).reshape(37, 53) @ x
    assert y.shape == (37,)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


# ---- RoPE --------------------------------------------------------------------

@pytest.mark.parametrize("d", [8, 64, 128])
def test_rope_identity_at_zero_and_pair_norms(d):
    v = RNG.standard_normal(d)
    assert np.array_equal(orc.rope(v, 0, 1e4), v)
    r = orc.rope(v, 1234, 5e5)
    h = d // 2
    assert np.allclose(v[:h] ** 2 + v[h:] ** 2, r[:h] ** 2 + r[h:] ** 2, rtol=1e-12)


def test_rope_is_a_rotation_group_in_position():
    d = 64
    v = RNG.standard_normal(d)
    assert np.allclose(orc.rope(orc.rope(v, 17, 1e4), 25, 1e4), orc.rope(v, 42, 1e4), atol=1e-12)


def test_rope_dot_product_depends_only_on_offset():
    d = 64
    q, k = RNG.standard_normal(d), RNG.standard_normal(d)
    a = orc.rope(q, 30, 1e4) @ orc.rope(k, 11, 1e4)
    b = orc.rope(q, 130, 1e4) @ orc.rope(k, 111, 1e4)
    c = orc.rope(q, 31, 1e4) @ orc.rope(k, 11, 1e4)
    assert abs(a - b) < 1e-10
    assert abs(a - c) > 1e-6


def test_rope_pairing_direction_and_frequencies():
    d, theta = 16, 1e4
    h = d // 2
    angles = []
    for i in range(h):
        e = np.zeros(d)
        e[i] = 1.0
        r = orc.rope(e, 1, theta)
        # the unit vector stays in the plane of (i, i + d/2): half-split pairing
        others = np.delete(r, [i, i + h])
        assert np.all(others == 0)
        # it turns from the first-half axis towards the second-half axis
        assert r[i + h] > 0
        angles.append(math.atan2(r[i + h], r[i]))
        # the second-half unit vector turns towards minus the first-half axis
        e2 = np.zeros(d)
        e2[i + h] = 1.0
        r2 = orc.rope(e2, 1, theta)
        assert abs(r2[i] + r[i + h]) < 1e-15 and abs(r2[i + h] - r[i]) < 1e-15
    angles = np.array(angles)
    # pair 0 turns by exactly the position (1 rad); frequencies form a
    # geometric progression with ratio theta^(-2/d)
    assert abs(angles[0] - 1.0) < 1e-15
    assert np.allclose(angles[1:] / angles[:-1], theta ** (-2.0 / d), rtol=1e-12)


# ---- SiLU / argmax -------------------------------------------------------------

def test_silu_identities():
    assert orc.silu(0.0) == 0.0
    assert abs(orc.silu(1.0) - 0.7310585786300049) < 1e-15      # sigmoid(1)
    for x in RNG.standard_normal(50) * 4:
        assert abs(orc.silu(x) - orc.silu(-x) - x) < 1e-13         # x*s(x) + x*s(-x) = x
    assert abs(orc.silu(40.0) - 40.0) < 1e-12


def test_argmax_bruteforce_and_ties():
    for _ in range(20):
        v = RNG.integers(-3, 4, 37).astype(np.float64)
        assert orc.argmax(v) == int(np.flatnonzero(v == v.max())[0])
    assert orc.argmax(np.array([1.0, 5.0, 5.0, 2.0])) == 1


# ---- attention -----------------------------------------------------------------

def _cache(nkv, S, d, fill=None):
    if fill is None:
        return bf16_bits(RNG.standard_normal((nkv, S, d)))
    return bf16_bits(np.broadcast_to(fill, (nkv, S, d)))


def test_attention_single_position_returns_v():
    nq, nkv, S, d = 8, 2, 16, 32
    q = RNG.standard_normal((nq, d))
    kc, vc = _cache(nkv, S, d), _cache(nkv, S, d)
    o = orc.attention(q, kc, vc, 1)
    for i in range(nq):
        assert np.allclose(o[i], widen(vc[i // 4, 0]), rtol=0, atol=1e-15)


def test_attention_weights_sum_to_one_and_positive():
    nq, nkv, d, C_ = 4, 4, 32, 20
    S = 32
    q = RNG.standard_normal((nq, d)) * 2
    kc = _cache(nkv, S, d)
    vc = np.zeros((nkv, S, d), np.uint16)
    for j in range(C_):                       # V_j = e_j: the output is the weights
        vc[:, j, j] = 0x3F80
    o = orc.attention(q, kc, vc, C_)
    assert np.allclose(o.sum(axis=1), 1.0, atol=1e-14)
    assert np.all(o[:, :C_] > 0) and np.all(o[:, C_:] == 0)
    # weights are ordered like the scores q.k_j
    for i in range(nq):
        s = widen(kc[i, :C_]) @ q[i]
        assert np.array_equal(np.argsort(o[i, :C_], kind="stable"), np.argsort(s, kind="stable"))


@pytest.mark.parametrize("d", [64, 128])   # the head dims of the 1B and 8B shapes
def test_attention_two_positions_sigmoid_closed_form(d):
    S = 8
    c, t = 1.5, 2.0
    q = np.zeros((1, d)); q[0, 0] = c
    kc = np.zeros((1, S, d), np.uint16)
    kc[0, 1, 0] = orc.double_to_bf16(t)       # s_0 = 0, s_1 = c*t/sqrt(d)
    vc = np.zeros((1, S, d), np.uint16)
    vc[0, 1, 0] = 0x3F80                      # V_1 = e_0
    o = orc.attention(q, kc, vc, 2)
    expect = 1.0 / (1.0 + math.exp(-c * t / math.sqrt(d)))
    assert abs(o[0, 0] - expect) < 1e-15


def test_attention_gqa_head_grouping_and_ignores_future():
    nq, nkv, S, d, C_ = 8, 2, 16, 16, 5
    q = RNG.standard_normal((nq, d))
    kc = _cache(nkv, S, d)
    vc = np.zeros((nkv, S, d), np.uint16)
    for h in range(nkv):
        vc[h, :C_] = orc.double_to_bf16(h + 1.0)
        vc[h, C_:] = orc.double_to_bf16(-100.0)   # beyond C: must be ignored
    o = orc.attention(q, kc, vc, C_)
    for i in range(nq):
        assert np.allclose(o[i], i // (nq // nkv) + 1.0, atol=1e-14)


def test_attention_constant_v_and_mha():
    nq = nkv = 3
    S, d, C_ = 10, 8, 7
    q = RNG.standard_normal((nq, d))
    kc = _cache(nkv, S, d)
    u = bf16_bits(RNG.standard_normal(d))
    vc = np.broadcast_to(u, (nkv, S, d)).copy()
    o = orc.attention(q, kc, vc, C_)
    assert np.allclose(o, widen(u)[None, :], atol=1e-14)


# ---- whole step ------------------------------------------------------------------

def _tiny_model(gains="random", tied=False, layers=2, seed=5):
    shape = wl.ModelShape("t", layers, 64, 4, 2, 16, 96, 200, tied, 1e4)
    w = wl.make_weights(shape, seed=seed, device="cpu", gains=gains, tied=tied, std=0.2)
    cfg = dict(layers=shape.layers, hidden=shape.hidden, n_q_heads=shape.n_q_heads,
               n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim, ffn=shape.ffn,
               vocab=shape.vocab, max_seq=24, rope_theta=shape.rope_theta,
               rms_eps=shape.rms_eps)
    return orc.OracleModel(cfg, w.numpy_bits()), shape


def test_cached_step_equals_full_recompute():
    model, shape = _tiny_model()
    tokens = wl.make_prompt(shape.vocab, 9, seed=3)
    kc, vc = model.new_cache()
    for p, t in enumerate(tokens):
        out = model.decode_step(kc, vc, int(t), p)
    ref = model.forward_recompute(tokens)
    assert out["next"] == ref["next"]
    scale = np.abs(ref["logits"]).max()
    assert np.max(np.abs(out["logits"] - ref["logits"])) <= 1e-10 * scale
    assert np.allclose(out["hidden"], ref["hidden"], rtol=1e-10, atol=1e-12)


def test_step_ignores_cache_beyond_position():
    model, shape = _tiny_model()
    kc, vc = model.new_cache()
    kc2, vc2 = model.new_cache()
    for l in range(shape.layers):
        kc2[l][:, 5:] = 0x4120     # garbage at positions 5.. (overwritten at 4? no: pos 4 only)
        vc2[l][:, 5:] = 0xC120
    for p, t in enumerate([3, 1, 4, 1, 5]):
        a = model.decode_step(kc, vc, t, p)
        b = model.decode_step(kc2, vc2, t, p)
    assert np.array_equal(a["logits"], b["logits"])


def test_step_without_attention_and_mlp_reduces_to_embedding_head():
    # with W_o = 0 and W_d = 0 the residual stream stays the embedding row,
    # so logits = W_lm @ rmsnorm(E[t]) * g_f (a library matmul)
    model, shape = _tiny_model(tied=True)
    w = model.weights
    for l in range(shape.layers):
        w["wo"][l] = np.zeros_like(w["wo"][l])
        w["wd"][l] = np.zeros_like(w["wd"][l])
    model = orc.OracleModel(model.cfg, w)
    kc, vc = model.new_cache()
    tok = 17
    out = model.decode_step(kc, vc, tok, 0)
    e = widen(w["embed"][tok])
    assert np.array_equal(out["hidden"], e)
    xn = e / np.sqrt(np.mean(e ** 2) + shape.rms_eps) * widen(w["final_norm"])
    ref = widen(w["lm_head"]).reshape(shape.vocab, shape.hidden) @ xn
    assert np.allclose(out["logits"], ref, rtol=1e-12, atol=1e-12)
    assert out["next"] == int(np.argmax(ref))


def test_step_writes_rounded_kv_at_position_only():
    model, shape = _tiny_model()
    kc, vc = model.new_cache()
    model.decode_step(kc, vc, 7, 0)
    before = [a.copy() for a in kc]
    model.decode_step(kc, vc, 9, 1)
    for l in range(shape.layers):
        diff = np.argwhere(before[l] != kc[l])
        assert set(diff[:, 1].tolist()) <= {1}
        assert np.any(kc[l][:, 1] != 0)
