"""Pins of the CPU oracle to facts outside itself (CPU only).

Each test fixes one part of the oracle against a closed form, an invariant, a
special case that reduces to a library routine (numpy matmul, numpy complex
exponentials, scipy's logistic function), the formats' bit-level definitions,
or brute force -- never against a retyped copy of the oracle's own loop.
The cases are chosen so that a plausible mistake (a dropped term, a wrong
sign, a transposed matrix, an off-by-one position, a wrong head mapping)
fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (torch's round-to-nearest-even), as uint16 bits."""
    return synth.to_u16(torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16))


def widen(u16: np.ndarray) -> np.ndarray:
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ------------------------------------------------------------------ formats
def test_bit_patterns_golden():
    n = 0
    for line in open(os.path.join(GOLD, "bit_patterns.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        fmt, hx, val = line.split()
        want = float(eval(val, {"inf": math.inf}))  # noqa: S307 - fixture literal
        got = oracle.bf16_to_f32(int(hx, 16)) if fmt == "bf16" else oracle.f16_to_f32(int(hx, 16))
        assert got == want and math.copysign(1, got) == math.copysign(1, want), (fmt, hx, got, want)
        n += 1
    assert n >= 20


# ------------------------------------------------------------------ GEMV
def test_gemv_identity_and_one_hot():
    K = 40
    x = np.random.default_rng(0).standard_normal(K).astype(np.float32)
    eye = bf16_bits(np.eye(K))
    np.testing.assert_array_equal(oracle.gemv_bf16(eye, x), x)
    sel = np.zeros((3, K), np.float32)
    sel[0, 7] = 1.0
    sel[1, 39] = 2.0
    sel[2, 0] = -0.5
    np.testing.assert_array_equal(oracle.gemv_bf16(bf16_bits(sel), x), [x[7], 2 * x[39], -0.5 * x[0]])


def test_gemv_vs_numpy_nonsquare():
    rng = np.random.default_rng(1)
    N, K = 37, 53  # non-square: a transposed operand cannot pass
    W = bf16_bits(rng.standard_normal((N, K)) * 0.1)
    x = rng.standard_normal(K).astype(np.float32)
    want = widen(W) @ x.astype(np.float64)
    got = oracle.gemv_bf16(W, x)
    bound = 2 ** -23 * np.abs(widen(W)) @ np.abs(x.astype(np.float64)) + 1e-30
    assert np.all(np.abs(got - want) <= bound)


# ------------------------------------------------------------------ RMSNorm
def test_rmsnorm_unit_rms_closed_form():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(2048) * 3).astype(np.float32)
    ones = bf16_bits(np.ones(2048))
    eps = 1e-5
    out = oracle.rmsnorm(x, ones, eps).astype(np.float64)
    ms = np.mean(x.astype(np.float64) ** 2)
    # eps sits inside the square root: rms(out) = sqrt(ms / (ms + eps)) exactly
    assert abs(np.sqrt(np.mean(out ** 2)) - np.sqrt(ms / (ms + eps))) < 1e-7
    # constant input c: every output is c / sqrt(c^2 + eps)
    c = np.float32(0.003)
    outc = oracle.rmsnorm(np.full(64, c, np.float32), bf16_bits(np.ones(64)), eps)
    np.testing.assert_allclose(outc, c / np.sqrt(np.float64(c) ** 2 + eps), rtol=1e-6)


def test_rmsnorm_scale_invariance_and_gains():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(300).astype(np.float32)
    ones = bf16_bits(np.ones(300))
    a = oracle.rmsnorm(x, ones, 0.0)
    b = oracle.rmsnorm((x * 8.0).astype(np.float32), ones, 0.0)
    np.testing.assert_allclose(a, b, rtol=1e-6)
    g = bf16_bits(np.linspace(-2, 2, 300))  # position-dependent gains catch a reversed index
    np.testing.assert_allclose(oracle.rmsnorm(x, g, 0.0), a * widen(g), rtol=1e-6, atol=1e-7)


# ------------------------------------------------------------------ RoPE
def test_rope_unit_rotation_golden():
    # d = 2, pos = 1, theta irrelevant (i = 0): rotation by exactly 1 radian,
    # counter-clockwise: (1,0) -> (cos 1, sin 1); (0,1) -> (-sin 1, cos 1)
    np.testing.assert_allclose(oracle.rope([1.0, 0.0], 1, 10000.0), [math.cos(1), math.sin(1)], rtol=1e-7)
    np.testing.assert_allclose(oracle.rope([0.0, 1.0], 1, 10000.0), [-math.sin(1), math.cos(1)], rtol=1e-7)


@pytest.mark.parametrize("d,theta,pos", [(8, 10000.0, 5), (64, 500000.0, 1023), (128, 1e6, 16383)])
def test_rope_is_complex_rotation(d, theta, pos):
    rng = np.random.default_rng(d)
    v = rng.standard_normal(d).astype(np.float32)
    h = d // 2
    z = v[:h].astype(np.float64) + 1j * v[h:].astype(np.float64)
    freq = theta ** (-2.0 * np.arange(h) / d)
    zr = z * np.exp(1j * pos * freq)
    got = oracle.rope(v, pos, theta)
    np.testing.assert_allclose(got[:h], zr.real, atol=2e-6)
    np.testing.assert_allclose(got[h:], zr.imag, atol=2e-6)


def test_rope_invariants():
    rng = np.random.default_rng(4)
    q = rng.standard_normal(64).astype(np.float32)
    k = rng.standard_normal(64).astype(np.float32)
    np.testing.assert_array_equal(oracle.rope(q, 0, 500000.0), q)  # identity at position 0
    r = oracle.rope(q, 777, 500000.0)
    pair = lambda v: v[:32] ** 2 + v[32:] ** 2  # noqa: E731
    np.testing.assert_allclose(pair(r), pair(q), rtol=1e-5)  # each pair keeps its norm
    dots = [float(np.dot(oracle.rope(q, p, 5e5), oracle.rope(k, p - 9, 5e5))) for p in (9, 100, 1000)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-4)  # depends only on the offset


# ------------------------------------------------------------------ SiLU / softmax / attention
def test_silu_closed_form():
    assert oracle.silu(0.0) == 0.0
    for z in (-30.0, -3.5, -0.1, 0.7, 2.0, 30.0):
        assert abs(oracle.silu(z) - z * expit(z)) <= 1e-15 * max(1.0, abs(z))
    assert abs(oracle.silu(40.0) - 40.0) < 1e-12


def test_attend_single_position_and_uniform():
    rng = np.random.default_rng(5)
    d = 64
    q = rng.standard_normal(d).astype(np.float32)
    Kr = rng.standard_normal((1, d)).astype(np.float32)
    Vr = rng.standard_normal((1, d)).astype(np.float32)
    np.testing.assert_array_equal(oracle.attend(q, Kr, Vr), Vr[0])
    K = rng.standard_normal((17, d)).astype(np.float32)
    V = rng.standard_normal((17, d)).astype(np.float32)
    np.testing.assert_allclose(oracle.attend(np.zeros(d, np.float32), K, V), V.astype(np.float64).mean(0),
                               rtol=1e-6, atol=1e-7)
    # the weights sum to one: a constant value column comes back unchanged
    np.testing.assert_allclose(oracle.attend(q, K, np.full((17, d), 3.25, np.float32)), 3.25, rtol=1e-7)


def test_attend_scale_closed_form():
    # d=4, q=(1,0,0,0), k0=(2,0,0,0), k1=0: scores 2/sqrt(4)=1 and 0
    q = np.array([1, 0, 0, 0], np.float32)
    K = np.array([[2, 0, 0, 0], [0, 0, 0, 0]], np.float32)
    V = np.array([[1, 0, 0, 0], [0, 1, 0, 0]], np.float32)
    e = math.e
    np.testing.assert_allclose(oracle.attend(q, K, V), [e / (1 + e), 1 / (1 + e), 0, 0], rtol=1e-7)


def test_attend_vs_library_softmax():
    from scipy.special import softmax
    rng = np.random.default_rng(6)
    d, n = 128, 300
    q = rng.standard_normal(d).astype(np.float32)
    K = rng.standard_normal((n, d)).astype(np.float32)
    V = rng.standard_normal((n, d)).astype(np.float32)
    p = softmax(K.astype(np.float64) @ q.astype(np.float64) / np.sqrt(d))
    np.testing.assert_allclose(oracle.attend(q, K, V), p @ V.astype(np.float64), rtol=1e-5, atol=1e-6)


def test_argmax_lowest_index_on_ties():
    assert oracle.argmax(np.array([1, 3, 3, 2], np.float32)) == 1
    assert oracle.argmax(np.array([-1, -1, -1], np.float32)) == 0
    assert oracle.argmax(np.array([0, 0, 5], np.float32)) == 2


# ------------------------------------------------------------------ SwiGLU first stage
def test_swiglu_stage1_vs_library():
    rng = np.random.default_rng(7)
    B, K, N = 3, 96, 70
    x = rng.standard_normal((B, K)).astype(np.float16)
    wg = (rng.standard_normal((K, N)) * 0.1).astype(np.float16)
    wu = (rng.standard_normal((K, N)) * 0.1).astype(np.float16)
    u = lambda a: a.view(np.uint16)  # noqa: E731
    got = oracle.swiglu_stage1_f16(u(x), u(wg), u(wu))
    g = x.astype(np.float64) @ wg.astype(np.float64)
    up = x.astype(np.float64) @ wu.astype(np.float64)
    np.testing.assert_allclose(got, g * expit(g) * up, rtol=1e-6, atol=1e-7)
    # SiLU goes on the gate, not on the up projection
    got0 = oracle.swiglu_stage1_f16(u(x), u(wg), u(np.zeros_like(wu)))
    assert np.all(got0 == 0)


# ------------------------------------------------------------------ the decoder
SMALL = synth.ModelShape("small", n_layers=2, hidden=64, n_heads=4, n_kv_heads=2, head_dim=16,
                         intermediate=96, vocab=50, rms_eps=1e-5, rope_theta=10000.0, tied=False,
                         qk_norm=False, batch=1, prefill=8, steps=4, max_seq=24)


def np_weights(shape, seed=0, scale=0.1):
    """Random bf16 weights as uint16 arrays, gains 1 (for closed-form cases)."""
    rng = np.random.default_rng(seed)
    H, d, I, nq, nkv = shape.hidden, shape.head_dim, shape.intermediate, shape.n_heads, shape.n_kv_heads
    r = lambda *s: bf16_bits(rng.standard_normal(s) * scale)  # noqa: E731
    one = lambda n: bf16_bits(np.ones(n))  # noqa: E731
    w = {"embed": r(shape.vocab, H), "final_norm": one(H), "lm_head": None if shape.tied else r(shape.vocab, H),
         "layers": []}
    for _ in range(shape.n_layers):
        w["layers"].append({"attn_norm": one(H), "wq": r(nq * d, H), "wk": r(nkv * d, H), "wv": r(nkv * d, H),
                            "wo": r(H, nq * d), "q_norm": one(d) if shape.qk_norm else None,
                            "k_norm": one(d) if shape.qk_norm else None, "mlp_norm": one(H),
                            "wg": r(I, H), "wu": r(I, H), "wd": r(H, I)})
    return w


def np_rms(x, eps):
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


@pytest.mark.parametrize("tied", [False, True])
def test_zero_layer_model_closed_form(tied):
    s = SMALL.replace(n_layers=0, tied=tied)
    w = np_weights(s, seed=11)
    m = oracle.OracleModel(s, w)
    tok = 17
    logits, nxt = m.step([tok])
    head = widen(w["embed"] if tied else w["lm_head"])
    want = head @ np_rms(widen(w["embed"][tok]), s.rms_eps)
    np.testing.assert_allclose(logits[0], want, rtol=1e-5, atol=1e-6)
    assert nxt[0] == int(np.argmax(logits[0]))


def test_attention_path_closed_form_uniform_scores():
    """W_q = 0 makes every score 0: each query head returns the plain mean of
    its KV head's values over positions 0..p, KV head = q head // (nq/nkv).
    With W_down = 0 the MLP adds nothing, so the logits have a closed form."""
    s = SMALL.replace(n_layers=1)
    w = np_weights(s, seed=12)
    L0 = w["layers"][0]
    L0["wq"][:] = 0
    L0["wd"][:] = 0
    m = oracle.OracleModel(s, w)
    toks = [3, 41, 7, 29, 11]
    for t in toks:
        logits, _ = m.step([t])
    eps, d, G = s.rms_eps, s.head_dim, s.n_heads // s.n_kv_heads
    X0 = widen(w["embed"][toks])                                    # [T, H]
    Vr = np_rms(X0, eps) @ widen(L0["wv"]).T                        # [T, nkv*d]
    vbar = Vr.mean(0).reshape(s.n_kv_heads, d)
    o = np.concatenate([vbar[h // G] for h in range(s.n_heads)])
    x1 = X0[-1] + widen(L0["wo"]) @ o
    want = widen(w["lm_head"]) @ np_rms(x1, eps)
    np.testing.assert_allclose(logits[0], want, rtol=2e-5, atol=2e-5)


def test_mlp_path_closed_form():
    """W_o = 0 removes attention from the residual stream; the MLP then gives
    x1 = x0 + W_d (SiLU(W_g h) * (W_u h)), h = RMSNorm(x0)."""
    s = SMALL.replace(n_layers=1)
    w = np_weights(s, seed=13)
    L0 = w["layers"][0]
    L0["wo"][:] = 0
    m = oracle.OracleModel(s, w)
    logits, _ = m.step([23])
    x0 = widen(w["embed"][23])
    h = np_rms(x0, s.rms_eps)
    g, u = widen(L0["wg"]) @ h, widen(L0["wu"]) @ h
    x1 = x0 + widen(L0["wd"]) @ (g * expit(g) * u)
    want = widen(w["lm_head"]) @ np_rms(x1, s.rms_eps)
    np.testing.assert_allclose(logits[0], want, rtol=2e-5, atol=2e-5)


def test_layer0_cache_rows_are_rotated_keys_at_their_positions():
    s = SMALL
    w = np_weights(s, seed=14)
    m = oracle.OracleModel(s, w)
    toks = [5, 9, 13, 44, 2, 0, 49]
    for t in toks:
        m.step([t])
    L0 = w["layers"][0]
    for p, t in enumerate(toks):
        h = np_rms(widen(w["embed"][t]), s.rms_eps).astype(np.float32)
        k = oracle.gemv_bf16(L0["wk"], h).reshape(s.n_kv_heads, s.head_dim)
        v = oracle.gemv_bf16(L0["wv"], h).reshape(s.n_kv_heads, s.head_dim)
        for g in range(s.n_kv_heads):
            np.testing.assert_allclose(m.kc[0, 0, g, p], oracle.rope(k[g], p, s.rope_theta), rtol=1e-5, atol=1e-6)
            np.testing.assert_allclose(m.vc[0, 0, g, p], v[g], rtol=1e-6, atol=1e-7)
    assert np.all(m.kc[:, :, :, len(toks):] == 0) and np.all(m.vc[:, :, :, len(toks):] == 0)
    assert m.pos[0] == len(toks)


def test_qk_norm_gives_unit_rms_heads():
    s = SMALL.replace(qk_norm=True, rms_eps=1e-6)
    w = np_weights(s, seed=15)
    m = oracle.OracleModel(s, w)
    for t in [1, 2, 3]:
        m.step([t])
    # per-head RMSNorm with unit gains, then a rotation: each cached key head
    # has norm sqrt(d * ms / (ms + eps)) ~= sqrt(d)
    nrm = np.linalg.norm(m.kc[:, 0, :, :3].astype(np.float64), axis=-1)
    np.testing.assert_allclose(nrm, math.sqrt(s.head_dim), rtol=1e-4)


@pytest.mark.parametrize("qk_norm", [True, False])
def test_qk_norm_makes_logits_blind_to_query_scale(qk_norm):
    """Per-head RMSNorm of q divides out any scale of W_q, so multiplying one
    layer's W_q by 8 (exact in bf16) leaves the logits unchanged up to the eps
    term; without the q norm the scores grow 8x and the logits move.  A q
    branch that is dropped, or that normalises the wrong vector, fails one of
    the two cases."""
    s = SMALL.replace(qk_norm=qk_norm, rms_eps=1e-6)
    w = np_weights(s, seed=21)
    toks = [7, 19, 3, 44]
    base = oracle.OracleModel(s, w)
    for t in toks:
        ref, _ = base.step([t])
    w["layers"][1]["wq"] = bf16_bits(widen(w["layers"][1]["wq"]) * 8.0)
    scaled = oracle.OracleModel(s, w)
    for t in toks:
        got, _ = scaled.step([t])
    rel = float(np.max(np.abs(got - ref)) / np.max(np.abs(ref)))
    if qk_norm:
        assert rel < 1e-5
    else:
        assert rel > 1e-2


def test_qk_norm_gains_closed_form():
    """One layer with the MLP removed (W_down = 0), two positions, distinct
    per-element gains on the q and k head norms: the logits follow from numpy
    alone -- RMSNorm, the projections, per-head RMSNorm times its own gain,
    RoPE as a complex rotation of the (i, i + d/2) pairs, softmax attention
    with KV head = q head // (nq / nkv), O-projection, final norm and head.
    Swapping the two gain vectors, or applying one to both, fails it."""
    s = SMALL.replace(n_layers=1, qk_norm=True, rms_eps=1e-6)
    w = np_weights(s, seed=22)
    L0 = w["layers"][0]
    d, nq, nkv, eps = s.head_dim, s.n_heads, s.n_kv_heads, s.rms_eps
    L0["q_norm"] = bf16_bits(np.linspace(0.5, 2.0, d))
    L0["k_norm"] = bf16_bits(np.linspace(1.75, 0.25, d))
    L0["wd"][:] = 0
    toks = [11, 37]
    m = oracle.OracleModel(s, w)
    for t in toks:
        logits, _ = m.step([t])

    def rot(v, p):
        h = d // 2
        z = (v[..., :h] + 1j * v[..., h:]) * np.exp(1j * p * s.rope_theta ** (-2.0 * np.arange(h) / d))
        return np.concatenate([z.real, z.imag], axis=-1)

    X0 = widen(w["embed"][toks])
    Hn = np_rms(X0, eps)
    gq, gk = widen(L0["q_norm"]), widen(L0["k_norm"])
    K = np.stack([rot(np_rms((widen(L0["wk"]) @ Hn[p]).reshape(nkv, d), eps) * gk, p) for p in range(2)])
    V = np.stack([(widen(L0["wv"]) @ Hn[p]).reshape(nkv, d) for p in range(2)])
    Q = rot(np_rms((widen(L0["wq"]) @ Hn[1]).reshape(nq, d), eps) * gq, 1)
    o = []
    for h in range(nq):
        g = h // (nq // nkv)
        sc = K[:, g] @ Q[h] / math.sqrt(d)
        a = np.exp(sc - sc.max())
        o.append((a / a.sum()) @ V[:, g])
    x1 = X0[1] + widen(L0["wo"]) @ np.concatenate(o)
    want = widen(w["lm_head"]) @ np_rms(x1, eps)
    np.testing.assert_allclose(logits[0], want, rtol=2e-5, atol=2e-5)
    # the two gain vectors are far enough apart that a swap is visible
    L0["q_norm"], L0["k_norm"] = L0["k_norm"].copy(), L0["q_norm"].copy()
    swapped = oracle.OracleModel(s, w)
    for t in toks:
        lsw, _ = swapped.step([t])
    assert float(np.max(np.abs(lsw[0] - want))) > 1e-3 * float(np.max(np.abs(want)))


def test_incremental_decode_equals_full_recompute():
    s = SMALL.replace(n_layers=2, qk_norm=False)
    w = np_weights(s, seed=16)
    toks = [4, 8, 15, 16, 23, 42, 7, 1, 30, 12]
    m = oracle.OracleModel(s, w)
    for t in toks:
        logits, _ = m.step([t])
    full = oracle.OracleModel(s, w).forward_full(toks)
    np.testing.assert_allclose(logits[0], full, rtol=1e-5, atol=1e-6)


def test_batch_rows_are_independent():
    s = SMALL.replace(batch=2)
    w = np_weights(s, seed=17)
    both = oracle.OracleModel(s, w)
    a = oracle.OracleModel(s.replace(batch=1), w)
    b = oracle.OracleModel(s.replace(batch=1), w)
    ta, tb = [3, 1, 4, 1, 5], [9, 2, 6, 5, 3]
    for x, y in zip(ta, tb):
        lb, _ = both.step([x, y])
        la, _ = a.step([x])
        lb1, _ = b.step([y])
    np.testing.assert_array_equal(lb[0], la[0])
    np.testing.assert_array_equal(lb[1], lb1[0])


def test_out_of_range_arguments_rejected():
    s = SMALL
    m = oracle.OracleModel(s, np_weights(s, seed=18))
    with pytest.raises(ValueError):
        m.step([s.vocab])
    m.pos[0] = s.max_seq
    with pytest.raises(ValueError):
        m.step([0])


def test_tiny_workload_runs_and_is_finite():
    tw = synth.make_weights(synth.TINY)
    m = oracle.OracleModel.from_torch(synth.TINY, tw)
    toks = synth.make_tokens(synth.TINY, 6).numpy()
    for i in range(6):
        logits, nxt = m.step(toks[:, i])
    assert np.all(np.isfinite(logits))
    assert nxt[0] == int(np.argmax(logits[0]))
    # random-init logits: sigma ~= 0.02 * sqrt(H) = 0.32 for H = 256
    assert 0.1 < float(np.std(logits)) < 1.0
