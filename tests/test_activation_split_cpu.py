"""Why the tensor-core decode feeds every activation row to the MMA as two
bf16 rows (hi = bf16(x), lo = bf16(x - hi)): a CPU emulation of one decode
step of the Llama-3.2-1B architecture (cut to 4 layers, seeded weights, an
8-position cache), in which every projection input is first rounded the way
the MMA would see it.  Plain bf16 rounding moves the logits by a few 1e-3 of
their range after four layers (and grows with depth); the hi/lo pair keeps
the error three orders of magnitude lower.  Pure numpy, no GPU."""
import numpy as np

import synth


def bf16(x):
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000  # round to nearest even at 8 significant bits
    return u.astype(np.uint32).view(np.float32)


def as_exact(x):
    return x


def as_bf16(x):
    return bf16(x)


def as_hilo(x):
    hi = bf16(x)
    return hi + bf16(x - hi)


def rms(x, g, eps):
    return x / np.sqrt(np.mean(x * x) + eps) * g


def rope(v, p, theta, d):
    i = np.arange(d // 2)
    ang = p * theta ** (-2.0 * i / d)
    c, s = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    a, b = v[..., :d // 2], v[..., d // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], -1)


def test_hilo_split_keeps_decode_logits_near_exact():
    s = synth.LLAMA1B.replace(n_layers=4)
    ctx = 8
    tw = synth.make_weights(s, device="cpu")
    nq, nkv, d = s.n_heads, s.n_kv_heads, s.head_dim
    G = nq // nkv
    E = tw["embed"].float().numpy()
    W = [{k: (None if v is None else v.float().numpy()) for k, v in lw.items()} for lw in tw["layers"]]
    gf = tw["final_norm"].float().numpy()
    toks = synth.make_tokens(s, ctx + 1)[0].numpy()
    cache = [[np.zeros((nkv, ctx + 1, d), np.float32), np.zeros((nkv, ctx + 1, d), np.float32)]
             for _ in range(s.n_layers)]

    def step(tok, p, r, write):
        x = E[tok].copy()
        for l, lw in enumerate(W):
            h = r(rms(x, lw["attn_norm"], s.rms_eps))
            q = rope((lw["wq"] @ h).reshape(nq, d), p, s.rope_theta, d)
            k = rope((lw["wk"] @ h).reshape(nkv, d), p, s.rope_theta, d)
            v = (lw["wv"] @ h).reshape(nkv, d)
            K = np.concatenate([cache[l][0][:, :p], k[:, None]], 1)
            V = np.concatenate([cache[l][1][:, :p], v[:, None]], 1)
            if write:
                cache[l][0][:, p], cache[l][1][:, p] = k, v
            o = np.empty((nq, d), np.float32)
            for hh in range(nq):
                sc = K[hh // G] @ q[hh] / np.sqrt(d)
                w = np.exp(sc - sc.max())
                o[hh] = (w / w.sum()) @ V[hh // G]
            x = x + lw["wo"] @ r(o.reshape(-1))
            h2 = r(rms(x, lw["mlp_norm"], s.rms_eps))
            g, u = lw["wg"] @ h2, lw["wu"] @ h2
            x = x + lw["wd"] @ r(g / (1 + np.exp(-g)) * u)
        return E @ r(rms(x, gf, s.rms_eps))  # tied head

    for p in range(ctx):
        step(toks[p], p, as_exact, True)
    ref = step(toks[ctx], ctx, as_exact, False)
    scale = np.max(np.abs(ref))
    err_bf16 = np.max(np.abs(step(toks[ctx], ctx, as_bf16, False) - ref)) / scale
    err_hilo = np.max(np.abs(step(toks[ctx], ctx, as_hilo, False) - ref)) / scale
    assert err_hilo < 1e-4
    assert err_bf16 > 100 * err_hilo
