"""Parity of the isolated split-KV decode attention with the CPU oracle.

Both sides read the same bf16 cache bytes (the oracle widens them exactly);
positions at and beyond n_pos hold the bf16 NaN pattern, so any read past the
attended range shows up as NaN.  Tolerance: the GPU sums at most a few
thousand fp32 terms per output, each rounding at 2^-24 relative, against the
oracle's double sums, so 1e-4 * max|V| bounds the honest error with margin
while a wrong position, head or scale is off by O(max|V|).
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="no CUDA device")


def oracle_attention(q, k, v, n_pos):
    B, nq, d = q.shape
    nkv = k.shape[1]
    G = nq // nkv
    qn = q.cpu().numpy()
    kf = k[:, :, :n_pos].float().cpu().numpy()
    vf = v[:, :, :n_pos].float().cpu().numpy()
    out = np.empty((B, nq, d), dtype=np.float32)
    for b in range(B):
        for h in range(nq):
            out[b, h] = oracle.attend(np.ascontiguousarray(qn[b, h]), np.ascontiguousarray(kf[b, h // G]),
                                      np.ascontiguousarray(vf[b, h // G]))
    return out


CASES = [  # batch, nq, nkv, d, max_seq, n_pos, chunks
    (1, 32, 8, 64, 1280, 1025, 0),    # Llama-3.2-1B layer at the bench positions
    (3, 4, 2, 64, 96, 1, 0),          # a single position: returns V[0]
    (2, 8, 1, 128, 600, 517, 7),      # GQA group 8, ragged chunks
    (1, 32, 8, 128, 2048, 2048, 64),  # full cache, many chunks
    (2, 12, 4, 256, 64, 33, 3),       # group 3, d = 256
    (1, 8, 8, 128, 100, 100, 100),    # MHA, one position per chunk
    (16, 32, 8, 128, 1100, 1024, 0),  # Qwen3-8B batch 16 at 1k
    (2, 16, 2, 64, 3000, 2777, 0),    # group 8 at d = 64, ragged last stage
    (1, 16, 8, 128, 9000, 8191, 5),   # group 2, chunks of 1638 / 1639 positions
    (2, 32, 8, 128, 16400, 16384, 0),  # Qwen3-8B layer at 16k: long chunks over the stage ring
    (3, 8, 4, 64, 700, 129, 2),       # group 2 at d = 64: one full stage + one position
]


@needs_cuda
@pytest.mark.parametrize("B,nq,nkv,d,max_seq,n_pos,chunks", CASES)
def test_attention_matches_oracle(B, nq, nkv, d, max_seq, n_pos, chunks):
    import tile_synchronised_b200 as mk
    q, k, v = synth.make_attention_inputs(B, nq, nkv, d, max_seq, n_pos, q_std=2.0)
    got = mk.attention_decode(q.cuda(), k.cuda(), v.cuda(), n_pos, chunks=chunks)
    torch.cuda.synchronize()
    ref = oracle_attention(q, k, v, n_pos)
    g = got.cpu().numpy()
    assert np.isfinite(g).all()
    vmax = float(v[:, :, :n_pos].float().abs().max())
    assert float(np.max(np.abs(g - ref))) <= 1e-4 * vmax
    if n_pos == 1:  # softmax over one position is 1: the output is V[0] exactly
        G = nq // nkv
        v0 = v[:, :, 0].float().numpy()
        for h in range(nq):
            assert np.array_equal(g[:, h], v0[:, h // G])


@needs_cuda
def test_attention_chunking_changes_only_rounding():
    import tile_synchronised_b200 as mk
    q, k, v = synth.make_attention_inputs(2, 32, 8, 128, 1500, 1400, q_std=3.0)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    one = mk.attention_decode(q, k, v, 1400, chunks=1)
    many = mk.attention_decode(q, k, v, 1400, chunks=40)
    torch.cuda.synchronize()
    assert float((one - many).abs().max()) <= 1e-5 * float(one.abs().max())


@needs_cuda
def test_attention_rejects_bad_arguments():
    import tile_synchronised_b200 as mk
    from tile_synchronised_b200._lib import MkError
    q, k, v = synth.make_attention_inputs(1, 4, 2, 64, 32, 16)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    with pytest.raises(MkError, match="n_pos"):
        mk.attention_decode(q, k, v, 33)
    with pytest.raises(MkError, match="chunks"):
        mk.attention_decode(q, k, v, 16, chunks=17)
    with pytest.raises(MkError, match="scratch"):
        mk.attention_decode(q, k, v, 16, chunks=4, scratch=torch.empty(16, dtype=torch.uint8, device="cuda"))
