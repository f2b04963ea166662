"""The tcgen05 decode projection (mk_linear_tc) against the oracle's GEMV,
row by row, at the projection shapes of the batched decode configurations
and at ragged shapes (row tiles and K blocks that do not divide evenly)."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")

SHAPES = [
    # (B, K, M)
    (16, 4096, 4096),     # Llama-8B / Qwen3-8B O projection, batch 16 (K split 4)
    (32, 4096, 6144),     # Llama-8B QKV, batch 32 (K split 2)
    (32, 14336, 4096),    # Llama-8B down projection, batch 32
    (64, 4096, 14336),    # one half of gate/up, batch 64 (no split, 112 row tiles)
    (1, 2048, 2048),      # batch 1 padded to 16 columns
    (8, 4096, 4096),      # batch 8
    (5, 320, 200),        # ragged rows (2 tiles, the second partial), 5 K blocks over a pair
    (16, 4096, 128256),   # an LM head: 1002 row tiles, several waves
    (256, 1024, 1024),    # 256 columns (a 128-position prefill chunk as hi/lo pairs), K split 2
]


def reference(x, w):
    """Oracle GEMV per batch row, and the matching sum of |x_k w_k| that bounds
    any fp32 summation order."""
    xu = x.float().cpu().numpy()
    wu = synth.to_u16(w)
    wabs = wu & np.uint16(0x7FFF)
    ref = np.stack([oracle.gemv_bf16(wu, xu[b]) for b in range(xu.shape[0])])
    mag = np.stack([oracle.gemv_bf16(wabs, np.abs(xu[b])) for b in range(xu.shape[0])])
    return ref, mag


@needs_cuda
@pytest.mark.parametrize("B,K,M", SHAPES)
def test_linear_tc_matches_oracle(B, K, M):
    import tile_synchronised_b200 as mk
    x, w = synth.make_linear_inputs(B, K, M, device="cuda")
    y = mk.linear_tc(x, w)
    torch.cuda.synchronize()
    got = y.cpu().numpy()
    assert got.shape == (B, M) and np.isfinite(got).all()
    ref, mag = reference(x, w)
    # bf16 x bf16 products are exact in fp32; any order of K fp32 additions is
    # within K * 2^-24 * sum|x w| of the exact sum (the oracle's own rounding
    # to fp32 adds 2^-24 |y|)
    bound = 2.0 * K * 2.0 ** -24 * mag + 2.0 ** -23 * np.abs(ref) + 1e-30
    assert np.all(np.abs(got.astype(np.float64) - ref) <= bound)


@needs_cuda
def test_linear_tc_is_deterministic_and_writes_only_its_rows():
    import tile_synchronised_b200 as mk
    B, K, M = 5, 320, 200
    x, w = synth.make_linear_inputs(B, K, M, device="cuda")
    big = torch.full((B + 2, M), 7.0, dtype=torch.float32, device="cuda")
    y1 = mk.linear_tc(x, w, out=big[:B])
    y2 = mk.linear_tc(x, w)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert torch.all(big[B:] == 7.0)


STREAMK_SHAPES = [
    # (B, K, M): stream-K where the 128-row tiles do not fill the SMs evenly
    (16, 4096, 4096),     # 32 tiles: each split across ~4.6 CTAs (owners add 3-5 contributions)
    (32, 4096, 6144),     # Llama-8B QKV: 48 tiles
    (32, 14336, 4096),    # Llama-8B down: 224 K blocks per tile
    (32, 4096, 14336),    # 112 tiles: ranges of 48 units over tile boundaries
    (32, 4096, 24576),    # a Qwen3-8B packed gate/up: 192 tiles, up to 3 segments per CTA
    (1, 2048, 2048),      # batch 1 (N padded to 16)
    (64, 4096, 4096),     # batch 64: N = 64 accumulator columns per segment
    (3, 8192, 1000),      # ragged rows: the last tile is partial
    (5, 320, 200),        # 2 tiles x 5 K blocks over 2 CTAs
    (256, 2048, 2048),    # 256 columns: at most 2 segments of a CTA in tensor memory
]


@needs_cuda
@pytest.mark.parametrize("B,K,M", STREAMK_SHAPES)
def test_linear_tc_streamk_matches_oracle(B, K, M):
    import tile_synchronised_b200 as mk
    assert mk.linear_tc_streamk_grid(B, K, M) >= 2, "this shape should run the stream-K kernel"
    x, w = synth.make_linear_inputs(B, K, M, device="cuda")
    ws = torch.zeros(mk.linear_tc_streamk_workspace_bytes(), dtype=torch.uint8, device="cuda")
    y = mk.linear_tc_streamk(x, w, workspace=ws)
    y2 = mk.linear_tc_streamk(x, w, workspace=ws)
    torch.cuda.synchronize()
    got = y.cpu().numpy()
    assert got.shape == (B, M) and np.isfinite(got).all()
    assert torch.equal(y, y2), "stream-K sums contributions in a fixed order"
    # every flag is lowered again for the next call
    n_flags = 256
    assert int(ws[-4 * n_flags:].count_nonzero()) == 0
    ref, mag = reference(x, w)
    bound = 2.0 * K * 2.0 ** -24 * mag + 2.0 ** -23 * np.abs(ref) + 1e-30
    assert np.all(np.abs(got.astype(np.float64) - ref) <= bound)


@needs_cuda
def test_linear_tc_streamk_falls_back_where_tiles_fill_the_sms():
    import tile_synchronised_b200 as mk
    B, K, M = 16, 1024, 128256  # an LM head: 1002 tiles
    assert mk.linear_tc_streamk_grid(B, K, M) == 0
    x, w = synth.make_linear_inputs(B, K, M, device="cuda")
    y = mk.linear_tc_streamk(x, w)
    y0 = mk.linear_tc(x, w)
    torch.cuda.synchronize()
    assert torch.equal(y, y0)
