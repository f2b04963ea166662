"""The no-allocation attention entry point (collected last on purpose: it must
pass both alone and after every other GPU test has run in the process).

mk_attention_decode_noalloc runs the same kernels as mk_attention_decode with
its partial records in a fixed device array inside libmk.so.  Two consecutive
calls are compared with the scratch-argument entry point: the second call
checks that nothing left over from the first (the array is reused, never
cleared) leaks into the result.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="no CUDA device")


def _tol(ref):
    return 1e-6 * float(ref.abs().max())


@needs_cuda
def test_noalloc_matches_scratch_entry_point_on_consecutive_calls():
    import tile_synchronised_b200 as mk
    cases = [(1, 32, 8, 64, 1280, 1025, 0, 21), (2, 8, 1, 128, 600, 517, 7, 22)]
    for B, nq, nkv, d, max_seq, n_pos, chunks, seed in cases:
        q, k, v = (t.cuda() for t in synth.make_attention_inputs(B, nq, nkv, d, max_seq, n_pos, seed=seed))
        c = chunks or mk.attention_chunks(B, nkv, n_pos)
        for call in range(2):
            qc = q * (1.0 + call)  # the second call sees other scores
            ref = mk.attention_decode(qc, k, v, n_pos, chunks=c)
            out = torch.full_like(ref, float("nan"))
            mk.attention_decode_noalloc(qc, k, v, n_pos, out, chunks=c)
            torch.cuda.synchronize()
            assert torch.isfinite(out).all(), f"call {call}"
            assert float((out - ref).abs().max()) <= _tol(ref), f"call {call}"


@needs_cuda
def test_noalloc_refuses_oversize_and_fits_automatic_chunks():
    import tile_synchronised_b200 as mk
    from tile_synchronised_b200 import _lib
    limit = int(_lib.load().mk_attention_noalloc_limit_bytes())
    assert limit == 4 << 20
    # batch 16 x 32 heads x (128 + 2) floats = 266240 bytes per chunk: 15 chunks fit, 16 do not
    B, nq, nkv, d, max_seq, n_pos = 16, 32, 8, 128, 1100, 1024
    q, k, v = (t.cuda() for t in synth.make_attention_inputs(B, nq, nkv, d, max_seq, n_pos, seed=23))
    out = torch.empty((B, nq, d), dtype=torch.float32, device="cuda")
    with pytest.raises(_lib.MkError, match="above the fixed 4194304-byte scratch"):
        mk.attention_decode_noalloc(q, k, v, n_pos, out, chunks=16)
    mk.attention_decode_noalloc(q, k, v, n_pos, out, chunks=15)
    ref = mk.attention_decode(q, k, v, n_pos, chunks=15)
    torch.cuda.synchronize()
    assert float((out - ref).abs().max()) <= _tol(ref)
    # one chunk of 64 sequences x 64 heads x 258 floats is 4.2 MB: refused even with automatic chunks
    q2, k2, v2 = (t.cuda() for t in synth.make_attention_inputs(64, 64, 8, 256, 16, 16, seed=24))
    out2 = torch.empty((64, 64, 256), dtype=torch.float32, device="cuda")
    with pytest.raises(_lib.MkError, match="no-alloc"):
        mk.attention_decode_noalloc(q2, k2, v2, 16, out2)
