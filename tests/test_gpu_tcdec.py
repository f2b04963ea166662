"""The tensor-core batched decode step (mk_tcdec_*) against the oracle: the
megakernel prefills the cache, the tensor-core step decodes the next token of
every sequence on that cache, and the oracle, handed the same cache, checks
that step's logits, argmax and appended K row."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import check_argmax, host_weights, logits_close

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


@needs_cuda
@pytest.mark.parametrize("name,batch,prefill,seqs", [("llama8b", 8, 512, [0, 7]), ("qwen3_8b", 16, 1024, [0, 15]),
                                                     ("llama1b", 32, 256, [0, 31])])
def test_tcdec_step_matches_oracle(name, batch, prefill, seqs):
    import tile_synchronised_b200 as mk
    s = synth.MODELS[name]
    ms = prefill + 2
    tw = synth.make_weights(s, device="cuda")
    model = mk.Model(s, tw, batch=batch, max_seq=ms)
    tokens = synth.make_tokens(s, prefill + 1, batch=batch)
    model.prefill(tokens[:, :prefill].cuda())
    dec = mk.TcDecoder(s, tw, batch, ms, kv_cache=model.kv)
    lg = torch.empty((batch, s.vocab), dtype=torch.float32, device="cuda")
    nxt = dec.step(tokens[:, prefill].contiguous().cuda(), prefill, logits=lg).cpu().numpy()
    torch.cuda.synchronize()
    assert dec.status() == 0
    g = lg.cpu().numpy()
    k, v = model.kv_views()
    host = host_weights(tw)
    tnp = tokens.numpy()
    for b in seqs:
        orc = oracle.OracleModel(s, host, batch=1, max_seq=prefill + 1)
        orc.kc[:, 0, :, :prefill] = k[:, b, :, :prefill].float().cpu().numpy()
        orc.vc[:, 0, :, :prefill] = v[:, b, :, :prefill].float().cpu().numpy()
        orc.pos[0] = prefill
        ref, _ = orc.step([int(tnp[b, prefill])])
        d = logits_close(g[b:b + 1], ref)
        check_argmax(nxt[b:b + 1], g[b:b + 1], ref, d)
        for layer in (0, s.n_layers - 1):
            gk = k[layer, b, :, prefill].float().cpu().numpy()
            want = orc.kc[layer, 0, :, prefill]
            assert np.max(np.abs(gk - want)) <= 2e-2 * np.max(np.abs(want))


@needs_cuda
def test_tcdec_refuses_a_position_past_the_cache():
    import tile_synchronised_b200 as mk
    s = synth.LLAMA1B.replace(n_layers=2)
    tw = synth.make_weights(s, device="cuda")
    dec = mk.TcDecoder(s, tw, 2, 8)
    tok = torch.zeros(2, dtype=torch.int32, device="cuda")
    with pytest.raises(mk.MkError):
        dec.step(tok, 8)


@needs_cuda
def test_tcdec_graph_replay_is_bit_equal_to_eager_launches():
    """The step captured once in a CUDA graph replays at every position: a run
    of consecutive steps through the graph gives the same bits (logits,
    tokens, the K/V rows appended) as the same steps launched kernel by
    kernel, on fresh caches."""
    import tile_synchronised_b200 as mk
    s = synth.LLAMA1B.replace(n_layers=2)
    B, ms, n = 4, 64, 12
    tw = synth.make_weights(s, device="cuda")
    tokens = synth.make_tokens(s, n, batch=B).to(torch.int32).cuda()
    runs = {}
    for graph in (False, True):
        dec = mk.TcDecoder(s, tw, B, ms)
        dec.set_graph(graph)
        lg = torch.empty((B, s.vocab), dtype=torch.float32, device="cuda")
        steps = []
        for p in range(n):
            nxt = dec.step(tokens[:, p].contiguous(), p, logits=lg if p % 3 else None)
            steps.append((lg.clone() if p % 3 else None, nxt.clone()))
        torch.cuda.synchronize()
        assert dec.status() == 0
        runs[graph] = (steps, dec.kv.clone())
        dec.close()
    for p, ((la, na), (lb, nb)) in enumerate(zip(runs[False][0], runs[True][0])):
        assert torch.equal(na, nb), p
        if la is not None:
            assert torch.equal(la, lb), p
    assert torch.equal(runs[False][1], runs[True][1])
