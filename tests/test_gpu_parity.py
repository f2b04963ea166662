"""Parity of the CUDA decode step with the CPU oracle (needs a B200).

Small workloads run whole teacher-forced trajectories through both sides;
the full-size workloads run the GPU trajectory and hand the GPU's KV cache to
the oracle for single steps ("state handoff"), plus sampled layer-0 cache rows
recomputed from the embedding.  The comparison rules live in gpu_common.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import build_pair, check_argmax, host_weights, logits_close, widen_bf16

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="no CUDA device")


def run_trajectory(model, orc, tokens, prefill, steps, check_every=1):
    """Prefill both sides, then teacher-force `steps` tokens; compare logits/argmax."""
    B = model.batch
    model.prefill(tokens[:, :prefill].cuda())
    orc.prefill(tokens[:, :prefill].numpy())
    logits = torch.empty((B, model.shape.vocab), dtype=torch.float32, device="cuda")
    worst, undecided = 0.0, 0
    for s in range(steps):
        tok = tokens[:, prefill + s].contiguous()
        nxt = model.decode(tok.cuda(), logits=logits)
        ref, ref_next = orc.step(tok.numpy())
        if s % check_every == 0 or s == steps - 1:
            g = logits.cpu().numpy()
            d = logits_close(g, ref)
            worst = max(worst, d)
            undecided += check_argmax(nxt.cpu().numpy(), g, ref, d)
    assert model.status() == 0
    return worst, undecided


@needs_cuda
@pytest.mark.parametrize("sync", ["tags", "counters"])
def test_tiny_trajectory_and_kv_indexing(sync):
    s = synth.TINY
    tw, model, orc = build_pair(s, sync=sync)
    k, v = model.kv_views()
    k.view(torch.int16).fill_(-1)  # 0xFFFF: a NaN pattern in bf16
    v.view(torch.int16).fill_(-1)
    model.poison_activations()  # NaN words under a tag no step writes
    tokens = synth.make_tokens(s, s.prefill + s.steps)
    worst, undecided = run_trajectory(model, orc, tokens, s.prefill, s.steps)
    # near-tie steps (oracle top-2 margin within 2x the logit error) are counted,
    # not failed; at most 1 of 32 has been seen, so an eighth is allowed
    assert undecided <= s.steps // 8, (undecided, worst)
    p_final = s.prefill + s.steps
    assert model.position == p_final
    # every written slot matches the oracle's cache; every other slot keeps the poison bits
    for cache, ref in ((k, orc.kc), (v, orc.vc)):
        got = widen_bf16(cache[:, :, :, :p_final])
        want = ref[:, :, :, :p_final]
        assert np.all(np.isfinite(got))
        for l in range(s.n_layers):
            assert np.max(np.abs(got[l] - want[l])) <= 2e-2 * np.max(np.abs(want[l]))
        rest = cache[:, :, :, p_final:].contiguous().view(torch.int16)
        assert bool((rest == -1).all())


@needs_cuda
@pytest.mark.parametrize("variant,sync", [("graph", "tags"), ("graph_pdl", "tags"), ("megakernel", "counters"),
                                          ("tilesync", "tags"), ("tilesync", "counters")])
def test_variants_and_sync_modes_bit_equal(variant, sync):
    """The separate-kernel variants (plain graph, graph + PDL, and the
    tile-synchronised separate kernels in both sync modes), and the
    counter-synchronised megakernel, produce the same bits as the
    tag-synchronised megakernel."""
    s = synth.TINY
    tw = synth.make_weights(s, device="cuda")
    import tile_synchronised_b200 as mk
    a = mk.Model(s, tw, variant="megakernel")
    b = mk.Model(s, tw, variant=variant)
    b.set_sync(sync)
    tokens = synth.make_tokens(s, 24)
    a.prefill(tokens[:, :16].cuda())
    b.prefill(tokens[:, :16].cuda())
    la = torch.empty((1, s.vocab), device="cuda")
    lb = torch.empty((1, s.vocab), device="cuda")
    tok = torch.empty(1, dtype=torch.int32, device="cuda")
    for i in range(16, 24):
        tok.copy_(tokens[:, i])
        na = a.decode(tok, logits=la).clone()
        nb = b.decode(tok, logits=lb).clone()
        assert torch.equal(la, lb), f"step {i}: max|delta| {(la - lb).abs().max().item()}"
        assert torch.equal(na, nb)
    assert a.status() == 0 and b.status() == 0
    ka, va = a.kv_views()
    kb, vb = b.kv_views()
    assert torch.equal(ka[:, :, :, :24], kb[:, :, :, :24]) and torch.equal(va[:, :, :, :24], vb[:, :, :, :24])


@needs_cuda
@pytest.mark.parametrize("case", ["batch3", "qknorm_tied", "d128", "group8"])
def test_tiny_shape_variants(case):
    s = synth.TINY
    batch = 1
    if case == "batch3":
        batch = 3
    elif case == "qknorm_tied":
        s = s.replace(qk_norm=True, tied=True, rms_eps=1e-6, rope_theta=1e6)
    elif case == "d128":
        s = s.replace(head_dim=128, n_heads=4, n_kv_heads=1)
    elif case == "group8":
        s = s.replace(n_heads=8, n_kv_heads=1, head_dim=64, hidden=512, intermediate=1024)
    s = s.replace(batch=batch)
    tw, model, orc = build_pair(s, batch=batch)
    tokens = synth.make_tokens(s, 40, batch=batch)
    worst, undecided = run_trajectory(model, orc, tokens, 24, 16)
    # at most 3 of 16 steps per sequence have been near ties
    assert undecided <= 6 * batch, (undecided, worst)


@needs_cuda
@pytest.mark.parametrize("sync", ["tags", "counters"])
def test_shuffled_schedule_is_bit_equal(sync):
    """Race-detection substitute: the same step under a seeded reordering of
    the per-SM instruction lists (every dependency kept) gives the same bits
    as the planner's order.  8 CTAs, so that every CTA holds several
    instructions of each phase and the reordering changes which instruction
    waits behind which."""
    s = synth.TINY.replace(batch=3)
    tw = synth.make_weights(s, device="cuda")
    import tile_synchronised_b200 as mk
    a = mk.Model(s, tw, batch=3, num_sms=8)
    b = mk.Model(s, tw, batch=3, num_sms=8)
    a.set_sync(sync)
    b.set_sync(sync)
    b.shuffle_schedule(7)
    tokens = synth.make_tokens(s, 28, batch=3)
    a.prefill(tokens[:, :20].cuda())
    b.prefill(tokens[:, :20].cuda())
    la = torch.empty((3, s.vocab), device="cuda")
    lb = torch.empty((3, s.vocab), device="cuda")
    for i in range(20, 28):
        tok = tokens[:, i].contiguous().cuda()
        na = a.decode(tok, logits=la).clone()
        nb = b.decode(tok, logits=lb).clone()
        assert torch.equal(la, lb), f"step {i}: max|delta| {(la - lb).abs().max().item()}"
        assert torch.equal(na, nb)
    assert a.status() == 0 and b.status() == 0
    ka, va = a.kv_views()
    kb, vb = b.kv_views()
    assert torch.equal(ka[:, :, :, :28], kb[:, :, :, :28]) and torch.equal(va[:, :, :, :28], vb[:, :, :, :28])


@needs_cuda
def test_split_kv_chunk_count_does_not_change_results():
    s = synth.TINY
    tw = synth.make_weights(s, device="cuda")
    import tile_synchronised_b200 as mk
    outs = []
    for n in (148, 17, 2):
        m = mk.Model(s, tw, num_sms=n)
        tokens = synth.make_tokens(s, 80)
        m.prefill(tokens[:, :79].cuda())
        lg = torch.empty((1, s.vocab), device="cuda")
        m.decode(tokens[:, 79].contiguous().cuda(), logits=lg)
        assert m.status() == 0
        outs.append(lg.cpu().numpy())
    for o in outs[1:]:
        assert np.max(np.abs(o - outs[0])) <= 1e-3 * np.max(np.abs(outs[0]))


@needs_cuda
@pytest.mark.parametrize("sync", ["tags", "counters"])
def test_wait_timeout_is_reported_and_context_recovers(sync):
    s = synth.TINY
    tw = synth.make_weights(s, device="cuda")
    import tile_synchronised_b200 as mk
    from tile_synchronised_b200 import _lib
    m = mk.Model(s, tw)
    m.set_sync(sync)
    m.set_timeout_ns(20_000_000)  # 20 ms
    # instruction 0 of CTA 0 is a layer-0 QKV tile: without its signal (or,
    # with tags, with its outputs left stale) the attention instructions of
    # layer 0 can never start
    m.drop_signal(0)
    tok = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.decode(tok)
    assert m.status() == _lib.MK_ERR_TIMEOUT
    assert "gave up" in m.last_error()
    with pytest.raises(mk.MkError):
        m.decode(tok)  # poisoned until reset
    m.drop_signal(-1)
    m.reset()
    tokens = synth.make_tokens(s, 8)
    m.prefill(tokens[:, :7].cuda())
    lg = torch.empty((1, s.vocab), device="cuda")
    m.decode(tokens[:, 7].contiguous().cuda(), logits=lg)
    assert m.status() == 0
    orc = oracle.OracleModel.from_torch(s, tw)
    orc.prefill(tokens[:, :7].numpy())
    ref, _ = orc.step(tokens[:, 7].numpy())
    logits_close(lg.cpu().numpy(), ref)


@needs_cuda
@pytest.mark.parametrize("variant,bad", [("megakernel", "vocab"), ("megakernel", "negative"), ("graph", "vocab")])
def test_out_of_range_token_is_reported_and_context_recovers(variant, bad):
    """A token outside [0, vocab) is an invalid argument that lives in device
    memory: the step records it, mk_get_status reports MK_ERR_INVALID with the
    sequence and the token, the context refuses further steps until mk_reset,
    and after the reset the same context decodes correctly again."""
    s = synth.TINY
    tw = synth.make_weights(s, device="cuda")
    import tile_synchronised_b200 as mk
    from tile_synchronised_b200 import _lib
    m = mk.Model(s, tw, variant=variant)
    tokens = synth.make_tokens(s, 8)
    m.prefill(tokens[:, :6].cuda())
    assert m.status() == 0
    value = s.vocab if bad == "vocab" else -1
    m.decode(torch.full((1,), value, dtype=torch.int32, device="cuda"))
    assert m.status() == _lib.MK_ERR_INVALID
    assert f"token {value} of sequence 0" in m.last_error()
    with pytest.raises(mk.MkError):
        m.decode(tokens[:, 6].contiguous().cuda())  # poisoned until reset
    m.reset()
    m.prefill(tokens[:, :7].cuda())
    lg = torch.empty((1, s.vocab), device="cuda")
    m.decode(tokens[:, 7].contiguous().cuda(), logits=lg)
    assert m.status() == 0
    orc = oracle.OracleModel.from_torch(s, tw)
    orc.prefill(tokens[:, :7].numpy())
    ref, _ = orc.step(tokens[:, 7].numpy())
    logits_close(lg.cpu().numpy(), ref)


@needs_cuda
def test_position_bounds():
    s = synth.TINY.replace(max_seq=8)
    tw = synth.make_weights(s, device="cuda")
    import tile_synchronised_b200 as mk
    m = mk.Model(s, tw, max_seq=8)
    tokens = synth.make_tokens(s, 8)
    m.prefill(tokens[:, :6].cuda())
    assert m.position == 6
    tok = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.decode(tok)
    m.decode(tok)
    assert m.position == 8
    with pytest.raises(mk.MkError):
        m.decode(tok)
    with pytest.raises(mk.MkError):
        m.prefill(torch.zeros((1, 9), dtype=torch.int32))
    assert m.status() == 0


# ---------------------------------------------------------------- full-size workloads (state handoff)
def sampled_layer0_rows(shape, tw, k, v, tokens_np, b, positions):
    L0 = tw["layers"][0]
    wk = synth.to_u16(L0["wk"])
    wv = synth.to_u16(L0["wv"])
    emb = tw["embed"]
    ones = synth.to_u16(L0["attn_norm"])
    for p in positions:
        x = emb[int(tokens_np[b, p])].float().cpu().numpy()
        h = oracle.rmsnorm(x, ones, shape.rms_eps)
        kk = oracle.gemv_bf16(wk, h).reshape(shape.n_kv_heads, shape.head_dim)
        vv = oracle.gemv_bf16(wv, h).reshape(shape.n_kv_heads, shape.head_dim)
        for g in range(shape.n_kv_heads):
            kh = kk[g]
            if shape.qk_norm:
                kh = oracle.rmsnorm(kh, synth.to_u16(L0["k_norm"]), shape.rms_eps)
            want_k = oracle.rope(kh, p, shape.rope_theta)
            got_k = k[0, b, g, p].float().cpu().numpy()
            got_v = v[0, b, g, p].float().cpu().numpy()
            assert np.max(np.abs(got_k - want_k)) <= 2e-2 * np.max(np.abs(want_k))
            assert np.max(np.abs(got_v - vv[g])) <= 2e-2 * np.max(np.abs(vv[g]))


def handoff_step(shape, host, model, tokens, pos, seqs):
    """Decode the step at `pos` on the GPU with logits, then for each sequence
    in `seqs` hand the GPU's KV cache (widened to fp32) to the oracle and
    check that step's logits, argmax and appended K row."""
    batch = model.batch
    k, v = model.kv_views()
    lg = torch.empty((batch, shape.vocab), dtype=torch.float32, device="cuda")
    nxt = model.decode(tokens[:, pos].contiguous().cuda(), logits=lg).cpu().numpy()
    assert model.status() == 0
    assert model.position == pos + 1
    g = lg.cpu().numpy()
    tnp = tokens.numpy()
    for b in seqs:
        orc = oracle.OracleModel(shape, host, batch=1, max_seq=pos + 1)
        orc.kc[:, 0, :, :pos] = k[:, b, :, :pos].float().cpu().numpy()
        orc.vc[:, 0, :, :pos] = v[:, b, :, :pos].float().cpu().numpy()
        orc.pos[0] = pos
        ref, _ = orc.step([int(tnp[b, pos])])
        d = logits_close(g[b:b + 1], ref)
        check_argmax(nxt[b:b + 1], g[b:b + 1], ref, d)
        # the cache row this step appended agrees with the oracle's
        for l in (0, shape.n_layers - 1):
            gk = k[l, b, :, pos].float().cpu().numpy()
            assert np.max(np.abs(gk - orc.kc[l, 0, :, pos])) <= 2e-2 * np.max(np.abs(orc.kc[l, 0, :, pos]))


def full_size_case(shape, batch, prefill, extra_steps, seqs, max_seq=None, variant="megakernel"):
    import tile_synchronised_b200 as mk
    ms = max_seq or shape.max_seq
    tw = synth.make_weights(shape, device="cuda")
    model = mk.Model(shape, tw, batch=batch, max_seq=ms, variant=variant)
    tokens = synth.make_tokens(shape, prefill + extra_steps + 1, batch=batch)
    tnp = tokens.numpy()
    model.prefill(tokens[:, :prefill].cuda())
    for s in range(extra_steps):
        model.decode(tokens[:, prefill + s].contiguous().cuda())
    pos = prefill + extra_steps
    assert model.position == pos
    k, v = model.kv_views()
    sampled_layer0_rows(shape, tw, k, v, tnp, seqs[0], [0, 1, pos // 2, pos - 1])
    host = host_weights(tw)
    del tw
    handoff_step(shape, host, model, tokens, pos, seqs)


@needs_cuda
def test_llama1b_handoffs_across_the_benched_window():
    """The benched workload: a 1024-token prefill, then every step of the
    decode window with oracle handoffs at its first, middle and last positions
    (1025, 1152, 1279 of the 1280-slot cache) and sampled layer-0 cache rows."""
    import tile_synchronised_b200 as mk
    s = synth.LLAMA1B
    tw = synth.make_weights(s, device="cuda")
    model = mk.Model(s, tw, batch=1, max_seq=s.max_seq)
    tokens = synth.make_tokens(s, s.max_seq)
    model.prefill(tokens[:, :s.prefill].cuda())
    dev_tokens = tokens.to(dtype=torch.int32).cuda()
    k, v = model.kv_views()
    sampled_layer0_rows(s, tw, k, v, tokens.numpy(), 0, [0, 1, 511, s.prefill - 1])
    host = host_weights(tw)
    del tw
    pos = s.prefill
    for cp in (s.prefill + 1, s.prefill + 128, s.max_seq - 1):
        while pos < cp:
            model.decode(dev_tokens[:, pos].contiguous())
            pos += 1
        handoff_step(s, host, model, tokens, pos, [0])
        pos += 1
    assert model.position == s.max_seq


@needs_cuda
@pytest.mark.parametrize("batch,seqs", [(1, [0]), (8, [0, 7]), (32, [0, 31])])
def test_llama8b_full_size_handoff(batch, seqs):
    s = synth.LLAMA8B
    full_size_case(s, batch, s.prefill, 4, seqs)


@needs_cuda
@pytest.mark.parametrize("name,batch,prefill,seqs", [("llama8b", 32, 512, [0, 31]), ("qwen3_8b", 16, 1024, [0, 15]),
                                                     ("llama1b", 1, 1024, [0])])
def test_tensor_core_variant_full_size_handoff(name, batch, prefill, seqs):
    """The decode step with every projection on the tensor cores over the
    packed weights (MK_TENSOR_CORES), after a tensor-core prefill: a few steps
    (the first launched directly, the second captured, the rest replayed from
    the graph), then a full-depth oracle handoff of the first and last
    sequence."""
    s = synth.MODELS[name]
    full_size_case(s, batch, prefill, 3, seqs, max_seq=prefill + 8, variant="tensor_cores")


@needs_cuda
@pytest.mark.parametrize("batch", [1, 3])
def test_tensor_core_variant_trajectory(batch):
    s = synth.TINY.replace(batch=batch)
    tw, model, orc = build_pair(s, batch=batch, variant="tensor_cores")
    tokens = synth.make_tokens(s, 40, batch=batch)
    worst, undecided = run_trajectory(model, orc, tokens, 24, 16)
    assert undecided <= 6 * batch, (undecided, worst)


@needs_cuda
def test_qwen3_8b_handoff_at_1k():
    s = synth.QWEN3_8B
    full_size_case(s, 16, 1024, 2, [0, 15], max_seq=1040)


@needs_cuda
@pytest.mark.parametrize("C", [4096, 16383])
def test_qwen3_8b_full_depth_handoff_on_a_seeded_cache(C):
    """Full depth (36 layers) at the long-generation checkpoints 4k and 16k.
    Decoding there from a prefill takes minutes, so the cache positions below
    C are filled with seeded N(0, 1) bf16 values instead; the step at C is a
    plain function of whatever cache it reads, so the oracle, handed the same
    cache, checks that step for the first and last sequence of the batch."""
    import tile_synchronised_b200 as mk
    s = synth.QWEN3_8B
    B = 16
    tw = synth.make_weights(s, device="cuda")
    model = mk.Model(s, tw, batch=B, max_seq=C + 1)
    host = host_weights(tw)
    del tw
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    for t in model.kv_views():
        t[:, :, :, :C].normal_(generator=g)
    model.set_position(C)
    tokens = synth.make_tokens(s, C + 1, batch=B)
    handoff_step(s, host, model, tokens, C, [0, B - 1])


@needs_cuda
def test_qwen3_8b_two_layer_clone_1k_to_16k():
    """The Qwen3-8B batch-16 trajectory from a 1024-token prefill to the last
    slot of a 16384-position cache, on a clone cut to 2 layers (same widths,
    heads, qk-norm, theta and vocab) so that every step runs on the GPU in
    about a minute.  At 1k, 4k and 16k the oracle takes the GPU's cache and
    checks one step of two sequences."""
    import tile_synchronised_b200 as mk
    s = synth.QWEN3_8B.replace(n_layers=2)
    B, prefill, ms = 16, 1024, 16384
    tw = synth.make_weights(s, device="cuda")
    model = mk.Model(s, tw, batch=B, max_seq=ms)
    host = host_weights(tw)
    del tw
    tokens = synth.make_tokens(s, ms, batch=B)
    model.prefill(tokens[:, :prefill].cuda())
    dev_tokens = tokens.to(dtype=torch.int32).cuda()
    pos = prefill
    for cp in (1024, 4096, ms - 1):
        while pos < cp:
            model.decode(dev_tokens[:, pos].contiguous())
            pos += 1
        handoff_step(s, host, model, tokens, pos, [0, B - 1])
        pos += 1
    assert model.position == ms


# ---------------------------------------------------------------- the in-step gate/up tilings
@needs_cuda
@pytest.mark.parametrize("batch", [3, 8])
def test_row_tiled_gateup_trajectory(batch):
    """The row tiling of the fused gate/up stage inside the step (every gate/up
    instruction carries at most half of the batch rows, so each weight tile
    streams once per row group) against the oracle, and bit-equal to the
    column tiling on the same tokens."""
    import tile_synchronised_b200 as mk
    s = synth.TINY.replace(batch=batch)
    tw, row, orc = build_pair(s, batch=batch)
    row.set_swiglu_tiling(mk.MK_SWIGLU_ROW)
    assert row.swiglu_tiling() == mk.MK_SWIGLU_ROW
    sched, _ = row.schedule()
    gu = sched[sched["op"] == 4]
    assert int(gu["nb"].max()) == (min(batch, 4) + 1) // 2
    col = mk.Model(s, tw, batch=batch)
    assert col.swiglu_tiling() == mk.MK_SWIGLU_COL
    tokens = synth.make_tokens(s, 40, batch=batch)
    row.prefill(tokens[:, :24].cuda())
    col.prefill(tokens[:, :24].cuda())
    orc.prefill(tokens[:, :24].numpy())
    lr = torch.empty((batch, s.vocab), device="cuda")
    lc = torch.empty((batch, s.vocab), device="cuda")
    undecided = 0
    for i in range(24, 40):
        tok = tokens[:, i].contiguous()
        nr = row.decode(tok.cuda(), logits=lr).cpu().numpy()
        col.decode(tok.cuda(), logits=lc)
        assert torch.equal(lr, lc), f"step {i}: row and column tilings differ"
        ref, _ = orc.step(tok.numpy())
        g = lr.cpu().numpy()
        undecided += check_argmax(nr, g, ref, logits_close(g, ref))
    assert row.status() == 0 and col.status() == 0
    assert undecided <= 16 * batch // 4, undecided


@needs_cuda
def test_tune_picks_a_tiling_and_decoding_stays_within_tolerance():
    """The one-time profiling pass inside the step times both gate/up tilings,
    keeps the faster and restores the position; decoding then continues
    against the oracle."""
    import tile_synchronised_b200 as mk
    s = synth.TINY.replace(batch=8)
    tw, model, orc = build_pair(s, batch=8)
    tokens = synth.make_tokens(s, 40, batch=8)
    model.prefill(tokens[:, :24].cuda())
    orc.prefill(tokens[:, :24].numpy())
    chosen = model.tune()
    assert chosen in (mk.MK_SWIGLU_ROW, mk.MK_SWIGLU_COL)
    assert model.swiglu_tiling() == chosen
    assert model.position == 24
    lg = torch.empty((8, s.vocab), device="cuda")
    for i in range(24, 32):
        tok = tokens[:, i].contiguous()
        nxt = model.decode(tok.cuda(), logits=lg).cpu().numpy()
        ref, _ = orc.step(tok.numpy())
        g = lg.cpu().numpy()
        check_argmax(nxt, g, ref, logits_close(g, ref))
    assert model.status() == 0


# ---------------------------------------------------------------- the fused SwiGLU first stage
@needs_cuda
@pytest.mark.parametrize("B", synth.SWIGLU_BATCHES)
def test_swiglu_stage1_full_size(B):
    import tile_synchronised_b200 as mk
    x, wg, wu = synth.make_swiglu_inputs(B, device="cuda")
    ref = oracle.swiglu_stage1_f16(synth.to_u16(x), synth.to_u16(wg), synth.to_u16(wu))
    amax = float(np.max(np.abs(ref)))
    # tcgen05 tensor cores at every batch: B below a multiple of 16 pads with zero rows
    variants = [mk.MK_SWIGLU_ROW, mk.MK_SWIGLU_COL, mk.MK_SWIGLU_TC, mk.MK_SWIGLU_AUTO]
    for variant in variants:
        out = mk.swiglu_stage1(x, wg, wu, variant=variant)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        # fp16 output rounding (2^-11 relative) plus fp32 accumulation over K = 8192
        assert np.all(np.abs(got - ref) <= 2e-3 * np.abs(ref) + 1e-4 * amax), variant
    chosen, us_row, us_col, us_tc = mk.swiglu_tune(x, wg, wu, out)
    assert chosen in (mk.MK_SWIGLU_ROW, mk.MK_SWIGLU_COL, mk.MK_SWIGLU_TC)
    assert us_row > 0 and us_col > 0 and us_tc > 0


# ---------------------------------------------------------------- the prefill on the tensor cores
@needs_cuda
@pytest.mark.parametrize("case", ["tiny_b1", "tiny_b3_qknorm", "tiny_b4_ksplit", "llama1b"])
def test_tensor_core_prefill_matches_steps_and_oracle(case):
    """The tensor-core prefill (128 positions of a sequence per GEMM chunk,
    causal attention within the chunk) leaves a KV cache that agrees with the
    one the decode steps leave and with the oracle's, and the decode step that
    follows it matches the oracle.  The prompt lengths cover one ragged chunk
    and two and three chunks with a ragged tail; one plan packs a matrix as
    several K blocks."""
    import tile_synchronised_b200 as mk
    from tile_synchronised_b200 import _lib
    if case == "llama1b":
        s, B, T = synth.LLAMA1B, 1, 100
    elif case == "tiny_b1":
        s, B, T = synth.TINY, 1, 21
    elif case == "tiny_b4_ksplit":
        # 4 rows x 5120 fp32 exceed the 64 KB activation region: the plan
        # packs the down projection as two K blocks, read by a 4-D tensor map
        s, B, T = synth.TINY.replace(intermediate=5120), 4, 140
    else:
        s, B, T = synth.TINY.replace(qk_norm=True, rms_eps=1e-6), 3, 300
    ms = T + 4
    tw = synth.make_weights(s, device="cuda")
    tokens = synth.make_tokens(s, T + 1, batch=B)
    tc = mk.Model(s, tw, batch=B, max_seq=ms)
    tc.set_prefill("tc")
    steps = mk.Model(s, tw, batch=B, max_seq=ms)
    steps.set_prefill("steps")
    for m in (tc, steps):
        m.prefill(tokens[:, :T].cuda())
        assert m.position == T
    assert tc.status() == 0 and steps.status() == 0
    orc = oracle.OracleModel.from_torch(s, tw, batch=B, max_seq=ms)
    orc.prefill(tokens[:, :T].numpy())
    (kt, vt), (ks, vs) = tc.kv_views(), steps.kv_views()
    for got, other, ref in ((kt, ks, orc.kc), (vt, vs, orc.vc)):
        g = widen_bf16(got[:, :, :, :T])
        o = widen_bf16(other[:, :, :, :T])
        for l in range(s.n_layers):
            scale = np.max(np.abs(ref[l, :, :, :T]))
            assert np.max(np.abs(g[l] - ref[l, :, :, :T])) <= 2e-2 * scale, l
            assert np.max(np.abs(g[l] - o[l])) <= 2e-2 * scale, l
    lg = torch.empty((B, s.vocab), device="cuda")
    nxt = tc.decode(tokens[:, T].contiguous().cuda(), logits=lg).cpu().numpy()
    ref, _ = orc.step(tokens[:, T].numpy())
    g = lg.cpu().numpy()
    check_argmax(nxt, g, ref, logits_close(g, ref))
    assert tc.status() == 0
    # a token outside the vocabulary in the prompt is reported like a decode step's
    bad = tokens[:, :T].clone()
    bad[B - 1, T // 2] = s.vocab
    tc.reset()
    tc.prefill(bad.cuda())
    assert tc.status() == _lib.MK_ERR_INVALID
    assert f"sequence {B - 1}" in tc.last_error()
