"""Host-side checks of the C-ABI library (no GPU): it builds, loads, exports
every symbol include/mk.h declares, and its native scheduler produces valid,
deadlock-free plans for every workload shape."""
import ctypes as C
import os
import re
import subprocess

import pytest

import synth
import tile_synchronised_b200 as mkpy
from tile_synchronised_b200 import _lib
from tile_synchronised_b200 import build as mkbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mk.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mk_[a-z0-9_]+)\s*\(", text)))


def test_library_builds_for_sm100a():
    path = mkbuild.build()
    assert os.path.exists(path)
    assert "arch=compute_100a,code=sm_100a" in " ".join(mkbuild.NVCC_FLAGS)


def test_every_declared_symbol_is_exported():
    syms = declared_symbols()
    assert len(syms) >= 19
    assert set(syms) == set(_lib.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", mkbuild.LIB], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (mk_[a-z0-9_]+)$", out, flags=re.M))
    missing = [s for s in syms if s not in exported]
    assert not missing, missing
    L = _lib.load()
    for s in syms:
        assert getattr(L, s) is not None


WORKLOADS = [(synth.TINY, 1), (synth.TINY, 3), (synth.LLAMA1B, 1), (synth.LLAMA8B, 1), (synth.LLAMA8B, 8),
             (synth.LLAMA8B, 32), (synth.QWEN3_8B, 16)]


@pytest.mark.parametrize("shape,batch", WORKLOADS, ids=[f"{s.name}-b{b}" for s, b in WORKLOADS])
def test_plans_validate(shape, batch):
    p = mkpy.Plan(shape, batch, shape.max_seq, num_sms=148)
    p.validate()
    info = p.info()
    assert info["n_ctas"] == 148
    assert 2 <= info["ring_stages"] <= 8
    # the workspace holds at least every streamed weight once (repacked, padded)
    assert p.workspace_bytes() >= shape.replace(batch=batch).weight_bytes() * 0.99
    s = shape
    assert p.kv_cache_bytes() == 2 * s.n_layers * batch * s.n_kv_heads * s.max_seq * s.head_dim * 2


@pytest.mark.parametrize("n_ctas", [1, 7, 132, 148])
def test_plans_validate_for_any_cta_count(n_ctas):
    p = mkpy.Plan(synth.TINY, 2, synth.TINY.max_seq, num_sms=n_ctas)
    p.validate()
    assert p.info()["n_ctas"] == n_ctas


SHUFFLE_CASES = [(synth.TINY, 3, 8), (synth.LLAMA1B, 1, 148), (synth.LLAMA8B, 8, 148), (synth.QWEN3_8B, 16, 148)]


@pytest.mark.parametrize("shape,batch,n_ctas", SHUFFLE_CASES, ids=[f"{s.name}-b{b}-c{n}" for s, b, n in SHUFFLE_CASES])
def test_shuffled_schedules_keep_every_instruction_and_validate(shape, batch, n_ctas):
    """The race-detection substitute: a seeded reordering of the per-SM lists
    that keeps each list in phase order.  It must keep every instruction
    exactly once (the same multiset), keep each CTA's phases in order, move
    the LM head's publishing flag to the last LM instruction of every CTA that
    has one, pass the deadlock / count simulation, and differ from the
    planner's order."""
    import numpy as np
    base = mkpy.Plan(shape, batch, shape.max_seq, num_sms=n_ctas)
    ref, ref_base = base.schedule()
    key = lambda a: np.sort(a[["op", "layer", "tile", "kb0", "b0"]], order=["op", "layer", "tile", "kb0", "b0"])  # noqa: E731
    phase_rank = {1: 0, 2: 1, 7: 2, 3: 3, 4: 4, 5: 5, 6: 6}
    for seed in (1, 2, 3):
        p = mkpy.Plan(shape, batch, shape.max_seq, num_sms=n_ctas)
        p.shuffle_schedule(seed)
        p.validate()
        got, got_base = p.schedule()
        assert len(got) == len(ref) and np.array_equal(key(got), key(ref))
        assert not np.array_equal(got[["op", "layer", "tile", "b0"]], ref[["op", "layer", "tile", "b0"]])
        for c in range(n_ctas):
            lst = got[got_base[c]:got_base[c + 1]]
            order = [(int(i["layer"]) if i["op"] != 6 else 1 << 20, phase_rank[int(i["op"])]) for i in lst]
            assert order == sorted(order), f"CTA {c} is out of phase order"
            lm = np.flatnonzero(lst["op"] == 6)
            if len(lm):
                flags = lst["flags"][lm] & 2
                assert flags[-1] == 2 and not flags[:-1].any()


def _create(shape, batch=1, **kw):
    lib = _lib.load()
    cfg = mkpy.make_config(shape, batch, shape.max_seq, "megakernel", 148)
    for k, v in kw.items():
        setattr(cfg, k, v)
    ctx = C.c_void_p()
    st = lib.mk_create(C.byref(cfg), -1, C.byref(ctx))
    if st == 0:
        lib.mk_destroy(ctx)
    return st


def test_create_rejects_bad_configs():
    assert _create(synth.TINY) == _lib.MK_OK
    assert _create(synth.TINY, head_dim=96) == _lib.MK_ERR_UNSUPPORTED
    assert _create(synth.TINY, n_kv_heads=3) == _lib.MK_ERR_UNSUPPORTED
    assert _create(synth.TINY, batch=0) == _lib.MK_ERR_INVALID
    assert _create(synth.TINY, batch=65) == _lib.MK_ERR_UNSUPPORTED
    assert _create(synth.TINY, hidden=260) == _lib.MK_ERR_UNSUPPORTED
    assert _create(synth.TINY, dtype=1) == _lib.MK_ERR_UNSUPPORTED
    assert _create(synth.TINY, num_sms=0) == _lib.MK_ERR_INVALID  # no device to ask


def test_device_calls_refuse_without_device():
    lib = _lib.load()
    p = mkpy.Plan(synth.TINY, 1, synth.TINY.max_seq)
    w = _lib.MkWeights()
    assert lib.mk_load_weights(p.ctx, C.byref(w), None, None, None) == _lib.MK_ERR_STATE
    assert lib.mk_decode_step(p.ctx, None, None, None, None) == _lib.MK_ERR_STATE
    assert "mk_load_weights" in lib.mk_last_error(p.ctx).decode() or lib.mk_last_error(p.ctx)


def test_swiglu_argument_checks_need_no_device():
    lib = _lib.load()
    dummy = C.c_void_p(256)
    # misaligned pointer, bad sizes, null: all refused before any launch
    assert lib.mk_swiglu_stage1(C.c_void_p(8), dummy, dummy, dummy, 1, 8192, 7168, 0, None) == _lib.MK_ERR_INVALID
    assert lib.mk_swiglu_stage1(dummy, dummy, dummy, dummy, 0, 8192, 7168, 0, None) == _lib.MK_ERR_INVALID
    assert lib.mk_swiglu_stage1(dummy, dummy, dummy, dummy, 65, 8192, 7168, 0, None) == _lib.MK_ERR_INVALID
    assert lib.mk_swiglu_stage1(dummy, dummy, dummy, dummy, 1, 8200, 7168, 0, None) == _lib.MK_ERR_INVALID
    assert lib.mk_swiglu_stage1(None, dummy, dummy, dummy, 1, 8192, 7168, 0, None) == _lib.MK_ERR_INVALID


def test_attention_argument_checks_need_no_device():
    lib = _lib.load()
    d = C.c_void_p(256)
    f = lib.mk_attention_decode
    ok = (1, 32, 8, 64, 128, 100, 4)  # batch, nq, nkv, d, max_seq, n_pos, chunks
    need = lib.mk_attention_scratch_bytes(1, 32, 64, 4)
    assert need == 32 * 4 * 66 * 4
    assert lib.mk_attention_scratch_bytes(0, 32, 64, 4) == 0
    assert f(None, d, d, *ok, d, d, need, None) == _lib.MK_ERR_INVALID
    assert "null" in lib.mk_last_error(None).decode()
    assert f(C.c_void_p(8), d, d, *ok, d, d, need, None) == _lib.MK_ERR_INVALID
    assert "aligned" in lib.mk_last_error(None).decode()
    assert f(d, d, d, 1, 32, 8, 96, 128, 100, 4, d, d, need, None) == _lib.MK_ERR_UNSUPPORTED
    assert f(d, d, d, 1, 32, 2, 64, 128, 100, 4, d, d, need, None) == _lib.MK_ERR_INVALID  # 16 heads per KV head
    assert f(d, d, d, 1, 32, 8, 64, 128, 129, 4, d, d, need, None) == _lib.MK_ERR_INVALID  # n_pos > max_seq
    assert f(d, d, d, 1, 32, 8, 64, 128, 3, 4, d, d, need, None) == _lib.MK_ERR_INVALID   # chunks > n_pos
    assert "chunks" in lib.mk_last_error(None).decode()
    assert f(d, d, d, *ok, d, d, need - 4, None) == _lib.MK_ERR_INVALID                  # scratch too small
    assert "scratch" in lib.mk_last_error(None).decode()


def test_noalloc_attention_refuses_oversize_without_a_device():
    lib = _lib.load()
    d = C.c_void_p(256)
    assert lib.mk_attention_noalloc_limit_bytes() == 4 << 20
    # 16 x 32 heads x 16 chunks x 130 floats = 4259840 bytes > 4 MiB
    st = lib.mk_attention_decode_noalloc(d, d, d, 16, 32, 8, 128, 1100, 1024, 16, d, None)
    assert st == _lib.MK_ERR_INVALID
    assert "4259840" in lib.mk_last_error(None).decode()


def test_linear_tc_plan_and_argument_checks_need_no_device():
    lib = _lib.load()
    d = C.c_void_p(256)
    # K split per row tile: a cluster of 2 or 4 CTAs while the grid stays within 148 SMs and
    # every CTA keeps two K blocks
    assert mkpy.linear_tc_split(16, 4096, 4096) == 4      # 32 row tiles -> 128 CTAs
    assert mkpy.linear_tc_split(32, 4096, 6144) == 2      # 48 row tiles -> 96 CTAs
    assert mkpy.linear_tc_split(16, 4096, 14336) == 1     # 112 row tiles
    assert mkpy.linear_tc_split(16, 4096, 128256) == 1    # LM head: 1002 row tiles
    assert mkpy.linear_tc_split(5, 320, 200) == 2         # 2 row tiles, 5 K blocks: 4 would leave 1 per CTA
    assert mkpy.linear_tc_split(64, 14336, 4096) == 4
    s = C.c_int()
    assert lib.mk_linear_tc_split(0, 4096, 4096, C.byref(s)) == _lib.MK_ERR_UNSUPPORTED
    assert lib.mk_linear_tc_split(257, 4096, 4096, C.byref(s)) == _lib.MK_ERR_UNSUPPORTED
    assert mkpy.linear_tc_split(256, 2048, 2048) == 2     # 256 columns: the partials of 4 CTAs would not fit
    assert lib.mk_linear_tc_split(16, 4000, 4096, C.byref(s)) == _lib.MK_ERR_UNSUPPORTED
    assert lib.mk_linear_tc_split(16, 4096, 4096, None) == _lib.MK_ERR_INVALID
    # refused before any launch
    assert lib.mk_linear_tc(None, d, d, 16, 4096, 4096, None) == _lib.MK_ERR_INVALID
    assert "null" in lib.mk_last_error(None).decode()
    assert lib.mk_linear_tc(C.c_void_p(8), d, d, 16, 4096, 4096, None) == _lib.MK_ERR_INVALID
    assert "aligned" in lib.mk_last_error(None).decode()
    assert lib.mk_linear_tc(d, d, d, 0, 4096, 4096, None) == _lib.MK_ERR_INVALID
    assert lib.mk_linear_tc(d, d, d, 16, 4000, 4096, None) == _lib.MK_ERR_UNSUPPORTED
    assert "multiple of 64" in lib.mk_last_error(None).decode()
    assert lib.mk_linear_tc(d, d, d, 257, 4096, 4096, None) == _lib.MK_ERR_UNSUPPORTED


def test_linear_tc_streamk_plan_and_argument_checks_need_no_device():
    lib = _lib.load()
    d = C.c_void_p(256)
    need = mkpy.linear_tc_streamk_workspace_bytes()
    assert need == 256 * 256 * 128 * 4 + 256 * 4  # contributions of up to 256 CTAs x 256 columns, then the flags
    # one CTA per SM (148 without a device) whenever each gets at least 4 units of 128 rows x 64 K
    assert mkpy.linear_tc_streamk_grid(16, 4096, 4096) == 148    # 32 tiles x 64 K blocks
    assert mkpy.linear_tc_streamk_grid(32, 4096, 24576) == 148   # 192 tiles: 1.3 waves of the plain kernel
    assert mkpy.linear_tc_streamk_grid(32, 4096, 28672) == 0     # 224 tiles: 1.5 waves, plain does as well
    assert mkpy.linear_tc_streamk_grid(5, 320, 200) == 2         # 10 units
    assert mkpy.linear_tc_streamk_grid(1, 128, 128) == 0         # 2 units: too few to share
    assert mkpy.linear_tc_streamk_grid(16, 4096, 128256) == 0    # 1002 tiles: many waves already
    assert mkpy.linear_tc_streamk_grid(16, 4096, 18944) == 0     # 148 tiles: exactly one wave
    assert mkpy.linear_tc_streamk_grid(256, 2048, 16384) == 0    # 256 columns, 128 tiles: plain
    assert mkpy.linear_tc_streamk_grid(256, 2048, 2048) == 128   # 256 columns, 16 tiles: stream-K
    assert lib.mk_linear_tc_streamk(None, d, d, 16, 4096, 4096, d, need, None) == _lib.MK_ERR_INVALID
    assert lib.mk_linear_tc_streamk(d, d, d, 16, 4096, 4096, None, need, None) == _lib.MK_ERR_INVALID
    assert lib.mk_linear_tc_streamk(d, d, d, 16, 4096, 4096, C.c_void_p(264), need, None) == _lib.MK_ERR_INVALID
    assert "aligned" in lib.mk_last_error(None).decode()
    assert lib.mk_linear_tc_streamk(d, d, d, 16, 4096, 4096, d, need - 1, None) == _lib.MK_ERR_INVALID
    assert "workspace needs" in lib.mk_last_error(None).decode()
    assert lib.mk_linear_tc_streamk(d, d, d, 16, 4000, 4096, d, need, None) == _lib.MK_ERR_UNSUPPORTED


def _fake_weights(n_layers, keep):
    """An mk_weights struct whose every pointer is a fake, aligned address (the
    host-side checks never dereference them)."""
    arrs = [(C.c_void_p * n_layers)(*([4096] * n_layers)) for _ in range(11)]
    keep.extend(arrs)
    return _lib.MkWeights(4096, 4096, 4096, *[C.cast(a, C.POINTER(C.c_void_p)) for a in arrs])


def test_tcdec_host_checks_need_no_device():
    lib = _lib.load()
    keep = []
    s = synth.LLAMA8B
    cfg = mkpy.make_config(s, 8, 520, "megakernel", 148)
    w = _fake_weights(s.n_layers, keep)
    dec = C.c_void_p()
    assert lib.mk_tcdec_create(C.byref(cfg), C.byref(w), C.byref(dec)) == _lib.MK_OK
    n = C.c_size_t()
    assert lib.mk_tcdec_workspace_bytes(dec, C.byref(n)) == _lib.MK_OK
    # x, hi/lo rows, the projection outputs (hi and lo rows each), q, attention out, scratch for 64 chunks,
    # then the step's own token, argmax, position and logits buffers
    B, H, I, V, QD, KD = 8, s.hidden, s.intermediate, s.vocab, s.n_heads * s.head_dim, s.n_kv_heads * s.head_dim
    floor = 4 * B * H + 2 * 2 * B * max(H, QD, I) + 4 * 2 * B * (QD + 2 * KD + H + 2 * I + V) + 2 * 4 * B * QD \
        + lib.mk_attention_scratch_bytes(B, s.n_heads, s.head_dim, 64) + 4 * B + 4 * B + 8 + 4 * B * V
    assert floor <= n.value <= floor + 18 * 256
    # a step before bind, and a bind with a misaligned workspace, are refused
    d = C.c_void_p(4096)
    assert lib.mk_tcdec_step(dec, d, 0, d, None, None) == _lib.MK_ERR_STATE
    assert lib.mk_tcdec_bind(dec, C.c_void_p(4096 + 16), d) == _lib.MK_ERR_INVALID
    assert "aligned" in lib.mk_tcdec_last_error(dec).decode()
    assert lib.mk_tcdec_destroy(dec) == _lib.MK_OK
    # shapes it does not take
    for bad, code in ((mkpy.make_config(s, 33, 520, "megakernel", 148), _lib.MK_ERR_UNSUPPORTED),
                      (mkpy.make_config(synth.TINY, 1, 96, "megakernel", 148), _lib.MK_ERR_UNSUPPORTED)):
        wt = _fake_weights(bad.n_layers, keep)
        assert lib.mk_tcdec_create(C.byref(bad), C.byref(wt), C.byref(dec)) == code
    assert "64" in lib.mk_tcdec_last_error(None).decode()  # tiny: intermediate 688 is not a multiple of 64
    # a null weight pointer
    w2 = _fake_weights(s.n_layers, keep)
    w2.final_norm = None
    assert lib.mk_tcdec_create(C.byref(cfg), C.byref(w2), C.byref(dec)) == _lib.MK_ERR_INVALID


def test_header_is_plain_c(tmp_path):
    """include/mk.h is a C header: no torch or C++ types cross the boundary."""
    src = tmp_path / "use_mk.c"
    src.write_text('#include "mk.h"\nint main(void) { mk_ctx *c = 0; mk_tcdec *d = 0; (void)c; (void)d;\n'
                   '  return (int)sizeof(mk_config) + (int)sizeof(mk_weights); }\n')
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), "-c",
                        str(src), "-o", str(tmp_path / "use_mk.o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_attention_chunk_rule_needs_no_device():
    # without a device the rule assumes 148 SMs
    ch = mkpy.attention_chunks
    assert ch(1, 8, 1025) == 18       # about one CTA per SM over the 8 (sequence, KV head) pairs
    assert ch(1, 8, 100) == 6         # at least 16 positions a chunk
    assert ch(3, 4, 1) == 1
    assert ch(16, 8, 1024) == 2       # 1024 positions: 2 chunks of 512 fill the slots best
    assert ch(16, 8, 16384) == 9      # long cache: 1152 CTAs, 97 % of the last of 4 waves of 2 per SM
    assert ch(4, 8, 32768) == 9       # 288 CTAs, one wave of 2 per SM
    assert ch(1, 8, 32768) == 34      # the first count whose wave is 90 % full: 272 of 296 slots
    assert ch(0, 8, 1024) == 0 and ch(1, 0, 1024) == 0 and ch(1, 8, 0) == 0
