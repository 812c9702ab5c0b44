"""The C-ABI library loads on a CPU-only box, exports every symbol that
include/rfa.h declares, and rejects invalid arguments on the host before any
CUDA call (no GPU needed for these paths)."""
import ctypes
import os
import re

import pytest
import torch

import rope_flashattention_b200 as rfa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from rope_flashattention_b200 import build

    build.build_library()
    return rfa.load_library()


def header_symbols():
    src = open(os.path.join(ROOT, "include", "rfa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rfa_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    syms = header_symbols()
    assert syms == sorted(rfa.EXPORTS)
    for name in ("rfa_rope_sincos", "rfa_fused_rope_attention"):
        assert name in syms


def test_every_declared_symbol_is_exported(lib):
    for name in header_symbols():
        assert hasattr(lib, name), name


def test_only_the_boundary_is_exported(lib):
    out = os.popen(f"nm -D --defined-only {rfa.LIB_PATH}").read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert {s for s in exported if s.startswith("rfa_")} == set(header_symbols())


def test_status_strings_and_version(lib):
    assert rfa.status_string(0) == "RFA_OK"
    assert rfa.status_string(5) == "RFA_ERR_TIMEOUT"
    assert rfa.status_string(99) == "RFA_ERR_UNKNOWN"
    assert lib.rfa_version() >= 100


def _p(**kw):
    p = rfa.AttnParams()
    p.B, p.Hq, p.Hkv, p.S, p.D, p.layout, p.causal = 1, 2, 2, 128, 64, 0, 1
    p.io_dtype, p.scale, p.rope_base = rfa.DT_BF16, 0.0, 10000.0
    p.ntk_enable, p.ntk_train_len, p.ntk_factor = 0, 0, 1.0
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_params_struct_matches_c_layout():
    assert ctypes.sizeof(rfa.AttnParams) == 64
    assert rfa.AttnParams.rope_base.offset == 40
    assert rfa.AttnParams.ntk_factor.offset == 56
    assert rfa.AttnParams.rope_interleaved.offset == 36


def _ru(x, a=256):
    return (x + a - 1) // a * a


# per-sequence seeds: flag/first position, the in-tile step (cos, sin) and the invFreq row
SEED_BYTES = 16 + 8 * 64 + 4 * 64
SCHED_BYTES = 256  # the attention kernel's two work counters


def test_workspace_size(lib):
    f = lib.rfa_fused_rope_attention_workspace
    # cos/sin table (D/2 fp16 cos + D/2 fp16 sin per token) + one seed block per sequence + counters
    assert f(ctypes.byref(_p()), 128) == _ru(128 * 64 * 2) + _ru(SEED_BYTES) + SCHED_BYTES
    assert f(ctypes.byref(_p(D=128, B=3)), 1000) == _ru(1000 * 128 * 2) + _ru(3 * SEED_BYTES) + SCHED_BYTES
    assert f(ctypes.byref(_p(D=96)), 128) == 0          # unsupported head dim
    assert f(ctypes.byref(_p(Hq=3, Hkv=2)), 128) == 0    # Hq % Hkv != 0
    assert f(ctypes.byref(_p(io_dtype=0)), 128) == 0     # UNDEFINED dtype
    assert f(ctypes.byref(_p()), 0) == 0


FAKE = ctypes.c_void_p(1 << 20)  # never dereferenced: every call below fails validation first


@pytest.mark.parametrize("kw,code", [
    (dict(io_dtype=0), rfa.RFA_ERR_INVALID_ARG),
    (dict(io_dtype=rfa.DT_FP32), rfa.RFA_ERR_UNSUPPORTED),
    (dict(D=96), rfa.RFA_ERR_UNSUPPORTED),
    (dict(D=63), rfa.RFA_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), rfa.RFA_ERR_INVALID_ARG),
    (dict(Hkv=0), rfa.RFA_ERR_INVALID_ARG),
    (dict(S=0), rfa.RFA_ERR_INVALID_ARG),
    (dict(layout=7), rfa.RFA_ERR_INVALID_ARG),
    (dict(layout=1, B=17), rfa.RFA_ERR_INVALID_ARG),
    (dict(rope_base=-1.0), rfa.RFA_ERR_INVALID_ARG),
    (dict(scale=-0.5), rfa.RFA_ERR_INVALID_ARG),
    (dict(ntk_enable=1, ntk_train_len=0), rfa.RFA_ERR_INVALID_ARG),
    (dict(ntk_enable=1, ntk_train_len=8, ntk_factor=0.5), rfa.RFA_ERR_INVALID_ARG),
    (dict(rope_interleaved=2), rfa.RFA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), rfa.RFA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), rfa.RFA_ERR_INVALID_ARG),
    (dict(rope_base=float("inf")), rfa.RFA_ERR_INVALID_ARG),
    (dict(B=0), rfa.RFA_ERR_INVALID_ARG),
    (dict(Hq=0), rfa.RFA_ERR_INVALID_ARG),
])
def test_attention_rejects_invalid_params(lib, kw, code):
    rc = lib.rfa_fused_rope_attention(ctypes.byref(_p(**kw)), FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE,
                                      1 << 30, None)
    assert rc == code


def test_attention_rejects_null_and_workspace(lib):
    p = _p()
    f = lib.rfa_fused_rope_attention
    assert f(ctypes.byref(p), None, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, 1 << 30, None) == rfa.RFA_ERR_INVALID_ARG
    assert f(ctypes.byref(p), FAKE, FAKE, FAKE, None, None, None, FAKE, FAKE, 1 << 30, None) == rfa.RFA_ERR_INVALID_ARG
    assert f(None, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, 1 << 30, None) == rfa.RFA_ERR_INVALID_ARG
    # misaligned q
    assert f(ctypes.byref(p), ctypes.c_void_p((1 << 20) + 2), FAKE, FAKE, FAKE, None, None, FAKE, FAKE, 1 << 30,
             None) == rfa.RFA_ERR_INVALID_ARG
    # workspace too small or missing
    assert f(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, 100, None) == rfa.RFA_ERR_WORKSPACE
    assert f(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, None, FAKE, None, 1 << 30, None) == rfa.RFA_ERR_WORKSPACE
    # packed layout: host lengths required and positive
    pt = _p(layout=1, B=2)
    assert f(ctypes.byref(pt), FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, 1 << 30, None) == rfa.RFA_ERR_INVALID_ARG
    lens = (ctypes.c_int32 * 2)(5, 0)
    assert f(ctypes.byref(pt), FAKE, FAKE, FAKE, FAKE, ctypes.cast(lens, ctypes.c_void_p), None, FAKE, FAKE, 1 << 30,
             None) == rfa.RFA_ERR_INVALID_ARG


@pytest.mark.parametrize("batch,ntok,hs,dt,code", [
    (1, 128, 64, rfa.DT_UNDEFINED, rfa.RFA_ERR_INVALID_ARG),   # UNDEFINED is not usable
    (1, 128, 48, rfa.DT_FP16, rfa.RFA_ERR_INVALID_ARG),        # headSize % 32
    (1, 128, 4096, rfa.DT_FP16, rfa.RFA_ERR_INVALID_ARG),      # headSize <= 2048
    (17, 128, 64, rfa.DT_FP16, rfa.RFA_ERR_INVALID_ARG),       # batch <= 16
    (0, 128, 64, rfa.DT_FP16, rfa.RFA_ERR_INVALID_ARG),
    (1, 256001, 64, rfa.DT_FP16, rfa.RFA_ERR_INVALID_ARG),     # ntokens <= 256000
    (1, 0, 64, rfa.DT_FP16, rfa.RFA_ERR_INVALID_ARG),
    (1, 128, 64, 9, rfa.RFA_ERR_INVALID_ARG),
])
def test_sincos_rejects_invalid_args(lib, batch, ntok, hs, dt, code):
    rc = lib.rfa_rope_sincos(FAKE, FAKE, FAKE, batch, ntok, hs, dt, FAKE, FAKE, None)
    assert rc == code


def test_sincos_rejects_null(lib):
    assert lib.rfa_rope_sincos(None, FAKE, FAKE, 1, 8, 64, rfa.DT_FP16, FAKE, FAKE, None) == rfa.RFA_ERR_INVALID_ARG
    assert lib.rfa_rope_sincos(FAKE, FAKE, FAKE, 1, 8, 64, rfa.DT_FP16, None, FAKE, None) == rfa.RFA_ERR_INVALID_ARG


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "rope_flashattention_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in txt.lower().replace("the oracle", ""), f


def test_binding_refuses_tensors_on_several_devices():
    """Every pointer of a call is read on one device; the binding refuses a
    call whose tensors sit on different GPUs (no compute, no GPU needed)."""
    d0, d1 = torch.device("cuda", 0), torch.device("cuda", 1)
    assert rfa._one_device([("q", d0), ("k", d0), ("v", d0)]) == d0
    with pytest.raises(ValueError, match="one GPU"):
        rfa._one_device([("q", d0), ("k", d0), ("out", d1)])
    with pytest.raises(ValueError):
        rfa._one_device([])
    with pytest.raises(TypeError, match="CUDA tensor"):
        rfa._same_device(q=torch.zeros(4), k=None)


def _ra(**kw):
    p = rfa.RopeApplyParams()
    p.layout, p.T, p.B, p.S, p.Hq, p.Hkv, p.D = rfa.LAYOUT_TND, 16, 0, 0, 2, 1, 64
    p.io_dtype, p.table_dtype, p.interleaved = rfa.DT_BF16, rfa.DT_FP16, 0
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_rope_apply_params_struct_matches_c_layout():
    assert ctypes.sizeof(rfa.RopeApplyParams) == 40
    assert rfa.RopeApplyParams.interleaved.offset == 36


MIS = ctypes.c_void_p(0x10002)  # not 16-byte aligned


@pytest.mark.parametrize("kw,code", [
    (dict(D=24), rfa.RFA_ERR_INVALID_ARG),            # D % 16
    (dict(D=528), rfa.RFA_ERR_INVALID_ARG),           # D <= 512
    (dict(D=0), rfa.RFA_ERR_INVALID_ARG),
    (dict(io_dtype=rfa.DT_FP32), rfa.RFA_ERR_UNSUPPORTED),
    (dict(io_dtype=rfa.DT_UNDEFINED), rfa.RFA_ERR_INVALID_ARG),
    (dict(table_dtype=rfa.DT_UNDEFINED), rfa.RFA_ERR_INVALID_ARG),
    (dict(interleaved=2), rfa.RFA_ERR_INVALID_ARG),
    (dict(T=0), rfa.RFA_ERR_INVALID_ARG),
    (dict(layout=rfa.LAYOUT_BNSD, B=2, S=0), rfa.RFA_ERR_INVALID_ARG),
    (dict(layout=7), rfa.RFA_ERR_INVALID_ARG),
    (dict(Hq=0), rfa.RFA_ERR_INVALID_ARG),            # q given without heads
    (dict(Hq=-1), rfa.RFA_ERR_INVALID_ARG),
])
def test_rope_apply_rejects_invalid_params(lib, kw, code):
    p = _ra(**kw)
    rc = lib.rfa_rope_apply(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 0, None)
    assert rc == code


def test_rope_apply_rejects_bad_pointers(lib):
    p = _ra()
    call = lambda *a: lib.rfa_rope_apply(ctypes.byref(p), *a, None)
    assert call(FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None, 0) == rfa.RFA_ERR_INVALID_ARG   # no sin
    assert call(FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None, 0) == rfa.RFA_ERR_INVALID_ARG   # no q_out
    assert call(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 0) == rfa.RFA_ERR_INVALID_ARG   # keys go nowhere
    assert call(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 8) == rfa.RFA_ERR_INVALID_ARG   # slots without cache
    assert call(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0) == rfa.RFA_ERR_INVALID_ARG   # cache of 0 rows
    assert call(FAKE, FAKE, MIS, FAKE, FAKE, FAKE, None, None, 0) == rfa.RFA_ERR_INVALID_ARG    # misaligned table
    assert call(FAKE, None, FAKE, FAKE, FAKE, FAKE, None, None, 0) == rfa.RFA_ERR_INVALID_ARG   # k heads, no k
    assert lib.rfa_rope_apply(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 0, None) == rfa.RFA_ERR_INVALID_ARG


def _kv(**kw):
    p = rfa.KvCacheParams(8, 2, 64, rfa.DT_BF16, rfa.DT_FP16, 0, 1e-6)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_kv_cache_params_struct_matches_c_layout():
    assert ctypes.sizeof(rfa.KvCacheParams) == 28
    assert rfa.KvCacheParams.eps.offset == 24


@pytest.mark.parametrize("kw,code", [
    (dict(D=48), rfa.RFA_ERR_INVALID_ARG),           # D a power of two
    (dict(D=8), rfa.RFA_ERR_INVALID_ARG),
    (dict(D=1024), rfa.RFA_ERR_INVALID_ARG),
    (dict(T=0), rfa.RFA_ERR_INVALID_ARG),
    (dict(Hkv=0), rfa.RFA_ERR_INVALID_ARG),
    (dict(eps=-1.0), rfa.RFA_ERR_INVALID_ARG),
    (dict(eps=float("nan")), rfa.RFA_ERR_INVALID_ARG),
    (dict(interleaved=3), rfa.RFA_ERR_INVALID_ARG),
    (dict(io_dtype=rfa.DT_FP32), rfa.RFA_ERR_UNSUPPORTED),
    (dict(table_dtype=rfa.DT_UNDEFINED), rfa.RFA_ERR_INVALID_ARG),
])
def test_kv_cache_rejects_invalid_params(lib, kw, code):
    p = _kv(**kw)
    assert lib.rfa_kv_rms_norm_rope_cache(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16,
                                          None) == code


def test_kv_cache_rejects_bad_pointers(lib):
    p = _kv()
    call = lambda *a: lib.rfa_kv_rms_norm_rope_cache(ctypes.byref(p), *a, None)
    assert call(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0) == rfa.RFA_ERR_INVALID_ARG      # no cache rows
    assert call(FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, 16) == rfa.RFA_ERR_INVALID_ARG     # no gamma
    assert call(FAKE, FAKE, MIS, FAKE, FAKE, FAKE, FAKE, FAKE, 16) == rfa.RFA_ERR_INVALID_ARG      # misaligned
    assert call(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 16) == rfa.RFA_ERR_INVALID_ARG     # no slots
    assert call(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 16) == rfa.RFA_ERR_INVALID_ARG     # no v cache


def _dp(**kw):
    p = rfa.DecodeParams(2, 8, 2, 1, 128, 1024, 1024, 1, rfa.DT_BF16, 0, 0.0, 0, 10000.0)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_decode_params_struct_matches_c_layout():
    assert ctypes.sizeof(rfa.DecodeParams) == 56
    assert rfa.DecodeParams.num_splits.offset == 44
    assert rfa.DecodeParams.rope_base.offset == 48


def test_decode_workspace_plans_splits(lib):
    # 2 x 2 kv groups over 1024 keys (8 tiles): split into single tiles -> 8 splits
    # (the workspace holds the split partials only: the kernel forms the queries' cos/sin itself)
    p = _dp()
    rq, D = 2 * 8 * 1, 128
    assert lib.rfa_decode_rope_attention_workspace(ctypes.byref(p)) == _ru(8 * rq * D * 4) + _ru(8 * rq * 2 * 4)
    # 128 x 8 groups: enough CTAs without splitting, so nothing but the 256-byte minimum
    p = _dp(B=128, Hq=32, Hkv=8, Sq=1)
    assert lib.rfa_decode_rope_attention_workspace(ctypes.byref(p)) == 256


def _decode_ws(lib, splits, **kw):
    p = _dp(**kw)
    rq = p.B * p.Hq * p.Sq
    want = max(256, _ru(splits * rq * p.D * 4) + _ru(splits * rq * 2 * 4) if splits > 1 else 0)
    return lib.rfa_decode_rope_attention_workspace(ctypes.byref(p)), want


def test_decode_plan_weighs_waves_against_cta_cost(lib):
    # Cost of a plan: waves x (tiles per split + 6), one CTA per SM on 148 SMs.
    # 8 x 8 kv groups over 32768 keys (256 tiles): 2 splits of 128 tiles, one wave of
    # 128 CTAs (cost 134), beat 4 of 64 (2 waves, 140), 9 of 29 (4 waves, 140) and 3 of
    # 86 (192 CTAs: 2 waves, 184)
    got, want = _decode_ws(lib, 2, B=8, Hq=32, Hkv=8, Sq=1, Smax=32768, max_kv_len=32768)
    assert got == want
    # one sequence, 8 kv groups over 256 tiles: 18 splits of 15 tiles fill one wave
    # (144 CTAs, cost 21); 37 of 7 take two (26), 9 of 29 one (35)
    got, want = _decode_ws(lib, 18, B=1, Hq=32, Hkv=8, Sq=1, Smax=32768, max_kv_len=32768)
    assert got == want
    # 32 x 8 groups over 4096 keys (32 tiles): no split (2 waves, 76) against 2 (4 waves, 88)
    got, want = _decode_ws(lib, 1, B=32, Hq=32, Hkv=8, Sq=1, Smax=4096, max_kv_len=4096)
    assert got == want


@pytest.mark.parametrize("n,splits", [(1, 1), (3, 3), (7, 4), (100, 8)])
def test_decode_num_splits_is_taken_as_given(lib, n, splits):
    # 1024 keys = 8 tiles, split into parts of ceil(8 / n) whole tiles: 7 asked -> parts of
    # 2 tiles -> 4 splits; more parts than tiles -> one tile each
    got, want = _decode_ws(lib, splits, num_splits=n)
    assert got == want


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=6, Hkv=4), rfa.RFA_ERR_INVALID_ARG),       # Hq % Hkv
    (dict(Sq=0), rfa.RFA_ERR_INVALID_ARG),
    (dict(max_kv_len=2048), rfa.RFA_ERR_INVALID_ARG),   # > Smax
    (dict(Sq=4, max_kv_len=3), rfa.RFA_ERR_INVALID_ARG),
    (dict(D=96), rfa.RFA_ERR_UNSUPPORTED),
    (dict(Hq=64, Hkv=1, Sq=4), rfa.RFA_ERR_UNSUPPORTED),  # G * Sq > 128
    (dict(io_dtype=rfa.DT_UNDEFINED), rfa.RFA_ERR_INVALID_ARG),
    (dict(rope_interleaved=2), rfa.RFA_ERR_INVALID_ARG),
    (dict(rope_base=0.0), rfa.RFA_ERR_INVALID_ARG),
    (dict(num_splits=-1), rfa.RFA_ERR_INVALID_ARG),
])
def test_decode_rejects_invalid_params(lib, kw, code):
    p = _dp(**kw)
    assert lib.rfa_decode_rope_attention_workspace(ctypes.byref(p)) == 0
    assert lib.rfa_decode_rope_attention(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 1 << 30,
                                         None) == code


def test_decode_rejects_null_and_workspace(lib):
    p = _dp()
    call = lambda *a: lib.rfa_decode_rope_attention(ctypes.byref(p), *a, None)
    assert call(FAKE, FAKE, FAKE, None, FAKE, None, FAKE, FAKE, 1 << 30) == rfa.RFA_ERR_INVALID_ARG   # no q_pos
    assert call(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 16) == rfa.RFA_ERR_WORKSPACE          # too small
    assert call(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, 1 << 30) == rfa.RFA_ERR_WORKSPACE     # none
