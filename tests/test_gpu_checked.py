"""The bounds-checked build (librfa_checked.so, compiled with -DRFA_CHECKED).

Every computed global-memory index, shared-memory offset, TMA coordinate and
segment offset in the kernels is tested before use there; a failed test
records RFA_ERR_INVALID_ARG in the device status word (and the access is
skipped), instead of trapping.  These tests run the small, ragged and packed
cases of the fused kernel, the sin/cos table, the Rope operator with a cache
write, the cache op and decode (split and merged) through that build: every
call must leave the status word at RFA_OK and match the fp64 oracle within
the usual tolerances (max abs 2e-2, relative Frobenius 5e-3; sin/cos 2e-3).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu
MAX_ABS = 2e-2
REL_FRO = 5e-3


@pytest.fixture(scope="module")
def rfa():
    import rope_flashattention_b200 as m

    m.load_library()
    with m.use_library(m.CHECKED_LIB_PATH):
        yield m


def _compare(got, ref):
    got = np.asarray(got, np.float64)
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref).max()
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err <= MAX_ABS and fro <= REL_FRO, (err, fro)


def _inv(B, D, base, lens=None, ntk=None):
    rows = []
    for b in range(B):
        bb = base if ntk is None else oracle.ntk_base(base, D, int(lens[b]), ntk[0], ntk[1])
        rows.append(oracle.inv_freq(bb, D))
    return np.stack(rows)


def test_checked_build_is_loaded(rfa):
    import ctypes

    lib = rfa.load_library()
    assert lib._name.endswith("librfa_checked.so")
    assert isinstance(lib.rfa_version(), int)
    del ctypes


@pytest.mark.parametrize("B,Hq,Hkv,S,D,seed", [(1, 2, 2, 128, 64, 1), (2, 4, 2, 129, 128, 2), (1, 6, 2, 520, 128, 3),
                                               (1, 6, 3, 77, 64, 4)])
@pytest.mark.parametrize("interleaved", [False, True])
def test_bnsd_small_and_ragged(rfa, B, Hq, Hkv, S, D, seed, interleaved):
    q = workloads.randn16((B, Hq, S, D), seed)
    k = workloads.randn16((B, Hkv, S, D), seed + 1)
    v = workloads.randn16((B, Hkv, S, D), seed + 2)
    pos = torch.arange(S, dtype=torch.int32).repeat(B, 1).contiguous()
    out = rfa.fused_rope_attention(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), layout="BNSD", interleaved=interleaved)
    assert rfa.get_device_status() == rfa.RFA_OK
    ref = oracle.attention_full(q, k, v, pos.numpy(), _inv(B, D, 10000.0), interleaved=interleaved)
    _compare(out.float().cpu().numpy(), ref)


def test_bnsd_arbitrary_positions_table_path(rfa):
    B, Hq, Hkv, S, D = 2, 4, 2, 300, 128
    g = workloads.gen(11)
    pos = torch.randint(-5000, 90000, (B, S), generator=g, dtype=torch.int32)
    q = workloads.randn16((B, Hq, S, D), 12)
    k = workloads.randn16((B, Hkv, S, D), 13)
    v = workloads.randn16((B, Hkv, S, D), 14)
    out = rfa.fused_rope_attention(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), layout="BNSD")
    assert rfa.get_device_status() == rfa.RFA_OK
    ref = oracle.attention_full(q, k, v, pos.numpy(), _inv(B, D, 10000.0))
    _compare(out.float().cpu().numpy(), ref)


@pytest.mark.parametrize("lens,Hq,Hkv,D,ntk", [([1, 127, 128, 129, 300, 5], 4, 2, 128, None),
                                               ([64, 1, 200], 2, 2, 64, None),
                                               ([100, 700, 300], 4, 1, 128, (256, 2.0))])
def test_packed_sequences(rfa, lens, Hq, Hkv, D, ntk):
    T = sum(lens)
    q = workloads.randn16((T, Hq, D), 20)
    k = workloads.randn16((T, Hkv, D), 21)
    v = workloads.randn16((T, Hkv, D), 22)
    pos = torch.cat([torch.arange(n, dtype=torch.int32) for n in lens])
    kw = dict(layout="TND", seq_lens=lens)
    if ntk:
        kw.update(ntk_train_len=ntk[0], ntk_factor=ntk[1])
    out = rfa.fused_rope_attention(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), **kw)
    assert rfa.get_device_status() == rfa.RFA_OK
    ref = oracle.attention_full(q, k, v, pos.numpy(), _inv(len(lens), D, 10000.0, lens, ntk), layout=oracle.TND,
                                seq_lens=lens)
    _compare(out.float().cpu().numpy(), ref)


def test_sincos_table(rfa):
    pos, inv, lens = workloads.sincos_problem(1000, 128, 5, seed=30)
    s, c = rfa.rope_sincos(pos.cuda(), inv.cuda(), lens.cuda(), 128, out_dtype=torch.float16)
    assert rfa.get_device_status() == rfa.RFA_OK
    rs, rc = oracle.rope_sincos(pos.numpy(), inv.double().numpy(), lens.numpy(), 128)
    assert np.abs(s.float().cpu().numpy() - rs).max() <= 2e-3
    assert np.abs(c.float().cpu().numpy() - rc).max() <= 2e-3


def test_rope_apply_cache_write_and_kv_cache_op(rfa):
    T, Hq, Hkv, D = 300, 4, 2, 128
    pos = torch.arange(T, dtype=torch.int32)
    inv = torch.from_numpy(oracle.inv_freq(10000.0, D).astype(np.float32))[None]
    s, c = rfa.rope_sincos(pos.cuda(), inv.cuda(), torch.tensor([T], dtype=torch.int32).cuda(), D,
                           out_dtype=torch.float16)
    q = workloads.randn16((T, Hq, D), 40).cuda()
    k = workloads.randn16((T, Hkv, D), 41).cuda()
    slots = torch.randperm(T, generator=workloads.gen(42)).to(torch.int32).cuda()
    cache = torch.zeros((T, Hkv, D), dtype=k.dtype, device="cuda")
    qo, ko = rfa.rope_apply(q, k, s, c, cache_slots=slots, k_cache=cache)
    assert rfa.get_device_status() == rfa.RFA_OK
    assert torch.equal(cache[slots.long()], ko)
    rs, rc = s.double().cpu().numpy(), c.double().cpu().numpy()
    ref_q = oracle.rope_apply(q.float().cpu().numpy().reshape(-1, D), rs, rc, np.repeat(np.arange(T), Hq))
    assert np.abs(qo.float().cpu().numpy().reshape(-1, D) - ref_q).max() <= 2e-2
    v = workloads.randn16((T, Hkv, D), 43).cuda()
    gamma = torch.rand(D, generator=workloads.gen(44)).cuda()
    kc, vc = torch.zeros_like(cache), torch.zeros_like(cache)
    rfa.kv_rms_norm_rope_cache(k, v, gamma, 1e-6, s, c, slots, kc, vc)
    assert rfa.get_device_status() == rfa.RFA_OK
    assert torch.equal(vc[slots.long()], v)


@pytest.mark.parametrize("lens,Smax,splits", [([1000, 3001], 4096, 0), ([300, 700], 1024, 1)])
def test_decode(rfa, lens, Smax, splits):
    B, Hq, Hkv, Sq, D = len(lens), 32, 8, 1, 128
    q = workloads.randn16((B, Hq, Sq, D), 50)
    kc = workloads.randn16((B, Smax, Hkv, D), 51)
    vc = workloads.randn16((B, Smax, Hkv, D), 52)
    q_pos = torch.tensor([[L - 1] for L in lens], dtype=torch.int32)
    out = rfa.decode_rope_attention(q.cuda(), kc.cuda(), vc.cuda(), q_pos.cuda(),
                                    torch.tensor(lens, dtype=torch.int32).cuda(), num_splits=splits)
    assert rfa.get_device_status() == rfa.RFA_OK
    ref = oracle.decode_attention(q, kc, vc, q_pos.numpy(), lens, np.stack([oracle.inv_freq(10000.0, D)] * B))
    _compare(out.float().cpu().numpy(), ref)
