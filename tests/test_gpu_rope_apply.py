"""GPU parity of rfa_rope_apply (the Rope operator on sin/cos tables) against
oracle.rope_apply, through the C ABI.

Bar: each output element within one rounding of the exact value, i.e.
|got - ref| <= 2^-8 |ref| (bf16 keeps 8 significant bits; 2^-10 for fp16)
plus 1e-5 for the fp32 arithmetic near zero.  KV-cache rows are compared
bit-exactly with the returned keys.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rfa():
    import rope_flashattention_b200 as m

    m.load_library()
    return m


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _close(got, ref, dtype):
    rel = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -10
    got = _f64(got)
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref)
    assert np.all(err <= rel * np.abs(ref) + 1e-5), f"max err {err.max():.3e}"


def _tables(rfa, T, D, seed, tab_dtype, interleaved):
    """sin/cos [T, D]: DynamicNTK tables for rotate-half pairs, the same angles
    repeated per adjacent pair for the interleaved variant."""
    lens = torch.tensor([T], dtype=torch.int32)
    g = workloads.gen(seed)
    pos = torch.randint(0, 20000, (T,), generator=g, dtype=torch.int32)
    inv = torch.from_numpy(oracle.inv_freq(10000.0, D).astype(np.float32))[None]
    s, c = rfa.rope_sincos(pos.cuda(), inv.cuda(), lens.cuda(), D, out_dtype=torch.float32)
    if interleaved:  # angle of pair i in columns 2i, 2i+1
        s = s[:, : D // 2].repeat_interleave(2, dim=1)
        c = c[:, : D // 2].repeat_interleave(2, dim=1)
    return s.to(tab_dtype).contiguous(), c.to(tab_dtype).contiguous()


def _ref_rows(x, s, c, inter, layout):
    """oracle on every (token, head) row of x with the token's table row"""
    s64, c64 = _f64(s), _f64(c)
    xs = _f64(x)
    if layout == "TND":
        T, H, D = xs.shape
        rows = np.repeat(np.arange(T), H)
        return oracle.rope_apply(xs.reshape(-1, D), s64, c64, rows, inter).reshape(T, H, D)
    B, H, S, D = xs.shape
    rows = (np.arange(B)[:, None, None] * S + np.arange(S)[None, None, :]).repeat(H, axis=1).reshape(-1)
    return oracle.rope_apply(xs.reshape(-1, D), s64, c64, rows, inter).reshape(B, H, S, D)


@pytest.mark.parametrize("io,tab,inter", [
    (torch.bfloat16, torch.float16, False),
    (torch.bfloat16, torch.float32, True),
    (torch.float16, torch.bfloat16, False),
    (torch.float16, torch.float16, True),
])
def test_tnd_gqa(rfa, io, tab, inter):
    T, Hq, Hkv, D = 300, 4, 2, 128
    q = workloads.randn16((T, Hq, D), 1, io).cuda()
    k = workloads.randn16((T, Hkv, D), 2, io).cuda()
    s, c = _tables(rfa, T, D, 3, tab, inter)
    qo, ko = rfa.rope_apply(q, k, s, c, interleaved=inter)
    assert rfa.get_device_status() == 0
    _close(qo, _ref_rows(q, s, c, inter, "TND"), io)
    _close(ko, _ref_rows(k, s, c, inter, "TND"), io)


@pytest.mark.parametrize("inter", [False, True])
def test_bnsd_d64_in_place(rfa, inter):
    B, Hq, Hkv, S, D = 2, 3, 1, 77, 64
    q = workloads.randn16((B, Hq, S, D), 4, torch.float16).cuda()
    k = workloads.randn16((B, Hkv, S, D), 5, torch.float16).cuda()
    s, c = _tables(rfa, B * S, D, 6, torch.float32, inter)
    rq, rk = _ref_rows(q, s, c, inter, "BNSD"), _ref_rows(k, s, c, inter, "BNSD")
    qo, ko = rfa.rope_apply(q, k, s, c, layout="BNSD", interleaved=inter, inplace=True)
    assert rfa.get_device_status() == 0
    assert qo.data_ptr() == q.data_ptr() and ko.data_ptr() == k.data_ptr()
    _close(q, rq, torch.float16)
    _close(k, rk, torch.float16)


def test_q_only_and_k_only(rfa):
    T, H, D = 33, 2, 32
    x = workloads.randn16((T, H, D), 7).cuda()
    s, c = _tables(rfa, T, D, 8, torch.float16, False)
    qo, ko = rfa.rope_apply(x, None, s, c)
    assert ko is None
    _close(qo, _ref_rows(x, s, c, False, "TND"), torch.bfloat16)
    qo2, ko2 = rfa.rope_apply(None, x, s, c)
    assert qo2 is None
    assert torch.equal(qo, ko2)
    assert rfa.get_device_status() == 0


def test_kv_cache_write(rfa):
    T, Hq, Hkv, D, rows = 64, 4, 2, 128, 100
    q = workloads.randn16((T, Hq, D), 9).cuda()
    k = workloads.randn16((T, Hkv, D), 10).cuda()
    s, c = _tables(rfa, T, D, 11, torch.float16, False)
    g = workloads.gen(12)
    slots = torch.randperm(rows, generator=g)[:T].to(torch.int32)
    slots[::7] = -1  # padding tokens: not cached
    cache = torch.full((rows, Hkv, D), 7.0, dtype=torch.bfloat16).cuda()
    before = cache.clone()
    qo, ko = rfa.rope_apply(q, k, s, c, cache_slots=slots.cuda(), k_cache=cache)
    assert rfa.get_device_status() == 0
    _close(ko, _ref_rows(k, s, c, False, "TND"), torch.bfloat16)
    sl = slots.numpy()
    for t in range(T):
        if sl[t] >= 0:
            assert torch.equal(cache[sl[t]], ko[t])
    untouched = np.setdiff1d(np.arange(rows), sl[sl >= 0])
    assert torch.equal(cache[untouched], before[untouched])
    # keys only to the cache
    cache2 = before.clone()
    qo2, ko2 = rfa.rope_apply(q, k, s, c, cache_slots=slots.cuda(), k_cache=cache2, keys_out=False)
    assert ko2 is None and torch.equal(cache2, cache) and torch.equal(qo2, qo)
    assert rfa.get_device_status() == 0


def test_cache_slot_out_of_range_sets_status(rfa):
    T, Hkv, D, rows = 8, 1, 64, 4
    k = workloads.randn16((T, Hkv, D), 13).cuda()
    s, c = _tables(rfa, T, D, 14, torch.float16, False)
    slots = torch.tensor([3, 1, 0, 2, 4, 9, -1, -5], dtype=torch.int32).cuda()  # 4 and 9 beyond the cache
    cache = torch.zeros((rows, Hkv, D), dtype=torch.bfloat16).cuda()
    _, ko = rfa.rope_apply(None, k, s, c, cache_slots=slots, k_cache=cache)
    assert rfa.get_device_status() == rfa.RFA_ERR_INVALID_ARG
    assert rfa.get_device_status() == 0  # read and cleared
    for t, r in enumerate([3, 1, 0, 2]):
        assert torch.equal(cache[r], ko[t])


def test_gqa_prefill_size(rfa):
    # 8192 tokens, 32 query and 8 kv heads, D 128: every row against the oracle
    T, Hq, Hkv, D = 8192, 32, 8, 128
    q = workloads.randn16((T, Hq, D), 15).cuda()
    k = workloads.randn16((T, Hkv, D), 16).cuda()
    s, c = _tables(rfa, T, D, 17, torch.float16, False)
    qo, ko = rfa.rope_apply(q, k, s, c)
    assert rfa.get_device_status() == 0
    _close(qo, _ref_rows(q, s, c, False, "TND"), torch.bfloat16)
    _close(ko, _ref_rows(k, s, c, False, "TND"), torch.bfloat16)


# ---------------------------------------------------------------- RMSNorm + RoPE + KV-cache write
@pytest.mark.parametrize("io,tab,inter,D", [
    (torch.bfloat16, torch.float16, False, 128),
    (torch.bfloat16, torch.float32, True, 64),
    (torch.float16, torch.bfloat16, False, 256),
])
def test_kv_rms_norm_rope_cache(rfa, io, tab, inter, D):
    T, Hkv, rows = 97, 4, 160
    k = (workloads.randn16((T, Hkv, D), 50, io).float() * 3.0).to(io).cuda()
    v = workloads.randn16((T, Hkv, D), 51, io).cuda()
    gamma = (0.5 + torch.rand(D, generator=workloads.gen(52))).float().cuda()
    s, c = _tables(rfa, T, D, 53, tab, inter)
    g = workloads.gen(54)
    slots = torch.randperm(rows, generator=g)[:T].to(torch.int32)
    slots[::5] = -1
    kc = torch.full((rows, Hkv, D), 3.0, dtype=io).cuda()
    vc = torch.full((rows, Hkv, D), -3.0, dtype=io).cuda()
    kc0, vc0 = kc.clone(), vc.clone()
    rfa.kv_rms_norm_rope_cache(k, v, gamma, 1e-6, s, c, slots.cuda(), kc, vc, interleaved=inter)
    assert rfa.get_device_status() == 0
    rk, rv = oracle.kv_rms_norm_rope_cache(_f64(k), _f64(v), gamma.double().cpu().numpy(), 1e-6, _f64(s), _f64(c),
                                           slots.numpy(), _f64(kc0), _f64(vc0), inter)
    _close(kc, rk, io)
    assert np.array_equal(_f64(vc), rv)  # values copied bit for bit (and untouched rows kept)


def test_kv_cache_op_slot_beyond_cache_sets_status(rfa):
    T, Hkv, D, rows = 4, 1, 64, 2
    k = workloads.randn16((T, Hkv, D), 55).cuda()
    v = workloads.randn16((T, Hkv, D), 56).cuda()
    s, c = _tables(rfa, T, D, 57, torch.float16, False)
    kc = torch.zeros((rows, Hkv, D), dtype=torch.bfloat16).cuda()
    vc = torch.zeros_like(kc)
    slots = torch.tensor([1, 2, 0, 7], dtype=torch.int32).cuda()
    rfa.kv_rms_norm_rope_cache(k, v, torch.ones(D).cuda(), 0.0, s, c, slots, kc, vc)
    assert rfa.get_device_status() == rfa.RFA_ERR_INVALID_ARG
    assert rfa.get_device_status() == 0
    assert torch.equal(vc[1], v[0]) and torch.equal(vc[0], v[2])


# ---------------------------------------------------------------- evict-first (streaming) launches
# A launch that moves more than half of L2 reads and writes its rows with the
# evict-first hint; the values must not change.  Each test runs one such launch
# and the same rows as many small launches (ordinary accesses) and compares
# the results bit for bit.

@pytest.mark.parametrize("inter", [False, True])
def test_rope_apply_streaming_launch_matches_small_launches(rfa, inter):
    T, Hq, Hkv, D, rows = 8192, 32, 8, 128, 9000
    q = workloads.randn16((T, Hq, D), 60).cuda()
    k = workloads.randn16((T, Hkv, D), 61).cuda()
    s, c = _tables(rfa, T, D, 62, torch.float16, inter)
    slots = torch.randperm(rows, generator=workloads.gen(63))[:T].to(torch.int32).cuda()
    cache = torch.zeros((rows, Hkv, D), dtype=torch.bfloat16).cuda()
    qo, ko = rfa.rope_apply(q, k, s, c, cache_slots=slots, k_cache=cache, interleaved=inter)
    assert rfa.get_device_status() == 0
    cache2 = torch.zeros_like(cache)
    for t0 in range(0, T, 512):
        sl = slice(t0, t0 + 512)
        qs, ks = rfa.rope_apply(q[sl].contiguous(), k[sl].contiguous(), s[sl].contiguous(), c[sl].contiguous(),
                                cache_slots=slots[sl].contiguous(), k_cache=cache2, interleaved=inter)
        assert torch.equal(qs, qo[sl]) and torch.equal(ks, ko[sl])
    assert rfa.get_device_status() == 0
    assert torch.equal(cache, cache2)


def test_kv_cache_op_streaming_launch_matches_small_launches(rfa):
    T, Hkv, D = 32768, 8, 128
    k = workloads.randn16((T, Hkv, D), 64).cuda()
    v = workloads.randn16((T, Hkv, D), 65).cuda()
    gamma = (0.5 + torch.rand(D, generator=workloads.gen(66))).float().cuda()
    s, c = _tables(rfa, T, D, 67, torch.float16, False)
    slots = torch.randperm(T, generator=workloads.gen(68)).to(torch.int32).cuda()
    kc, vc = torch.zeros_like(k), torch.zeros_like(v)
    rfa.kv_rms_norm_rope_cache(k, v, gamma, 1e-6, s, c, slots, kc, vc)
    assert rfa.get_device_status() == 0
    kc2, vc2 = torch.zeros_like(k), torch.zeros_like(v)
    for t0 in range(0, T, 1024):
        sl = slice(t0, t0 + 1024)
        rfa.kv_rms_norm_rope_cache(k[sl].contiguous(), v[sl].contiguous(), gamma, 1e-6, s[sl].contiguous(),
                                   c[sl].contiguous(), slots[sl].contiguous(), kc2, vc2)
    assert rfa.get_device_status() == 0
    assert torch.equal(kc, kc2) and torch.equal(vc, vc2)
