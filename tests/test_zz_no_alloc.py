"""The workspace-free entry point, rfa_fused_rope_attention_noalloc.

It exists for callers that cannot allocate device memory where they call the
library -- code running during CUDA-graph stream capture, plugins whose host
framework owns all device buffers and hands a kernel only its inputs and
outputs, real-time callers that must not block on an allocator.  Instead of a
caller workspace it uses a fixed scratch area inside the library's module.

The test calls it through the C ABI twice in a row and checks each result
against the workspace entry point, rfa_fused_rope_attention.  Both run the
same kernels on the same inputs, so the outputs must agree bit for bit
(stricter than the attention tolerances of the oracle parity tests, max abs
2e-2 and relative Frobenius 5e-3).  The second call checks that the scratch
left over from the first call does not matter.  Also checks that a problem larger than the fixed
scratch is refused before anything runs.  Kept in a file of its own that
pytest collects last.
"""
import ctypes

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rfa():
    import rope_flashattention_b200 as m

    m.load_library()
    return m


def _same(a, b):
    assert torch.isfinite(a.float()).all()
    assert torch.equal(a, b), f"max abs difference {(a.float() - b.float()).abs().max().item():.3e}"


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(rfa, p, q, k, v, pos, lens, out):
    lens_arr = None if lens is None else ctypes.cast((ctypes.c_int32 * len(lens))(*lens), ctypes.c_void_p)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return rfa.load_library().rfa_fused_rope_attention_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(pos),
                                                               lens_arr, None, _ptr(out), stream)


def test_noalloc_matches_workspace_entry_point_twice(rfa):
    B, Hq, Hkv, S, D = 2, 4, 2, 300, 128
    q = workloads.randn16((B, Hq, S, D), 70).cuda()
    k = workloads.randn16((B, Hkv, S, D), 71).cuda()
    v = workloads.randn16((B, Hkv, S, D), 72).cuda()
    pos = torch.arange(S, dtype=torch.int32).repeat(B, 1).contiguous().cuda()
    ref = rfa.fused_rope_attention(q, k, v, pos, layout="BNSD", rope_base=10000.0)
    assert rfa.get_device_status() == 0
    p = rfa._params(q, k, "BNSD", None, True, None, 10000.0, 0, 1.0)
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        assert _call_noalloc(rfa, p, q, k, v, pos, None, out) == rfa.RFA_OK
        assert rfa.get_device_status() == 0
        _same(out, ref)


def test_noalloc_packed_sequences_twice(rfa):
    lens = [5, 200, 129, 64]
    T, Hq, Hkv, D = sum(lens), 4, 1, 64
    q = workloads.randn16((T, Hq, D), 80).cuda()
    k = workloads.randn16((T, Hkv, D), 81).cuda()
    v = workloads.randn16((T, Hkv, D), 82).cuda()
    pos = torch.cat([torch.arange(n, dtype=torch.int32) * 2 + 7 for n in lens]).cuda()  # not consecutive
    kw = dict(layout="TND", seq_lens=lens, rope_base=10000.0, ntk_train_len=100, ntk_factor=2.0)
    ref = rfa.fused_rope_attention(q, k, v, pos, **kw)
    assert rfa.get_device_status() == 0
    p = rfa._params(q, k, "TND", lens, True, None, 10000.0, 100, 2.0)
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        assert _call_noalloc(rfa, p, q, k, v, pos, lens, out) == rfa.RFA_OK
        assert rfa.get_device_status() == 0
        _same(out, ref)


def test_noalloc_refuses_problems_beyond_its_scratch(rfa):
    # 65537 tokens > the fixed scratch's 65536: refused on the host, nothing enqueued.
    B, Hq, S, D = 1, 1, 65537, 128
    q = torch.zeros((B, Hq, S, D), dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros((B, S), dtype=torch.int32, device="cuda")
    p = rfa._params(q, q, "BNSD", None, True, None, 10000.0, 0, 1.0)
    out = torch.empty_like(q)
    assert _call_noalloc(rfa, p, q, q, q, pos, None, out) == rfa.RFA_ERR_WORKSPACE
    assert rfa.get_device_status() == 0
