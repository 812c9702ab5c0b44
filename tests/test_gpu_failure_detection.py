"""Failure detection on the GPU without a GPU fault.

Two ways to make a kernel's bounded waits run out on purpose:
- rfa_set_hold_items: the attention kernels publish no work item, so every
  role waits on an item barrier that nothing arrives on (a flag that nothing
  sets) until the limit from rfa_set_wait_limit_ns runs out.  Deterministic.
- a 1 ns limit on a memory-bound call: any wait that mbarrier.try_wait could
  not absorb in its own suspend window (about 8,000 cycles on B200) runs out
  mid-pipeline, with copies and MMAs in flight that must be drained.
Either way the kernel must record RFA_ERR_TIMEOUT, stop its roles, drain and
return; afterwards the context must still be usable: with the defaults
restored, the same call gives the oracle's result.  Nothing here traps,
faults or hangs a GPU: every wait in the kernels is bounded, and the drains
before a CTA exits keep their own 2 s limit.
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


def _with_tiny_limit(rfa, call):
    try:
        rfa.set_wait_limit_ns(1)
        call()
        return rfa.get_device_status()
    finally:
        rfa.set_wait_limit_ns(0)  # back to the default, whatever happened


def _held(rfa, call):
    try:
        rfa.set_wait_limit_ns(2_000_000)  # 2 ms
        rfa.set_hold_items(True)
        call()
        return rfa.get_device_status()
    finally:
        rfa.set_hold_items(False)
        rfa.set_wait_limit_ns(0)


def test_fused_kernel_wait_runs_out_and_context_survives(rfa):
    B, Hq, Hkv, S, D = 2, 4, 2, 1024, 128
    q = workloads.randn16((B, Hq, S, D), 90).cuda()
    k = workloads.randn16((B, Hkv, S, D), 91).cuda()
    v = workloads.randn16((B, Hkv, S, D), 92).cuda()
    pos = torch.arange(S, dtype=torch.int32).repeat(B, 1).contiguous().cuda()
    assert rfa.get_device_status() == 0
    st = _held(rfa, lambda: rfa.fused_rope_attention(q, k, v, pos))
    assert st == rfa.RFA_ERR_TIMEOUT
    out = rfa.fused_rope_attention(q, k, v, pos)
    assert rfa.get_device_status() == 0
    inv = np.stack([oracle.inv_freq(10000.0, D)] * B)
    rows = np.array([[0, 0, 0], [1, 3, 1023], [0, 2, 517], [1, 1, 128]], np.int32)
    ref = oracle.attention_rows(q.cpu(), k.cpu(), v.cpu(), pos.cpu().numpy(), inv, rows)
    got = out.float().cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert np.abs(got - ref).max() <= 2e-2


def test_decode_held_items_run_out_and_context_survives(rfa):
    B, Hq, Hkv, Sq, D, L = 2, 8, 2, 1, 128, 2048
    q = workloads.randn16((B, Hq, Sq, D), 96).cuda()
    kc = workloads.randn16((B, L, Hkv, D), 97).cuda()
    vc = workloads.randn16((B, L, Hkv, D), 98).cuda()
    q_pos = torch.full((B, Sq), L - 1, dtype=torch.int32).cuda()
    lens = torch.full((B,), L, dtype=torch.int32).cuda()
    st = _held(rfa, lambda: rfa.decode_rope_attention(q, kc, vc, q_pos, lens))
    assert st == rfa.RFA_ERR_TIMEOUT
    out = rfa.decode_rope_attention(q, kc, vc, q_pos, lens)
    assert rfa.get_device_status() == 0
    ref = oracle.decode_attention(q.cpu(), kc.cpu(), vc.cpu(), q_pos.cpu().numpy(), [L] * B,
                                  np.stack([oracle.inv_freq(10000.0, D)] * B))
    assert np.abs(out.float().cpu().numpy() - ref).max() <= 2e-2


def test_decode_wait_runs_out_and_context_survives(rfa):
    # A wait only reaches its limit once mbarrier.try_wait has given up suspending, so the
    # case must have waits longer than that: 8 sequences of 16K cached tokens keep HBM busy
    # and the tile loads queue behind one another.  A few attempts, in case one call's
    # waits all completed inside the hardware's suspend window.
    B, Hq, Hkv, Sq, D, L = 8, 32, 8, 1, 128, 16384
    q = workloads.randn16((B, Hq, Sq, D), 93).cuda()
    kc = workloads.randn16((B, L, Hkv, D), 94).cuda()
    vc = workloads.randn16((B, L, Hkv, D), 95).cuda()
    q_pos = torch.full((B, Sq), L - 1, dtype=torch.int32).cuda()
    lens = torch.full((B,), L, dtype=torch.int32).cuda()
    sts = []
    for _ in range(3):
        sts.append(_with_tiny_limit(rfa, lambda: rfa.decode_rope_attention(q, kc, vc, q_pos, lens)))
        if sts[-1] != 0:
            break
    assert sts[-1] == rfa.RFA_ERR_TIMEOUT, sts
    out = rfa.decode_rope_attention(q, kc, vc, q_pos, lens)
    assert rfa.get_device_status() == 0
    ref = oracle.decode_attention(q.cpu(), kc.cpu(), vc.cpu(), q_pos.cpu().numpy(), [L] * B,
                                  np.stack([oracle.inv_freq(10000.0, D)] * B))
    assert np.abs(out.float().cpu().numpy() - ref).max() <= 2e-2
