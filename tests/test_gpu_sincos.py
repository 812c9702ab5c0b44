"""GPU parity of rfa_rope_sincos against the fp64 oracle (through the C ABI).

Tolerance: max abs error <= 2e-3 for fp16/bf16/fp32 outputs.  The duplicated
halves and the segment indexing are checked exactly.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.fixture(scope="module")
def rfa():
    import rope_flashattention_b200 as m

    m.load_library()
    return m


def _run(rfa, pos, inv, lens, D, dtype):
    s, c = rfa.rope_sincos(pos.cuda(), inv.cuda(), lens.cuda(), D, out_dtype=dtype)
    assert rfa.get_device_status() == 0
    return s, c


def _check(rfa, pos, inv, lens, D, dtype, rows=None):
    s, c = _run(rfa, pos, inv, lens, D, dtype)
    s, c = s.float().cpu().numpy(), c.float().cpu().numpy()
    np.testing.assert_array_equal(s[:, : D // 2], s[:, D // 2:])
    np.testing.assert_array_equal(c[:, : D // 2], c[:, D // 2:])
    if rows is None:
        rs, rc = oracle.rope_sincos(pos.numpy(), inv.double().numpy(), lens.numpy(), D)
        gs, gc = s, c
    else:
        # oracle on the sampled tokens only: a one-token "batch" per row
        seg = np.repeat(np.arange(len(lens)), lens.numpy())
        rs, rc = oracle.rope_sincos(pos.numpy()[rows], inv.double().numpy()[seg[rows]],
                                    np.ones(len(rows), np.int32), D)
        gs, gc = s[rows], c[rows]
    assert np.abs(gs - rs).max() <= TOL
    assert np.abs(gc - rc).max() <= TOL
    return s, c


def test_tiny_fp32_table(rfa):
    pos = torch.arange(128, dtype=torch.int32)
    inv = torch.from_numpy(oracle.inv_freq(10000.0, 64).astype(np.float32))[None]
    s, c = _check(rfa, pos, inv, torch.tensor([128], dtype=torch.int32), 64, torch.float32)
    assert np.all(s[0] == 0) and np.all(c[0] == 1)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
def test_ragged_batches(rfa, dtype):
    lens = torch.tensor([1, 31, 200, 7, 64], dtype=torch.int32)
    pos, inv, _ = workloads.sincos_problem(int(lens.sum()), 128, 5, seed=11)
    pos = torch.cat([torch.arange(int(n), dtype=torch.int32) * 3 - 40 for n in lens])  # negative positions too
    _check(rfa, pos, inv, lens, 128, dtype)


@pytest.mark.parametrize("hs", [32, 96, 2048])
def test_head_sizes(rfa, hs):
    pos, inv, lens = workloads.sincos_problem(300, hs, 3, seed=hs)
    _check(rfa, pos, inv, lens, hs, torch.float16)


def test_packed_workload_fp16(rfa):
    w = workloads.PACKED
    lens = workloads.packed_lengths(w)
    pos = workloads.positions(w)
    inv = workloads.random_inv_freq(w)
    _check(rfa, pos, inv, lens, w.D, torch.float16)


def test_ceiling_shape_sampled(rfa):
    pos, inv, lens = workloads.sincos_problem(256000, 128, 16, seed=7)
    rows = np.random.default_rng(0).choice(256000, 4000, replace=False)
    rows = np.concatenate([rows, [0, 15999, 16000, 255999]])
    _check(rfa, pos, inv, lens, 128, torch.float16, rows=rows)


def test_large_angles_fp32_accuracy(rfa):
    """Angles up to 1e6 rad (positions up to +-1e6, frequencies in [0.5, 1]):
    the angle is reduced by 2 pi with the fp32 product's rounding error carried
    along, so fp32 outputs stay within 2e-6 of the exact values (rounding the
    product to fp32 alone would err by up to 3e-2 here)."""
    g = workloads.gen(17)
    T, D = 4096, 64
    pos = torch.randint(-1000000, 1000001, (T,), generator=g, dtype=torch.int32)
    inv = 0.5 + 0.5 * torch.rand(1, D // 2, generator=g, dtype=torch.float32)
    lens = torch.tensor([T], dtype=torch.int32)
    s, c = _run(rfa, pos, inv, lens, D, torch.float32)
    rs, rc = oracle.rope_sincos(pos.numpy(), inv.double().numpy(), lens.numpy(), D)
    assert np.abs(s.cpu().numpy() - rs).max() <= 2e-6
    assert np.abs(c.cpu().numpy() - rc).max() <= 2e-6


def test_segment_indexing_exact(rfa):
    # row b of invFreq = 2^-(b+1): each token's angle identifies its batch exactly
    lens = torch.tensor([3, 9, 1, 20], dtype=torch.int32)
    pos = torch.cat([torch.arange(int(n), dtype=torch.int32) + 1 for n in lens])
    inv = torch.stack([torch.full((16,), 2.0 ** -(b + 1)) for b in range(4)])
    s, c = _run(rfa, pos, inv, lens, 32, torch.float32)
    seg = np.repeat(np.arange(4), lens.numpy())
    ang = pos.numpy() * 2.0 ** -(seg + 1.0)
    np.testing.assert_allclose(s.cpu().numpy()[:, 0], np.sin(ang), atol=1e-6)
    np.testing.assert_allclose(c.cpu().numpy()[:, 0], np.cos(ang), atol=1e-6)


def test_bad_lengths_set_status_and_write_nothing(rfa):
    pos = torch.zeros(10, dtype=torch.int32).cuda()
    inv = torch.zeros(2, 16).cuda()
    s = torch.full((10, 32), 7.0, device="cuda")
    c = torch.full((10, 32), 7.0, device="cuda")
    rfa.rope_sincos(pos, inv, torch.tensor([4, 5], dtype=torch.int32).cuda(), 32, torch.float32, s, c)
    assert rfa.get_device_status() == rfa.RFA_ERR_INVALID_ARG
    assert torch.all(s == 7.0) and torch.all(c == 7.0)
    assert rfa.get_device_status() == 0  # cleared


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_tables_larger_than_half_of_l2(rfa, dtype):
    """Tables larger than half of L2 are written with evict-first stores: within
    tolerance of the oracle on sampled rows, and bit-identical to the ordinary
    stores of a small launch over the first sequence alone."""
    pos, inv, lens = workloads.sincos_problem(256000, 128, 16, seed=9)
    rows = np.random.default_rng(1).choice(256000, 3000, replace=False)
    rows = np.concatenate([rows, [0, 15999, 16000, 255999]])
    s, c = _check(rfa, pos, inv, lens, 128, dtype, rows=rows)
    n0 = int(lens[0])
    s0, c0 = _run(rfa, pos[:n0], inv[:1], lens[:1], 128, dtype)
    np.testing.assert_array_equal(s[:n0], s0.float().cpu().numpy())
    np.testing.assert_array_equal(c[:n0], c0.float().cpu().numpy())
