"""The attention epilogue's two store paths give identical results.

With every sequence's positions consecutive and D = 128, whole output tiles
are staged in shared memory and written by TMA stores; tiles that run past a
sequence's end, and launches with other positions, are stored row by row (32-
byte stores when the output is 32-byte aligned, 16-byte ones otherwise).
Both paths write the same rounded values, so an output placed 16 bytes into a
larger buffer (16-byte but not 32-byte aligned) must equal, bit for bit, the
output of the same call into a fresh tensor, and the buffer's guard elements
around it must stay untouched.
"""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rfa():
    import rope_flashattention_b200 as m

    m.load_library()
    return m


def _offset_out(like, guard=8):
    """A tensor shaped like `like`, starting `guard` elements (16 bytes) into a
    buffer whose first and last `guard` elements hold a sentinel."""
    n = like.numel()
    buf = torch.full((n + 2 * guard,), -7.0, dtype=like.dtype, device=like.device)
    return buf, buf[guard:guard + n].view(like.shape)


def _check(rfa, q, k, v, pos, **kw):
    ref = rfa.fused_rope_attention(q, k, v, pos, **kw)
    buf, out = _offset_out(ref)
    assert out.data_ptr() % 16 == 0 and out.data_ptr() % 32 != 0
    got = rfa.fused_rope_attention(q, k, v, pos, out=out, **kw)
    torch.cuda.synchronize()
    assert rfa.get_device_status() == 0
    assert torch.equal(got, ref)
    assert torch.all(buf[:8] == -7.0) and torch.all(buf[-8:] == -7.0)


def test_bnsd_whole_tiles_misaligned_out(rfa):
    B, Hq, Hkv, S, D = 2, 8, 2, 640, 128
    q = workloads.randn16((B, Hq, S, D), 301).cuda()
    k = workloads.randn16((B, Hkv, S, D), 302).cuda()
    v = workloads.randn16((B, Hkv, S, D), 303).cuda()
    pos = torch.arange(S, dtype=torch.int32).repeat(B, 1).contiguous().cuda()
    _check(rfa, q, k, v, pos)


def test_packed_ragged_tiles_misaligned_out(rfa):
    lens = [300, 129, 512, 77]  # ragged last tiles: row stores there, TMA stores elsewhere
    T, Hq, Hkv, D = sum(lens), 8, 2, 128
    q = workloads.randn16((T, Hq, D), 311).cuda()
    k = workloads.randn16((T, Hkv, D), 312).cuda()
    v = workloads.randn16((T, Hkv, D), 313).cuda()
    pos = torch.cat([torch.arange(n, dtype=torch.int32) for n in lens]).cuda()
    _check(rfa, q, k, v, pos, layout="TND", seq_lens=lens)


def test_non_consecutive_positions_misaligned_out(rfa):
    # a break in the positions: the whole launch stores rows (16-byte stores here)
    B, Hq, Hkv, S, D = 1, 4, 2, 384, 128
    q = workloads.randn16((B, Hq, S, D), 321).cuda()
    k = workloads.randn16((B, Hkv, S, D), 322).cuda()
    v = workloads.randn16((B, Hkv, S, D), 323).cuda()
    pos = torch.arange(S, dtype=torch.int32)
    pos[200:] += 50
    pos = pos.repeat(B, 1).contiguous().cuda()
    _check(rfa, q, k, v, pos)
