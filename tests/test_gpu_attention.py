"""GPU parity of rfa_fused_rope_attention against the fp64 oracle.

Each case runs the CUDA path through the C ABI on seeded inputs and compares
it element by element with the oracle: in full at sizes that span several
128-row tiles and a ragged tail, and on seeded row samples at the full
workload sizes.  Bar (fp16/bf16 I/O): max abs error <= 2e-2 and relative
Frobenius error <= 5e-3.
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
    return m


def _inv_rows(B, D, base, lens=None, ntk=None):
    rows = []
    for b in range(B):
        bb = base
        if ntk is not None:
            L, f = ntk
            bb = oracle.ntk_base(base, D, int(lens[b]), L, f)
        rows.append(oracle.inv_freq(bb, D))
    return np.stack(rows)


def _compare(got, ref):
    got = np.asarray(got, np.float64)
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref)
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err.max() <= MAX_ABS, f"max abs {err.max():.3e}"
    assert fro <= REL_FRO, f"rel fro {fro:.3e}"
    return err.max(), fro


def run_bnsd(rfa, B, Hq, Hkv, S, D, *, seed=0, base=10000.0, causal=True, dtype=torch.bfloat16, ntk=None,
             pos=None, inv=None, scale=None, interleaved=False):
    q = workloads.randn16((B, Hq, S, D), seed, dtype)
    k = workloads.randn16((B, Hkv, S, D), seed + 1, dtype)
    v = workloads.randn16((B, Hkv, S, D), seed + 2, dtype)
    if pos is None:
        pos = torch.arange(S, dtype=torch.int32).repeat(B, 1).contiguous()
    kw = dict(layout="BNSD", causal=causal, rope_base=base, scale=scale, interleaved=interleaved)
    if ntk is not None:
        kw.update(ntk_train_len=ntk[0], ntk_factor=ntk[1])
    if inv is not None:
        kw["inv_freq"] = inv.cuda()
    out = rfa.fused_rope_attention(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), **kw)
    assert rfa.get_device_status() == 0
    inv_rows = inv.double().numpy() if inv is not None else _inv_rows(B, D, base, [S] * B, ntk)
    return q, k, v, pos, inv_rows, out.float().cpu().numpy()


def full_bnsd(rfa, B, Hq, Hkv, S, D, **kw):
    q, k, v, pos, inv, got = run_bnsd(rfa, B, Hq, Hkv, S, D, **kw)
    ref = oracle.attention_full(q, k, v, pos.numpy(), inv, causal=kw.get("causal", True), scale=kw.get("scale"),
                                interleaved=kw.get("interleaved", False))
    return _compare(got, ref)


def test_tiny_workload(rfa):
    w = workloads.TINY
    full_bnsd(rfa, w.B, w.Hq, w.Hkv, w.S, w.D, seed=w.seed, base=w.rope_base)


@pytest.mark.parametrize("S", [1, 5, 127, 128, 129, 300, 640])
def test_ragged_lengths_d128_gqa(rfa, S):
    full_bnsd(rfa, 2, 4, 2, S, 128, seed=S)


@pytest.mark.parametrize("S", [1, 77, 256, 383])
def test_ragged_lengths_d64(rfa, S):
    full_bnsd(rfa, 1, 6, 3, S, 64, seed=100 + S)


@pytest.mark.parametrize("D", [64, 128])
def test_non_causal(rfa, D):
    full_bnsd(rfa, 2, 2, 1, 333, D, seed=7, causal=False)


@pytest.mark.parametrize("D", [64, 128])
def test_fp16_io(rfa, D):
    full_bnsd(rfa, 1, 4, 4, 260, D, seed=9, dtype=torch.float16)


def test_odd_group_size_pairs_query_tiles(rfa):
    # G = 3 and an odd number of query tiles: the last work item has one tile
    full_bnsd(rfa, 1, 6, 2, 520, 128, seed=17)


@pytest.mark.parametrize("dtype,causal,zero_pos", [(torch.bfloat16, True, True), (torch.float16, False, False)])
def test_running_max_jumps_within_later_tiles(rfa, dtype, causal, zero_pos):
    """A few keys far larger than the rest make the row maximum jump by much
    more than 2^8 inside later key tiles, in different 32-key chunks (keys
    300, 420, 500, 520, 690: chunks 1, 1, 3, 0, 1 of tiles 2, 3, 3, 4, 5), so
    the part of the tile already exponentiated, the row sum and O must be
    rescaled mid-tile.  The large keys share one value row: how the weight
    splits among them (sensitive to the rounding of the rotated keys at such
    scores) then does not move the output.  The bf16 case puts every token
    at position 0, where the rotation is exactly the identity, so that the
    scores carry no rounding of rotated operands (bf16 keeps 8 bits, and at
    scores of ~10 that alone moves the weights of keys near the maximum)."""
    B, Hq, Hkv, S, D = 1, 2, 1, 700, 128
    big = ((300, 14.0), (420, 20.0), (500, 28.0), (520, 36.0), (690, 50.0))
    q = workloads.randn16((B, Hq, S, D), 91, dtype)
    k = workloads.randn16((B, Hkv, S, D), 92, dtype).float()
    v = workloads.randn16((B, Hkv, S, D), 93, dtype)
    for t, f in big:
        k[:, :, t] *= f
        v[:, :, t] = v[:, :, big[0][0]]
    k = k.to(dtype)
    pos = torch.arange(S, dtype=torch.int32).repeat(B, 1).contiguous()
    if zero_pos:
        pos.zero_()
    out = rfa.fused_rope_attention(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), layout="BNSD", causal=causal,
                                   rope_base=10000.0)
    assert rfa.get_device_status() == 0
    ref = oracle.attention_full(q, k, v, pos.numpy(), _inv_rows(B, D, 10000.0), causal=causal)
    _compare(out.float().cpu().numpy(), ref)


@pytest.mark.parametrize("D,S,dtype", [(128, 300, torch.bfloat16), (64, 257, torch.bfloat16), (128, 200, torch.float16)])
def test_adjacent_pairs(rfa, D, S, dtype):
    # RoPE on pairs (2i, 2i+1): recurrence path (consecutive positions)
    full_bnsd(rfa, 2, 4, 2, S, D, seed=200 + D, dtype=dtype, interleaved=True)


def test_adjacent_pairs_arbitrary_positions(rfa):
    # table path (positions not consecutive)
    B, S, D = 1, 290, 128
    g = workloads.gen(23)
    pos = torch.randint(-5000, 90000, (B, S), generator=g, dtype=torch.int32)
    full_bnsd(rfa, B, 6, 3, S, D, seed=24, pos=pos, interleaved=True)


def test_mqa_and_scale(rfa):
    full_bnsd(rfa, 1, 8, 1, 200, 128, seed=13, scale=0.05)


def test_ntk_scaling_beyond_train_len(rfa):
    full_bnsd(rfa, 1, 2, 1, 600, 128, seed=15, ntk=(256, 2.0))


def test_explicit_inv_freq_and_arbitrary_positions(rfa):
    B, S, D = 2, 290, 128
    g = workloads.gen(21)
    pos = torch.randint(-100000, 200000, (B, S), generator=g, dtype=torch.int32)
    inv = torch.rand(B, D // 2, generator=g, dtype=torch.float32)
    full_bnsd(rfa, B, 4, 2, S, D, seed=22, pos=pos, inv=inv)


def test_position_shift_invariance(rfa):
    """Rotated scores depend only on position differences: shifting every
    position by a constant leaves the output unchanged (within tolerance)."""
    B, Hq, Hkv, S, D = 1, 2, 1, 256, 128
    outs = []
    for c in (0, 1000):
        pos = (torch.arange(S, dtype=torch.int32) + c).repeat(B, 1).contiguous()
        outs.append(run_bnsd(rfa, B, Hq, Hkv, S, D, seed=31, pos=pos)[-1])
    d = np.abs(outs[0] - outs[1])
    assert d.max() <= MAX_ABS


def _packed(rfa, lens, Hq, Hkv, D, *, seed, base=10000.0, random_inv=False, ntk=None, rows=None, dtype=torch.bfloat16,
            interleaved=False):
    T = int(sum(lens))
    q = workloads.randn16((T, Hq, D), seed, dtype)
    k = workloads.randn16((T, Hkv, D), seed + 1, dtype)
    v = workloads.randn16((T, Hkv, D), seed + 2, dtype)
    pos = torch.cat([torch.arange(int(n), dtype=torch.int32) for n in lens])
    kw = dict(layout="TND", seq_lens=[int(x) for x in lens], rope_base=base, interleaved=interleaved)
    inv_t = None
    if random_inv:
        inv_t = torch.rand(len(lens), D // 2, generator=workloads.gen(seed + 3), dtype=torch.float32)
        kw["inv_freq"] = inv_t.cuda()
    if ntk is not None:
        kw.update(ntk_train_len=ntk[0], ntk_factor=ntk[1])
    out = rfa.fused_rope_attention(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), **kw)
    assert rfa.get_device_status() == 0
    got = out.float().cpu().numpy()
    inv = inv_t.double().numpy() if random_inv else _inv_rows(len(lens), D, base, lens, ntk)
    if rows is None:
        ref = oracle.attention_full(q, k, v, pos.numpy(), inv, layout=oracle.TND, seq_lens=lens, interleaved=interleaved)
        return _compare(got, ref)
    ref = oracle.attention_rows(q, k, v, pos.numpy(), inv, rows, layout=oracle.TND, seq_lens=lens,
                                interleaved=interleaved)
    t0 = np.concatenate([[0], np.cumsum(lens)])
    return _compare(got[t0[rows[:, 0]] + rows[:, 2], rows[:, 1]], ref)


def test_packed_ragged_sequences(rfa):
    _packed(rfa, [1, 127, 128, 129, 300, 5], 4, 2, 128, seed=40)


def test_packed_d64_random_inv(rfa):
    _packed(rfa, [64, 1, 200], 2, 2, 64, seed=50, random_inv=True)


def test_packed_adjacent_pairs(rfa):
    _packed(rfa, [130, 5, 260], 4, 1, 128, seed=65, interleaved=True)


def test_packed_per_sequence_ntk(rfa):
    _packed(rfa, [100, 700, 300], 4, 1, 128, seed=60, ntk=(256, 2.0))


# ---------------------------------------------------------------- full workload sizes, every output element
class _Err:
    """Max abs error and relative Frobenius error accumulated over chunks."""

    def __init__(self):
        self.max_abs, self.d2, self.r2 = 0.0, 0.0, 0.0

    def add(self, got, ref):
        got = np.asarray(got, np.float64)
        assert np.all(np.isfinite(got))
        d = got - ref
        self.max_abs = max(self.max_abs, float(np.abs(d).max()))
        self.d2 += float((d * d).sum())
        self.r2 += float((ref * ref).sum())

    def check(self):
        fro = (self.d2 / max(self.r2, 1e-300)) ** 0.5
        assert self.max_abs <= MAX_ABS, f"max abs {self.max_abs:.3e}"
        assert fro <= REL_FRO, f"rel fro {fro:.3e}"
        return self.max_abs, fro


def _bench_path(rfa, q, k, v, pos, inv, kw):
    """The launch sequence bench.py times: the cos/sin table kernels into a
    workspace, then the fused attention kernel reading it."""
    table = rfa.rope_attention_table(q, k, pos, inv_freq=inv, **kw)
    out = rfa.fused_rope_attention_with_table(q, k, v, table, **kw)
    assert rfa.get_device_status() == 0
    return out


@pytest.mark.parametrize("key", ["qwen7b", "gqa8k", "ntk16k"])
def test_full_size_bnsd_every_element(rfa, key):
    """The whole output of a full-size BNSD workload against the oracle, one
    kv group of query heads at a time (every row, every column)."""
    w = workloads.BY_KEY[key]
    q, k, v = workloads.make_qkv(w)
    pos = workloads.positions(w)
    kw = dict(layout="BNSD", rope_base=w.rope_base)
    ntk = None
    if w.ntk_train_len:
        kw.update(ntk_train_len=w.ntk_train_len, ntk_factor=w.ntk_factor)
        ntk = (w.ntk_train_len, w.ntk_factor)
    got = _bench_path(rfa, q.cuda(), k.cuda(), v.cuda(), pos.cuda(), None, kw).float().cpu().numpy()
    inv = _inv_rows(w.B, w.D, w.rope_base, [w.S] * w.B, ntk)
    G = w.Hq // w.Hkv
    err = _Err()
    for b in range(w.B):
        for kvh in range(w.Hkv):
            heads = np.arange(kvh * G, (kvh + 1) * G)
            hh, ii = np.meshgrid(heads, np.arange(w.S), indexing="ij")
            rows = np.stack([np.full(hh.size, b), hh.ravel(), ii.ravel()], axis=1).astype(np.int32)
            ref = oracle.attention_rows(q, k, v, pos.numpy(), inv, rows)
            err.add(got[b, heads].reshape(-1, w.D), ref)
    err.check()


def test_full_size_packed_every_element(rfa):
    """The whole output of the packed workload (16 sequences, T = 57,209,
    per-sequence invFreq rows) against the oracle, one sequence and kv group
    at a time."""
    w = workloads.PACKED
    lens = workloads.seq_lengths(w)
    q, k, v = workloads.make_qkv(w)
    pos = workloads.positions(w)
    inv_t = workloads.random_inv_freq(w)
    kw = dict(layout="TND", seq_lens=lens, rope_base=w.rope_base)
    got = _bench_path(rfa, q.cuda(), k.cuda(), v.cuda(), pos.cuda(), inv_t.cuda(), kw).float().cpu().numpy()
    inv = inv_t.double().numpy()
    t0 = np.concatenate([[0], np.cumsum(lens)])
    G = w.Hq // w.Hkv
    err = _Err()
    for b in range(w.B):
        for kvh in range(w.Hkv):
            heads = np.arange(kvh * G, (kvh + 1) * G)
            hh, ii = np.meshgrid(heads, np.arange(lens[b]), indexing="ij")
            rows = np.stack([np.full(hh.size, b), hh.ravel(), ii.ravel()], axis=1).astype(np.int32)
            ref = oracle.attention_rows(q, k, v, pos.numpy(), inv, rows, layout=oracle.TND, seq_lens=lens)
            err.add(got[t0[b] + rows[:, 2], rows[:, 1]], ref)
    err.check()


def test_long_sequence_65536_last_tiles(rfa):
    """S = 65536 (512 key tiles): the key angles advance through 512 steps of
    the recurrence.  Every row of the last two query tiles (which read all 512
    key tiles) and one seeded row of every other query tile, both heads."""
    B, Hq, Hkv, S, D = 1, 2, 1, 65536, 128
    base = 500000.0
    q = workloads.randn16((B, Hq, S, D), 301)
    k = workloads.randn16((B, Hkv, S, D), 302)
    v = workloads.randn16((B, Hkv, S, D), 303)
    pos = torch.arange(S, dtype=torch.int32)[None].contiguous()
    kw = dict(layout="BNSD", rope_base=base)
    got = _bench_path(rfa, q.cuda(), k.cuda(), v.cuda(), pos.cuda(), None, kw).float().cpu().numpy()
    rng = np.random.default_rng(304)
    rows = []
    for h in range(Hq):
        rows += [(0, h, i) for i in range(S - 256, S)]
        rows += [(0, h, t * 128 + int(rng.integers(128))) for t in range(S // 128 - 2)]
    rows = np.array(rows, np.int32)
    ref = oracle.attention_rows(q, k, v, pos.numpy(), _inv_rows(B, D, base), rows)
    _compare(got[rows[:, 0], rows[:, 1], rows[:, 2]], ref)


def test_positions_wrapping_past_int32_max(rfa):
    """Positions p0 + i counted past INT32_MAX wrap to negative int32 values,
    so the sequence's positions are not consecutive and its keys must take
    their angles from the table, not the recurrence (which would continue past
    the wrap, 2^32 * invFreq radians away).  Small inverse frequencies keep the
    angles of positions near 2^31 accurate in fp32."""
    B, Hq, Hkv, S, D = 1, 2, 1, 300, 128
    p0 = 2**31 - 150
    wrapped = (torch.arange(S, dtype=torch.int64) + p0 + 2**31) % 2**32 - 2**31
    pos = wrapped.to(torch.int32)[None].contiguous()
    assert int(pos[0, -1]) < 0 < int(pos[0, 0])
    inv = (torch.linspace(0.5, 1.0, D // 2) * 1e-9)[None].to(torch.float32).contiguous()
    full_bnsd(rfa, B, Hq, Hkv, S, D, seed=310, pos=pos, inv=inv)
