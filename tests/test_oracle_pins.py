"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test ties one oracle function to a closed form, an independent library
(mpmath, numpy's complex exponential, torch's CPU attention), a textbook
special case, an invariant the pages state, or brute force on tiny inputs.
Together they catch a dropped term, a wrong sign, a wrong pairing or index,
and a transposed operand anywhere in the oracle.
"""
import math
import os

import mpmath as mp
import numpy as np
import pytest
import torch

import oracle
import workloads

mp.mp.dps = 30


def _golden(golden_dir):
    vals = {}
    with open(os.path.join(golden_dir, "circular_values.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, s, c = line.split()
            vals[float(a)] = (float(s), float(c))
    return vals


def test_golden_values_agree_with_mpmath(golden_dir):
    for a, (s, c) in _golden(golden_dir).items():
        assert abs(s - float(mp.sin(mp.mpf(a)))) < 1e-17
        assert abs(c - float(mp.cos(mp.mpf(a)))) < 1e-17


# ---------------------------------------------------------------- widening
def test_widen16_matches_torch_conversion():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, 4096, dtype=np.uint16)
    for code, tdt in ((oracle.BF16, torch.bfloat16), (oracle.FP16, torch.float16)):
        ref = torch.from_numpy(bits.view(np.int16)).view(tdt).double().numpy()
        got = np.array([oracle.widen16(int(b), code) for b in bits])
        fin = np.isfinite(ref)
        np.testing.assert_array_equal(got[fin], ref[fin])
        assert np.all(np.isnan(got[np.isnan(ref)]))
    assert oracle.widen16(0x3F80, oracle.BF16) == 1.0
    assert oracle.widen16(0x3C00, oracle.FP16) == 1.0
    assert oracle.widen16(0x0001, oracle.FP16) == 2.0 ** -24
    assert oracle.widen16(0xC000, oracle.BF16) == -2.0


# ---------------------------------------------------------------- invFreq / NTK
@pytest.mark.parametrize("base,D", [(10000.0, 64), (10000.0, 128), (500000.0, 128), (30527.7367488067, 128)])
def test_inv_freq_matches_mpmath(base, D):
    got = oracle.inv_freq(base, D)
    assert got.shape == (D // 2,)
    assert got[0] == 1.0
    for j in range(D // 2):
        ref = mp.mpf(1) / mp.power(mp.mpf(base), mp.mpf(2 * j) / D)
        assert abs(got[j] - float(ref)) <= 4e-16 * float(ref)


def test_inv_freq_geometric_and_midpoint():
    inv = oracle.inv_freq(10000.0, 128)
    ratios = inv[1:] / inv[:-1]
    np.testing.assert_allclose(ratios, 10000.0 ** (-2.0 / 128), rtol=1e-13)
    assert abs(inv[32] - 0.01) < 1e-15  # base^(-1/2) at j = D/4


def test_ntk_base_no_interpolation_up_to_train_len():
    for S in (1, 100, 8191, 8192):
        assert oracle.ntk_base(10000.0, 128, S, 8192, 2.0) == 10000.0


def test_ntk_base_long_context_value():
    # factor 2, S = 2L: base * 3^(D/(D-2)), evaluated independently with mpmath.
    got = oracle.ntk_base(10000.0, 128, 16384, 8192, 2.0)
    ref = 10000 * mp.power(3, mp.mpf(128) / 126)
    assert abs(got - float(ref)) < 1e-9
    assert abs(got - 30527.74) < 5e-3
    # factor 1 reduces to the classic NTK-aware scale (S/L)^(D/(D-2)).
    got1 = oracle.ntk_base(10000.0, 64, 4096, 1024, 1.0)
    assert abs(got1 - float(10000 * mp.power(4, mp.mpf(64) / 62))) < 1e-8
    # continuous at S = L + 1 -> just above base
    assert 10000.0 < oracle.ntk_base(10000.0, 128, 8193, 8192, 2.0) < 10010.0


# ---------------------------------------------------------------- sin/cos table
def test_sincos_golden_exact_angles(golden_dir):
    g = _golden(golden_dir)
    pos = np.array([0, 1, 2, 0, 1], np.int32)
    lens = np.array([3, 2], np.int32)
    # head size 8 -> 4 frequencies per row; batch 1 uses doubled frequencies.
    inv = np.array([[1.0, 0.5, 0.25, 0.0], [2.0, 1.0, 0.5, 0.25]])
    s, c = oracle.rope_sincos(pos, inv, lens, 8)
    assert s.shape == (5, 8)
    # token 0 (pos 0): sin 0, cos 1 everywhere
    assert np.all(s[0] == 0.0) and np.all(c[0] == 1.0)
    # token 1 (pos 1, batch 0): angles 1, 0.5, 0.25, 0 then repeated
    for j, a in enumerate([1.0, 0.5, 0.25]):
        assert abs(s[1, j] - g[a][0]) < 1e-16 and abs(c[1, j] - g[a][1]) < 1e-16
        assert s[1, j + 4] == s[1, j] and c[1, j + 4] == c[1, j]
    # token 2 (pos 2, batch 0): angles 2, 1, 0.5
    for j, a in enumerate([2.0, 1.0, 0.5]):
        assert abs(s[2, j] - g[a][0]) < 1e-16 and abs(c[2, j] - g[a][1]) < 1e-16
    # token 4 (pos 1, batch 1): its own row 2, 1, 0.5, 0.25 (segment indexing)
    for j, a in enumerate([2.0, 1.0, 0.5, 0.25]):
        assert abs(s[4, j] - g[a][0]) < 1e-16 and abs(c[4, j] - g[a][1]) < 1e-16


def test_sincos_matches_mpmath_large_positions():
    rng = np.random.default_rng(1)
    T, D = 64, 16
    pos = rng.integers(-20000, 256000, T).astype(np.int32)
    inv32 = rng.random((2, D // 2)).astype(np.float32)
    lens = np.array([40, 24], np.int32)
    s, c = oracle.rope_sincos(pos, inv32.astype(np.float64), lens, D)
    seg = np.repeat([0, 1], lens)
    for t in range(T):
        for j in range(D):
            a = mp.mpf(int(pos[t])) * mp.mpf(float(inv32[seg[t], j % (D // 2)]))
            assert abs(s[t, j] - float(mp.sin(a))) < 1e-10
            assert abs(c[t, j] - float(mp.cos(a))) < 1e-10


def test_sincos_pythagoras_and_duplicated_halves():
    pos, inv, lens = workloads.sincos_problem(1000, 128, 7, seed=3)
    s, c = oracle.rope_sincos(pos.numpy(), inv.numpy(), lens.numpy(), 128)
    np.testing.assert_allclose(s * s + c * c, 1.0, atol=1e-14)
    np.testing.assert_array_equal(s[:, :64], s[:, 64:])
    np.testing.assert_array_equal(c[:, :64], c[:, 64:])


def test_sincos_segment_indexing_is_exact():
    # Row b of invFreq is b+1 everywhere: a token mis-assigned to another batch
    # shows an angle off by a whole multiple of its position.
    lens = np.array([5, 1, 7, 3], np.int32)
    pos = np.concatenate([np.arange(n) + 1 for n in lens]).astype(np.int32)
    inv = np.repeat(np.arange(1, 5, dtype=np.float64)[:, None], 2, axis=1) * 0.125
    s, c = oracle.rope_sincos(pos, inv, lens, 4)
    seg = np.repeat(np.arange(4), lens)
    ang = np.arctan2(s[:, 0], c[:, 0])
    want = pos * (seg + 1) * 0.125
    np.testing.assert_allclose(ang, np.arctan2(np.sin(want), np.cos(want)), atol=1e-14)


def test_sincos_rejects_bad_lengths():
    pos = np.zeros(10, np.int32)
    inv = np.zeros((2, 4))
    with pytest.raises(ValueError):
        oracle.rope_sincos(pos, inv, np.array([5, 4], np.int32), 8)
    with pytest.raises(ValueError):
        oracle.rope_sincos(pos, inv, np.array([11, -1], np.int32), 8)


# ---------------------------------------------------------------- rotation
def test_rotation_textbook_two_by_two(golden_dir):
    s1, c1 = _golden(golden_dir)[1.0]
    inv = np.array([1.0])
    e0 = oracle.rope_rotate(np.array([[1.0, 0.0]]), [1], inv)[0]
    e1 = oracle.rope_rotate(np.array([[0.0, 1.0]]), [1], inv)[0]
    # columns of [[cos, -sin], [sin, cos]]
    np.testing.assert_allclose(e0, [c1, s1], atol=1e-16)
    np.testing.assert_allclose(e1, [-s1, c1], atol=1e-16)


def test_rotation_pairs_i_with_i_plus_half():
    D = 8
    inv = np.array([1.0, 0.5, 0.25, 2.0])
    for i in range(D):
        e = np.zeros((1, D))
        e[0, i] = 1.0
        out = oracle.rope_rotate(e, [1], inv)[0]
        partner = (i + D // 2) % D
        nz = set(np.flatnonzero(np.abs(out) > 0))
        assert nz <= {i, partner}
        ang = inv[i % (D // 2)]
        assert abs(out[i] - math.cos(ang)) < 1e-15
        sign = 1.0 if i < D // 2 else -1.0
        assert abs(out[partner] - sign * math.sin(ang)) < 1e-15


def test_rotation_is_complex_multiplication():
    rng = np.random.default_rng(2)
    n, D = 50, 128
    x = rng.standard_normal((n, D))
    pos = rng.integers(-5000, 70000, n).astype(np.int32)
    inv = oracle.inv_freq(10000.0, D)
    got = oracle.rope_rotate(x, pos, inv)
    z = (x[:, : D // 2] + 1j * x[:, D // 2:]) * np.exp(1j * pos[:, None].astype(np.float64) * inv[None, :])
    np.testing.assert_allclose(got[:, : D // 2], z.real, atol=1e-12)
    np.testing.assert_allclose(got[:, D // 2:], z.imag, atol=1e-12)


def test_rotation_identity_at_zero_and_pair_norms():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((20, 64))
    inv = oracle.inv_freq(10000.0, 64)
    np.testing.assert_array_equal(oracle.rope_rotate(x, np.zeros(20, np.int32), inv), x)
    y = oracle.rope_rotate(x, np.arange(20, dtype=np.int32) * 997, inv)
    n0 = x[:, :32] ** 2 + x[:, 32:] ** 2
    n1 = y[:, :32] ** 2 + y[:, 32:] ** 2
    np.testing.assert_allclose(n1, n0, rtol=1e-12, atol=1e-12)


def test_rotated_dot_product_depends_on_offset_only():
    rng = np.random.default_rng(4)
    D = 64
    q = rng.standard_normal((1, D))
    k = rng.standard_normal((1, D))
    inv = oracle.inv_freq(10000.0, D)
    for m, n in [(5, 3), (100, 7), (0, 40)]:
        ref = (oracle.rope_rotate(q, [m], inv) @ oracle.rope_rotate(k, [n], inv).T).item()
        for c in (1, 17, 1000, -300):
            got = (oracle.rope_rotate(q, [m + c], inv) @ oracle.rope_rotate(k, [n + c], inv).T).item()
            assert abs(got - ref) < 1e-9


# ---------------------------------------------------------------- attention
def _small(B=2, Hq=4, Hkv=2, S=37, D=64, seed=10, dtype=torch.bfloat16):
    q = workloads.randn16((B, Hq, S, D), seed, dtype)
    k = workloads.randn16((B, Hkv, S, D), seed + 1, dtype)
    v = workloads.randn16((B, Hkv, S, D), seed + 2, dtype)
    pos = np.tile(np.arange(S, dtype=np.int32), (B, 1))
    return q, k, v, pos


def _sdpa(q, k, v, causal, scale=None):
    G = q.shape[1] // k.shape[1]
    kk = k.repeat_interleave(G, dim=1)
    vv = v.repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(q, kk, vv, is_causal=causal, scale=scale).numpy()


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_attention_without_rotation_matches_torch_sdpa(causal, dtype):
    q, k, v, pos = _small(dtype=dtype)
    inv = np.zeros((2, 32))
    got = oracle.attention_full(q, k, v, pos, inv, causal=causal)
    ref = _sdpa(q.double(), k.double(), v.double(), causal)
    np.testing.assert_allclose(got, ref, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_attention_with_rotation_matches_complex_rope_plus_sdpa(causal):
    q, k, v, pos = _small(S=45, seed=20)
    pos = pos + np.array([[3], [-11]], np.int32)  # distinct offsets per batch
    inv = np.stack([oracle.inv_freq(10000.0, 64), oracle.inv_freq(500000.0, 64)])

    def crot(x, b):
        x = x.double().numpy()
        z = (x[..., :32] + 1j * x[..., 32:]) * np.exp(1j * pos[b][:, None] * inv[b][None, :])
        return np.concatenate([z.real, z.imag], axis=-1)

    qr = torch.from_numpy(np.stack([crot(q[b], b) for b in range(2)]))
    kr = torch.from_numpy(np.stack([crot(k[b], b) for b in range(2)]))
    ref = _sdpa(qr, kr, v.double(), causal, scale=0.07)
    got = oracle.attention_full(q, k, v, pos, inv, causal=causal, scale=0.07)
    np.testing.assert_allclose(got, ref, atol=1e-12)


def test_probability_rows_sum_to_one_and_respect_causality():
    q, k, v, pos = _small(S=33)
    inv = np.stack([oracle.inv_freq(10000.0, 64)] * 2)
    for (b, h, i) in [(0, 0, 0), (1, 3, 32), (0, 2, 17)]:
        p = oracle.attention_probs(q, k, pos, inv, b, h, i)
        assert abs(p.sum() - 1.0) < 1e-14
        assert np.all(p[i + 1:] == 0.0) and np.all(p[: i + 1] > 0.0)
        pn = oracle.attention_probs(q, k, pos, inv, b, h, i, causal=False)
        assert abs(pn.sum() - 1.0) < 1e-14 and np.all(pn > 0)


@pytest.mark.parametrize("causal", [True, False])
def test_probability_rows_match_complex_rope_and_torch_softmax(causal):
    """Every row P[b, h, i, :] equals torch.softmax (a library routine) of the
    scores of numpy's complex rotation of q and k (another route to the same
    rotation), in fp64: the scale, the rotation, the GQA kv head h // G, the
    causal edge and the position offsets of each batch all enter."""
    q, k, v, pos = _small(S=29, seed=40)
    pos = pos + np.array([[5], [-17]], np.int32)
    inv = np.stack([oracle.inv_freq(10000.0, 64), oracle.inv_freq(300.0, 64)])
    scale = 0.09

    def crot(x, b):
        x = x.double().numpy()
        z = (x[..., :32] + 1j * x[..., 32:]) * np.exp(1j * pos[b][:, None] * inv[b][None, :])
        return np.concatenate([z.real, z.imag], axis=-1)

    G = q.shape[1] // k.shape[1]
    S = q.shape[2]
    for b in range(2):
        qr, kr = crot(q[b], b), crot(k[b], b)
        for h in range(q.shape[1]):
            sc = torch.from_numpy(qr[h] @ kr[h // G].T * scale)
            if causal:
                sc = sc.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
            ref = torch.softmax(sc, dim=-1).numpy()
            for i in (0, 11, S - 1):
                got = oracle.attention_probs(q, k, pos, inv, b, h, i, causal=causal, scale=scale)
                np.testing.assert_allclose(got, ref[i], atol=1e-13, rtol=0)


def test_probability_rows_weight_the_values_into_the_output():
    """P[b, h, i, :] @ V[b, h // G] is the pinned attention output row."""
    q, k, v, pos = _small(S=31, seed=41)
    inv = np.stack([oracle.inv_freq(10000.0, 64)] * 2)
    out = oracle.attention_full(q, k, v, pos, inv)
    vv = v.double().numpy()
    for (b, h, i) in [(0, 0, 30), (1, 3, 12), (1, 2, 0)]:
        p = oracle.attention_probs(q, k, pos, inv, b, h, i)
        np.testing.assert_allclose(p @ vv[b, h // 2], out[b, h, i], atol=1e-13)


def test_constant_values_give_constant_output():
    q, k, _, pos = _small(S=50)
    v = torch.full((2, 2, 50, 64), 0.75, dtype=torch.bfloat16)
    inv = np.stack([oracle.inv_freq(10000.0, 64)] * 2)
    out = oracle.attention_full(q, k, v, pos, inv)
    np.testing.assert_allclose(out, 0.75, atol=1e-14)


def test_zero_query_gives_causal_prefix_mean():
    _, k, v, pos = _small(S=40)
    q = torch.zeros((2, 4, 40, 64), dtype=torch.bfloat16)
    inv = np.stack([oracle.inv_freq(10000.0, 64)] * 2)
    out = oracle.attention_full(q, k, v, pos, inv)
    vv = v.double().numpy().repeat(2, axis=1)
    prefix = np.cumsum(vv, axis=2) / np.arange(1, 41)[None, None, :, None]
    np.testing.assert_allclose(out, prefix, atol=1e-13)


def test_single_token_returns_its_value():
    q, k, v, pos = _small(S=1)
    inv = np.stack([oracle.inv_freq(10000.0, 64)] * 2)
    out = oracle.attention_full(q, k, v, pos + 123, inv)
    np.testing.assert_array_equal(out, v.double().numpy().repeat(2, axis=1))


def test_gqa_equals_mha_with_repeated_kv():
    q, k, v, pos = _small(Hq=8, Hkv=2, S=29)
    inv = np.stack([oracle.inv_freq(10000.0, 64)] * 2)
    gqa = oracle.attention_full(q, k, v, pos, inv)
    mha = oracle.attention_full(q, k.repeat_interleave(4, 1), v.repeat_interleave(4, 1), pos, inv)
    np.testing.assert_array_equal(gqa, mha)


def test_packed_equals_per_sequence_bnsd():
    lens = [7, 30, 1, 16]
    T, Hq, Hkv, D = sum(lens), 4, 2, 64
    q = workloads.randn16((T, Hq, D), 30)
    k = workloads.randn16((T, Hkv, D), 31)
    v = workloads.randn16((T, Hkv, D), 32)
    pos = np.concatenate([np.arange(n) * (b + 1) for b, n in enumerate(lens)]).astype(np.int32)
    inv = np.stack([oracle.inv_freq(10000.0 * (b + 1), D) for b in range(4)])
    packed = oracle.attention_full(q, k, v, pos, inv, layout=oracle.TND, seq_lens=lens)
    t0 = 0
    for b, n in enumerate(lens):
        sl = slice(t0, t0 + n)
        qb = q[sl].permute(1, 0, 2)[None].contiguous()
        kb = k[sl].permute(1, 0, 2)[None].contiguous()
        vb = v[sl].permute(1, 0, 2)[None].contiguous()
        ref = oracle.attention_full(qb, kb, vb, pos[sl][None], inv[b][None])
        np.testing.assert_array_equal(packed[sl], ref[0].transpose(1, 0, 2))
        t0 += n


def test_online_blockwise_softmax_equals_two_pass():
    """Brute force: the running-max / running-sum update over key blocks of
    any size reproduces the oracle's two-pass softmax."""
    q, k, v, pos = _small(B=1, Hq=2, Hkv=1, S=23, seed=40)
    inv = oracle.inv_freq(10000.0, 64)
    ref = oracle.attention_full(q, k, v, pos, inv[None])
    qr = oracle.rope_rotate(q[0].double().numpy().reshape(-1, 64), np.tile(pos[0], 2), inv).reshape(2, 23, 64)
    kr = oracle.rope_rotate(k[0, 0].double().numpy(), pos[0], inv)
    vv = v[0, 0].double().numpy()
    for blk in (1, 3, 5, 8, 23):
        for h in range(2):
            for i in range(23):
                m, l, o = -np.inf, 0.0, np.zeros(64)
                for j0 in range(0, i + 1, blk):
                    j1 = min(j0 + blk, i + 1)
                    s = kr[j0:j1] @ qr[h, i] / 8.0
                    m_new = max(m, s.max())
                    alpha = math.exp(m - m_new) if m > -np.inf else 0.0
                    p = np.exp(s - m_new)
                    l = l * alpha + p.sum()
                    o = o * alpha + p @ vv[j0:j1]
                    m = m_new
                np.testing.assert_allclose(o / l, ref[0, h, i], atol=1e-13)
