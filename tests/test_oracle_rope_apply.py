"""Pins of oracle.rope_apply, the Rope operator on given sin/cos tables (page
"DynamicNTKOperation", operator context: q, k, sin, cos in, rotated q, k out;
adjacent-pair variant from page "RoPE, RMSNorm, GQA/MQA, SwiGLU, MoE", sec. 6).

Each pin checks it against something other than its own formula: complex
multiplication in numpy, the pinned position-based rotation, the bare pair
permutation written with numpy slicing, and invariants of a rotation.
"""
import numpy as np

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def _angles(n, half, seed):
    return _rng(seed).uniform(-50.0, 50.0, (n, half))


def test_rotate_half_is_complex_multiplication():
    n, D = 7, 16
    x = _rng(1).standard_normal((n, D))
    th = _angles(n, D // 2, 2)
    sin_t = np.concatenate([np.sin(th), np.sin(th)], axis=1)
    cos_t = np.concatenate([np.cos(th), np.cos(th)], axis=1)
    got = oracle.rope_apply(x, sin_t, cos_t, np.arange(n))
    z = (x[:, : D // 2] + 1j * x[:, D // 2:]) * np.exp(1j * th)
    np.testing.assert_allclose(got, np.concatenate([z.real, z.imag], axis=1), rtol=0, atol=1e-12)


def test_adjacent_pairs_are_complex_multiplication():
    n, D = 5, 12
    x = _rng(3).standard_normal((n, D))
    th = _angles(n, D // 2, 4)
    sin_t = np.repeat(np.sin(th), 2, axis=1)  # cos/sin of pair i at columns 2i and 2i+1
    cos_t = np.repeat(np.cos(th), 2, axis=1)
    got = oracle.rope_apply(x, sin_t, cos_t, np.arange(n), interleaved=True)
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * th)
    want = np.empty_like(x)
    want[:, 0::2], want[:, 1::2] = z.real, z.imag
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_dynamic_ntk_tables_reproduce_position_rotation():
    # tables from the pinned sin/cos table, rows looked up per token: the same
    # as rotating by the positions directly
    D, lens = 32, np.array([3, 5], np.int32)
    pos = np.array([0, 1, 2, 100, -7, 3, 4, 65535], np.int32)
    inv = np.stack([oracle.inv_freq(10000.0, D), oracle.inv_freq(500000.0, D)])
    s, c = oracle.rope_sincos(pos, inv, lens, D)
    x = _rng(5).standard_normal((len(pos), D))
    got = oracle.rope_apply(x, s, c, np.arange(len(pos)))
    seg = np.repeat(np.arange(2), lens)
    want = np.concatenate([oracle.rope_rotate(x[t:t + 1], pos[t:t + 1], inv[seg[t]]) for t in range(len(pos))])
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_quarter_turn_is_the_pair_permutation():
    n, D = 4, 10
    x = _rng(6).standard_normal((n, D))
    ones, zeros = np.ones((1, D)), np.zeros((1, D))
    rows = np.zeros(n, np.int64)
    half = oracle.rope_apply(x, ones, zeros, rows)
    np.testing.assert_array_equal(half, np.concatenate([-x[:, D // 2:], x[:, : D // 2]], axis=1))
    adj = oracle.rope_apply(x, ones, zeros, rows, interleaved=True)
    want = np.empty_like(x)
    want[:, 0::2], want[:, 1::2] = -x[:, 1::2], x[:, 0::2]
    np.testing.assert_array_equal(adj, want)


def test_zero_sine_scales_elementwise_and_zero_angle_is_identity():
    n, D = 3, 8
    x = _rng(7).standard_normal((n, D))
    c = _rng(8).standard_normal((2, D))
    rows = np.array([1, 0, 1])
    for inter in (False, True):
        np.testing.assert_array_equal(oracle.rope_apply(x, np.zeros((2, D)), c, rows, inter), x * c[rows])
        np.testing.assert_array_equal(oracle.rope_apply(x, np.zeros((1, D)), np.ones((1, D)), np.zeros(n, np.int64),
                                                        inter), x)


def test_pair_norms_preserved():
    n, D = 6, 16
    x = _rng(9).standard_normal((n, D))
    th = _angles(n, D // 2, 10)
    s2 = np.concatenate([np.sin(th)] * 2, axis=1)
    c2 = np.concatenate([np.cos(th)] * 2, axis=1)
    out = oracle.rope_apply(x, s2, c2, np.arange(n))
    np.testing.assert_allclose(out[:, :8] ** 2 + out[:, 8:] ** 2, x[:, :8] ** 2 + x[:, 8:] ** 2, rtol=1e-12)
    s1, c1 = np.repeat(np.sin(th), 2, axis=1), np.repeat(np.cos(th), 2, axis=1)
    out = oracle.rope_apply(x, s1, c1, np.arange(n), interleaved=True)
    np.testing.assert_allclose(out[:, 0::2] ** 2 + out[:, 1::2] ** 2, x[:, 0::2] ** 2 + x[:, 1::2] ** 2, rtol=1e-12)


def test_attention_adjacent_pairs_is_rotate_half_on_permuted_dims():
    # pair (2i, 2i+1) of the adjacent variant is pair (i, i + D/2) once the
    # dims are reordered even-then-odd; q.k is unchanged by reordering both
    import torch

    import workloads

    B, Hq, Hkv, S, D = 1, 2, 1, 37, 16
    q = workloads.randn16((B, Hq, S, D), 31)
    k = workloads.randn16((B, Hkv, S, D), 32)
    v = workloads.randn16((B, Hkv, S, D), 33)
    pos = torch.arange(S, dtype=torch.int32)[None] * 3 - 5
    inv = oracle.inv_freq(100.0, D)[None]
    perm = np.concatenate([np.arange(0, D, 2), np.arange(1, D, 2)])
    got = oracle.attention_full(q, k, v, pos.numpy(), inv, interleaved=True)
    want = oracle.attention_full(q[..., perm].contiguous(), k[..., perm].contiguous(), v, pos.numpy(), inv)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    # and it is a different operation from rotate-half on the original order
    assert np.abs(got - oracle.attention_full(q, k, v, pos.numpy(), inv)).max() > 1e-3


def test_rms_norm_pins():
    import torch

    x = _rng(40).standard_normal((9, 24)) * 3.0
    g = _rng(41).uniform(0.5, 2.0, 24)
    # a library routine as the reference: torch's rms_norm in fp64
    want = torch.nn.functional.rms_norm(torch.from_numpy(x), (24,), torch.from_numpy(g), eps=1e-5).numpy()
    np.testing.assert_allclose(oracle.rms_norm(x, g, 1e-5), want, rtol=1e-13, atol=1e-13)
    # closed forms: unit RMS with gamma = 1, eps = 0; invariant to a positive scale; gamma elementwise
    one = oracle.rms_norm(x, np.ones(24), 0.0)
    np.testing.assert_allclose(np.sqrt((one ** 2).mean(axis=1)), 1.0, rtol=1e-13)
    np.testing.assert_allclose(oracle.rms_norm(7.5 * x, np.ones(24), 0.0), one, rtol=1e-13)
    np.testing.assert_allclose(oracle.rms_norm(x, g, 0.0), one * g, rtol=1e-13)


def test_kv_cache_op_is_norm_then_rope_at_slots():
    T, H, D, rows = 5, 2, 16, 8
    k = _rng(42).standard_normal((T, H, D))
    v = _rng(43).standard_normal((T, H, D))
    g = _rng(44).uniform(0.5, 2.0, D)
    th = _angles(T, D // 2, 45)
    s = np.concatenate([np.sin(th)] * 2, axis=1)
    c = np.concatenate([np.cos(th)] * 2, axis=1)
    slots = np.array([3, -1, 0, 7, 5])
    kc0, vc0 = np.full((rows, H, D), 9.0), np.full((rows, H, D), -9.0)
    kc, vc = oracle.kv_rms_norm_rope_cache(k, v, g, 1e-6, s, c, slots, kc0, vc0)
    for t, sl in enumerate(slots):
        if sl < 0:
            continue
        # rotate-half via complex multiplication of the normalised row
        kn = oracle.rms_norm(k[t], g, 1e-6)
        z = (kn[:, : D // 2] + 1j * kn[:, D // 2:]) * np.exp(1j * th[t])
        np.testing.assert_allclose(kc[sl], np.concatenate([z.real, z.imag], axis=1), rtol=0, atol=1e-12)
        np.testing.assert_array_equal(vc[sl], v[t])
    untouched = [r for r in range(rows) if r not in set(slots[slots >= 0].tolist())]
    np.testing.assert_array_equal(kc[untouched], kc0[untouched])
    np.testing.assert_array_equal(vc[untouched], vc0[untouched])


def test_decode_equals_last_rows_of_full_attention():
    # a cache filled with keys rotated by the pinned Rope operator at positions
    # 0..L-1: decoding the last Sq tokens reproduces the last Sq rows of the
    # pinned full causal attention, for both pairings and with GQA
    import torch

    import workloads

    B, Hq, Hkv, D, L, Sq = 2, 4, 2, 16, 23, 3
    for inter in (False, True):
        q = workloads.randn16((B, Hq, L, D), 60)
        k = workloads.randn16((B, Hkv, L, D), 61)
        v = workloads.randn16((B, Hkv, L, D), 62)
        pos = np.tile(np.arange(L, dtype=np.int32), (B, 1))
        inv = np.stack([oracle.inv_freq(100.0, D)] * B)
        full = oracle.attention_full(q, k, v, pos, inv, interleaved=inter)
        # rotated keys, token-major cache [B, L, Hkv, D]
        th = pos[..., None] * inv[:, None, :]                       # [B, L, D/2]
        if inter:
            s_t, c_t = np.repeat(np.sin(th), 2, -1), np.repeat(np.cos(th), 2, -1)
        else:
            s_t, c_t = np.concatenate([np.sin(th)] * 2, -1), np.concatenate([np.cos(th)] * 2, -1)
        kf = k.float().numpy().astype(np.float64).transpose(0, 2, 1, 3)  # [B, L, Hkv, D]
        rows = np.repeat(np.arange(B * L), Hkv)
        kr = oracle.rope_apply(kf.reshape(-1, D), s_t.reshape(-1, D), c_t.reshape(-1, D), rows, inter)
        kc = kr.reshape(B, L, Hkv, D)
        vc = v.float().numpy().astype(np.float64).transpose(0, 2, 1, 3)
        got = oracle.decode_attention(q[:, :, L - Sq:], kc, vc, pos[:, L - Sq:], [L] * B, inv, interleaved=inter)
        np.testing.assert_allclose(got, full[:, :, L - Sq:], rtol=0, atol=1e-12)
