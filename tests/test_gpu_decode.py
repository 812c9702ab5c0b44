"""GPU parity of rfa_decode_rope_attention (decode over a KV cache) against
oracle.decode_attention, through the C ABI.

The cache holds arbitrary bf16/fp16 values: the operation takes cached keys as
already rotated, so any contents are valid keys.  Bar as for the fused
attention: max abs error <= 2e-2 and relative Frobenius error <= 5e-3.
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


def _case(rfa, B, Hq, Hkv, Sq, D, Smax, lens, *, seed, dtype=torch.bfloat16, causal=True, interleaved=False,
          base=10000.0, inv=None, max_len=None, num_splits=0):
    q = workloads.randn16((B, Hq, Sq, D), seed, dtype)
    kc = workloads.randn16((B, Smax, Hkv, D), seed + 1, dtype)
    vc = workloads.randn16((B, Smax, Hkv, D), seed + 2, dtype)
    lens_t = torch.tensor(lens, dtype=torch.int32)
    # new tokens sit at the last Sq positions of each sequence
    q_pos = torch.stack([torch.arange(L - Sq, L, dtype=torch.int32) for L in lens])
    kw = dict(causal=causal, interleaved=interleaved, rope_base=base, max_kv_len=max_len, num_splits=num_splits)
    if inv is not None:
        kw["inv_freq"] = inv.cuda()
    out = rfa.decode_rope_attention(q.cuda(), kc.cuda(), vc.cuda(), q_pos.cuda(), lens_t.cuda(), **kw)
    st = rfa.get_device_status()
    inv_rows = inv.double().numpy() if inv is not None else np.stack([oracle.inv_freq(base, D)] * B)
    ref = oracle.decode_attention(q, kc, vc, q_pos.numpy(), lens, inv_rows, causal=causal, interleaved=interleaved)
    return out.float().cpu().numpy().astype(np.float64), ref, st


def _compare(got, ref):
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref)
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err.max() <= MAX_ABS, f"max abs {err.max():.3e}"
    assert fro <= REL_FRO, f"rel fro {fro:.3e}"


def test_gqa_single_token_split_keys(rfa):
    # 2 x 8 kv groups: the keys of each sequence are split across CTAs and merged
    got, ref, st = _case(rfa, 2, 32, 8, 1, 128, 4096, [1000, 3001], seed=1)
    assert st == 0
    _compare(got, ref)


def test_many_groups_one_split(rfa):
    # 80 x 8 kv groups fill the GPU without splitting the keys
    lens = [int(x) for x in np.random.default_rng(2).integers(1, 700, 80)]
    got, ref, st = _case(rfa, 80, 16, 8, 1, 128, 700, lens, seed=3)
    assert st == 0
    _compare(got, ref)


@pytest.mark.parametrize("D", [64, 128])
def test_several_new_tokens(rfa, D):
    # Sq = 4 new tokens with G = 8 (32 query rows per tile), ragged lengths, partial last tiles;
    # one key tile per split, so the second chain of every CTA is empty and reaches the merge
    # while the first still runs (the rows it exchanges must not share shared memory with the
    # query tile's cos/sin rows)
    got, ref, st = _case(rfa, 3, 16, 2, 4, D, 600, [300, 129, 5], seed=4)
    assert st == 0
    _compare(got, ref)


@pytest.mark.parametrize("dtype,inter,causal", [(torch.float16, False, False), (torch.bfloat16, True, True)])
def test_dtype_pairing_and_mask(rfa, dtype, inter, causal):
    got, ref, st = _case(rfa, 2, 8, 1, 2, 128, 900, [900, 257], seed=5, dtype=dtype, causal=causal,
                         interleaved=inter)
    assert st == 0
    _compare(got, ref)


def test_explicit_inv_freq(rfa):
    inv = torch.rand(2, 64, generator=workloads.gen(6), dtype=torch.float32)
    got, ref, st = _case(rfa, 2, 4, 4, 1, 128, 512, [512, 77], seed=7, inv=inv, max_len=512)
    assert st == 0
    _compare(got, ref)


def test_lengths_outside_the_bound_set_status(rfa):
    B, Hq, Hkv, Sq, D, Smax = 2, 4, 2, 2, 64, 256
    q = workloads.randn16((B, Hq, Sq, D), 8).cuda()
    kc = workloads.randn16((B, Smax, Hkv, D), 9).cuda()
    q_pos = torch.zeros((B, Sq), dtype=torch.int32).cuda()
    for lens in ([1, 100], [100, 200]):  # 1 < Sq; 200 > max_kv_len = 128
        out = rfa.decode_rope_attention(q, kc, kc, q_pos, torch.tensor(lens, dtype=torch.int32).cuda(),
                                        max_kv_len=128)
        assert rfa.get_device_status() == rfa.RFA_ERR_INVALID_ARG
        assert torch.isfinite(out.float()).all()
    assert rfa.get_device_status() == 0


# A CTA runs its split's key tiles in two chains (tile j into score/accumulator
# buffer j % 2) and merges them before the store: one-tile splits leave buffer 1
# empty, odd tile counts give buffer 0 one tile more, ragged tails and the
# bottom-right causal edge fall in either buffer.
@pytest.mark.parametrize("lens,Smax,num_splits,Sq", [
    ([1000, 3001], 3072, 1, 1),     # one split: 8 and 24 tiles, direct store
    ([129, 3001], 3072, 24, 1),     # one tile per split: buffer 1 never used
    ([640, 1663], 2048, 3, 1),      # 6 tiles per split: even, the last split ragged
    ([1100, 1999], 2048, 2, 3),     # 8 tiles per split, 3 new tokens on the causal edge
    ([300, 700], 768, 6, 4),        # one tile per split, short sequences, empty splits
])
def test_two_chain_merge_and_given_splits(rfa, lens, Smax, num_splits, Sq):
    got, ref, st = _case(rfa, 2, 32, 8, Sq, 128, Smax, lens, seed=11 + num_splits, num_splits=num_splits)
    assert st == 0
    _compare(got, ref)


def test_two_chain_merge_d64_fp16_noncausal(rfa):
    got, ref, st = _case(rfa, 3, 16, 4, 2, 64, 1500, [1500, 385, 2], seed=21, dtype=torch.float16, causal=False,
                         num_splits=2)
    assert st == 0
    _compare(got, ref)


def test_benchmarked_shape_32k_keys(rfa):
    """The shape bench.py times: 8 sequences x 32 query / 8 kv heads, one new
    token each, over 32768 cached keys, with the library's own split plan.
    Every output row (all 8 x 32) against the oracle, one sequence at a time
    so the fp64 copy of the cache stays small."""
    B, Hq, Hkv, Sq, D, L = 8, 32, 8, 1, 128, 32768
    q = workloads.randn16((B, Hq, Sq, D), 41)
    kc = workloads.randn16((B, L, Hkv, D), 42)
    vc = workloads.randn16((B, L, Hkv, D), 43)
    q_pos = torch.full((B, Sq), L - 1, dtype=torch.int32)
    lens = torch.full((B,), L, dtype=torch.int32)
    out = rfa.decode_rope_attention(q.cuda(), kc.cuda(), vc.cuda(), q_pos.cuda(), lens.cuda())
    assert rfa.get_device_status() == 0
    got = out.float().cpu().numpy().astype(np.float64)
    inv = oracle.inv_freq(10000.0, D)[None]
    ref = np.concatenate([oracle.decode_attention(q[b:b + 1], kc[b:b + 1], vc[b:b + 1], q_pos[b:b + 1].numpy(), [L],
                                                  inv) for b in range(B)])
    _compare(got, ref)


@pytest.mark.parametrize("D,dtype,inter", [(128, torch.bfloat16, False), (64, torch.float16, True)])
def test_full_query_tile_of_new_tokens(rfa, D, dtype, inter):
    """G * Sq = 128: the query tile is full (G = 8 heads x 16 new tokens), so the
    cos/sin rows the kernel forms for its query rows cover every row and chunk
    of the tile; positions end at different lengths per sequence and the keys
    are split across CTAs."""
    got, ref, st = _case(rfa, 2, 16, 2, 16, D, 2100, [2100, 777], seed=12, dtype=dtype, interleaved=inter)
    assert st == 0
    _compare(got, ref)
