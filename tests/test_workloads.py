"""CPU checks of the seeded input generators shared by the tests, the bench and the oracle: every
piece regenerates bit-identically on its own, and lengths, placements and scales have the shapes
and ranges the workloads state."""
import numpy as np
import pytest
import torch

import workloads as W


@pytest.mark.parametrize("name", sorted(W.ALL))
def test_pieces_regenerate_bit_identically(name):
    w = W.ALL[name]
    lens = W.context_lens(w)
    assert torch.equal(lens, W.context_lens(w))
    assert torch.equal(W.block_order(w), W.block_order(w))
    assert torch.equal(W.query(w).view(torch.int16), W.query(w).view(torch.int16))
    s = int(w.num_seqs) - 1
    for which in ("k", "v"):
        a = W.kv_source(w, s, which, lens)
        assert torch.equal(a.view(torch.int16), W.kv_source(w, s, which, lens).view(torch.int16))
    if w.kv_dtype == "e4m3":
        assert W.fp8_scales(w) == W.fp8_scales(w)


@pytest.mark.parametrize("name", sorted(W.ALL))
def test_shapes_and_ranges(name):
    w = W.ALL[name]
    lens = W.context_lens(w)
    assert lens.dtype == torch.int32 and lens.shape == (w.num_seqs,)
    kind = w.ctx[0]
    if kind == "uniform":
        lo, hi = w.ctx[1], w.ctx[2]
        own = lens - w.shared_prefix_tokens
        assert int(own.min()) >= lo and int(own.max()) <= hi
    order = W.block_order(w).numpy()
    assert sorted(order.tolist()) == list(range(w.num_blocks))  # a permutation of the pool
    assert W.max_blocks_per_seq(w, lens) * 16 >= int(lens.max())
    q = W.query(w)
    assert q.shape == (w.num_seqs, w.num_q_heads, w.head_dim)
    k = W.kv_source(w, 0, "k", lens)
    assert k.shape == (int(lens[0]), w.num_kv_heads, w.head_dim)
    assert torch.isfinite(k.float()).all()
    # N(0, 1) draws: mean and spread near 0 and 1 over the query
    qf = q.double().numpy().ravel()
    assert abs(qf.mean()) < 0.1 and 0.9 < qf.std() < 1.1


def test_prefix_workload_shares_its_first_tokens():
    w = W.ALL["prefix_gqa_small"]
    lens = W.context_lens(w)
    P = w.shared_prefix_tokens
    a, b = W.kv_source(w, 0, "k", lens), W.kv_source(w, 1, "k", lens)
    assert torch.equal(a[:P].view(torch.int16), b[:P].view(torch.int16))
    assert not torch.equal(a[P:P + 1].view(torch.int16), b[P:P + 1].view(torch.int16))


def test_fp8_scales_are_amax_over_448():
    w = W.ALL["long70b_fp8_small"]
    ks, vs = W.fp8_scales(w)
    lens = W.context_lens(w)
    kmax = max(float(W.kv_source(w, s, "k", lens).float().abs().max()) for s in range(w.num_seqs))
    vmax = max(float(W.kv_source(w, s, "v", lens).float().abs().max()) for s in range(w.num_seqs))
    assert ks == float(np.float32(kmax) / np.float32(448)) and vs == float(np.float32(vmax) / np.float32(448))
    # the largest source magnitude maps to the largest finite e4m3 value, none beyond it
    assert np.float32(kmax) / np.float32(ks) <= 448.0001
