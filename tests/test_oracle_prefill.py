"""Pins of the oracle's chunked prefill (CPU only): torch SDPA with an explicit causal mask, the
decode oracle for each chunk's rows, and a chunk split that must not change any row."""
import numpy as np
import torch

from oracle import attention, paging


def _setup(rng, ctxs, news, hq, hkv, d):
    nb = sum(-(-c // 16) for c in ctxs) + 5
    kv = rng.standard_normal((nb, hkv, 16, d)).astype(np.float16)
    vv = rng.standard_normal((nb, hkv, 16, d)).astype(np.float16)
    kb = kv.view(np.uint8).reshape(nb, hkv, 16, 2 * d)
    vb = vv.view(np.uint8).reshape(nb, hkv, 16, 2 * d)
    bt = paging.build_block_tables(ctxs, rng.permutation(nb), nb)
    qs = np.concatenate([[0], np.cumsum(news)]).astype(np.int64)
    q = rng.standard_normal((int(qs[-1]), hq, d))
    return kb, vb, kv.astype(np.float64), vv.astype(np.float64), bt, qs, q


def check_prefill_vs_sdpa(prefill=attention.prefill_paged):
    rng = np.random.default_rng(21)
    ctxs, news, hq, hkv, d = [37, 120, 70], [37, 16, 33], 8, 2, 16
    kb, vb, kv, vv, bt, qs, q = _setup(rng, ctxs, news, hq, hkv, d)
    got = prefill(q, kb, vb, bt, qs, ctxs, 0.3, hkv, "f16")
    for s, (n, new) in enumerate(zip(ctxs, news)):
        t = np.arange(n)
        K = torch.tensor(kv[bt[s][t // 16], :, t % 16, :]).permute(1, 0, 2)[None]  # [1, Hkv, n, D]
        V = torch.tensor(vv[bt[s][t // 16], :, t % 16, :]).permute(1, 0, 2)[None]
        Q = torch.tensor(q[qs[s]:qs[s + 1]]).permute(1, 0, 2)[None]  # [1, Hq, new, D]
        pos = torch.arange(n - new, n)[:, None]
        mask = torch.arange(n)[None, :] <= pos  # bottom-right aligned causal mask
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask, scale=0.3, enable_gqa=True)
        np.testing.assert_allclose(got[qs[s]:qs[s + 1]], ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


def test_prefill_vs_sdpa():
    check_prefill_vs_sdpa()


def test_each_row_is_a_decode_at_its_position():
    rng = np.random.default_rng(22)
    ctxs, news = [50, 17], [20, 17]
    kb, vb, kv, vv, bt, qs, q = _setup(rng, ctxs, news, 4, 4, 8)
    out = attention.prefill_paged(q, kb, vb, bt, qs, ctxs, 0.5, 4, "f16")
    for s in range(2):
        for i in range(news[s]):
            p = ctxs[s] - news[s] + i
            want = attention.decode_paged(q[qs[s] + i][None], kb, vb, bt[s:s + 1], [p + 1], 0.5, 4, "f16")
            assert np.array_equal(out[qs[s] + i], want[0])


def test_splitting_the_chunk_changes_nothing():
    rng = np.random.default_rng(23)
    kb, vb, kv, vv, bt, qs, q = _setup(rng, [64], [40], 4, 2, 8)
    whole = attention.prefill_paged(q, kb, vb, bt, qs, [64], 0.4, 2, "f16")
    first = attention.prefill_paged(q[:25], kb, vb, bt, [0, 25], [49], 0.4, 2, "f16")
    second = attention.prefill_paged(q[25:], kb, vb, bt, [0, 15], [64], 0.4, 2, "f16")
    assert np.array_equal(whole, np.concatenate([first, second]))
