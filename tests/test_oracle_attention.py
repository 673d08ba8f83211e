"""Pins of the oracle's decode against things other than itself (CPU only).

Each ``check_*`` raises AssertionError on a mismatch; ``test_oracle_mutations``
plants plausible mistakes in the oracle and shows these checks catch them.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention, paging
from tests import oracle_case


def _random_pools(rng, nb, hkv, d, dtype="f16"):
    vals = rng.standard_normal((nb, hkv, 16, d)).astype(np.float16)
    return vals.view(np.uint8).reshape(nb, hkv, 16, d * 2), vals.astype(np.float64)


def _case(rng, lens, hq, hkv, d, nb=None):
    """Random pools + oracle-built block tables for the given context lengths."""
    need = sum(-(-n // 16) for n in lens)
    nb = nb or need + 7
    kb, kv = _random_pools(rng, nb, hkv, d)
    vb, vv = _random_pools(rng, nb, hkv, d)
    order = rng.permutation(nb)
    bt = paging.build_block_tables(lens, order, nb, 16, 0, max(1, max(-(-n // 16) for n in lens)))
    q = rng.standard_normal((len(lens), hq, d))
    return kb, vb, kv, vv, bt, q


def check_vs_sdpa(decode_paged=attention.decode_paged, seed=0):
    """Equals torch's scaled_dot_product_attention (float64, GQA via enable_gqa) on the gathered context."""
    rng = np.random.default_rng(seed)
    for lens, hq, hkv, d in [([5, 16, 17, 40], 4, 4, 8), ([33, 1, 70], 8, 2, 16), ([31, 64], 6, 1, 8)]:
        kb, vb, kv, vv, bt, q = _case(rng, lens, hq, hkv, d)
        scale = 1.0 / math.sqrt(d) * 1.3
        got = decode_paged(q, kb, vb, bt, lens, scale, hkv, "f16")
        for s, n in enumerate(lens):
            blocks = [bt[s][t // 16] for t in range(n)]
            K = torch.tensor(np.stack([kv[blocks[t], :, t % 16, :] for t in range(n)]))  # [n, Hkv, D]
            V = torch.tensor(np.stack([vv[blocks[t], :, t % 16, :] for t in range(n)]))
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.tensor(q[s])[None, :, None, :], K.permute(1, 0, 2)[None], V.permute(1, 0, 2)[None],
                scale=scale, enable_gqa=True)[0, :, 0, :].numpy()
            np.testing.assert_allclose(got[s], ref, rtol=0, atol=1e-12)


def check_bruteforce(attend=attention.attend, seed=1):
    """Equals explicit per-score loops (math.exp, no max subtraction, fsum) on D=4, ctx <= 20."""
    rng = np.random.default_rng(seed)
    for n in [1, 2, 3, 7, 16, 20]:
        q = rng.standard_normal(4)
        K = rng.standard_normal((n, 4))
        V = rng.standard_normal((n, 4))
        scale = 0.7
        w = [math.exp(scale * sum(q[i] * K[t][i] for i in range(4))) for t in range(n)]
        z = math.fsum(w)
        ref = [math.fsum(w[t] * V[t][i] for t in range(n)) / z for i in range(4)]
        np.testing.assert_allclose(attend(q, K, V, scale), ref, rtol=1e-13, atol=1e-14)


def check_hand_example(golden, attend=attention.attend):
    rows = {r[0]: [float(x) for x in r[1:]] for r in golden("attention_hand_example.txt")}
    K = np.array([rows["K0"], rows["K1"]])
    V = np.array([rows["V0"], rows["V1"]])
    np.testing.assert_allclose(attend(np.array(rows["q"]), K, V, 1.0), rows["out"], rtol=0, atol=1e-14)


def check_gqa_mapping(decode_paged=attention.decode_paged):
    """Query head h reads KV head h // G: with V constant c_hk per KV head, out[h] == c_{h // G}."""
    rng = np.random.default_rng(5)
    lens, hq, hkv, d = [37, 5], 8, 2, 8
    kb, vb, kv, vv, bt, q = _case(rng, lens, hq, hkv, d)
    consts = np.array([3.0, -5.0])
    vvals = np.broadcast_to(consts[None, :, None, None], vv.shape).astype(np.float16)
    vb = np.ascontiguousarray(vvals).view(np.uint8).reshape(vb.shape)
    got = decode_paged(q, kb, vb, bt, lens, 0.3, hkv, "f16")
    for h in range(hq):
        np.testing.assert_allclose(got[:, h, :], consts[h // (hq // hkv)], rtol=0, atol=1e-13)


def test_hand_example(golden):
    check_hand_example(golden)


def test_vs_sdpa():
    check_vs_sdpa()


def test_bruteforce():
    check_bruteforce()


def test_gqa_mapping():
    check_gqa_mapping()


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(2)
    n, d = 37, 8
    K = np.tile(rng.standard_normal(d), (n, 1))
    V = rng.standard_normal((n, d))
    np.testing.assert_allclose(attention.attend(rng.standard_normal(d), K, V, 0.9), V.mean(axis=0),
                               rtol=0, atol=1e-14)


def test_zero_scale_gives_mean_of_values():
    rng = np.random.default_rng(3)
    K, V = rng.standard_normal((20, 8)), rng.standard_normal((20, 8))
    np.testing.assert_allclose(attention.attend(rng.standard_normal(8), K, V, 0.0), V.mean(axis=0), atol=1e-14)


def test_single_token_returns_its_value_exactly():
    rng = np.random.default_rng(4)
    V = rng.standard_normal((1, 8))
    assert np.array_equal(attention.attend(rng.standard_normal(8), rng.standard_normal((1, 8)), V, 0.5), V[0])


def test_dominant_key_returns_its_value():
    rng = np.random.default_rng(6)
    n, d = 50, 16
    q = rng.standard_normal(d)
    K = rng.standard_normal((n, d)) * 0.1
    V = rng.standard_normal((n, d))
    for p in [0, 17, n - 1]:
        K2 = K.copy()
        K2[p] = 80.0 * q / np.linalg.norm(q) ** 2  # score 80 vs others ~O(1)
        # The other weights are below exp(-70) relative to the dominant one.
        np.testing.assert_allclose(attention.attend(q, K2, V, 1.0), V[p], rtol=0, atol=1e-25)


def test_empty_context_is_zero():
    assert np.array_equal(attention.attend(np.ones(4), np.zeros((0, 4)), np.zeros((0, 4)), 1.0), np.zeros(4))


@pytest.mark.parametrize("name", ["tiny", "llama7b_mha_small", "llama3_8b_gqa_small", "prefix_gqa_small",
                                  "long70b_fp8_small", "mqa_small", "d64_gqa_small"])
def test_pool_path_equals_logical_path_bitwise(name):
    """Path B (through the oracle's scattered pool) == path A (logical rows), bit for bit."""
    case = oracle_case.build(W.ALL[name])
    a = oracle_case.expected_out(case)
    b = oracle_case.expected_out_paged(case)
    assert np.array_equal(a, b)


def test_result_independent_of_physical_placement():
    rng = np.random.default_rng(7)
    lens, hq, hkv, d = [45, 16, 3], 4, 2, 8
    kb, vb, kv, vv, bt, q = _case(rng, lens, hq, hkv, d, nb=30)
    out1 = attention.decode_paged(q, kb, vb, bt, lens, 0.4, hkv, "f16")
    # Move every used block to another physical id (a permutation of the pool) and rebuild the table.
    perm = rng.permutation(30)
    kb2 = np.empty_like(kb)
    vb2 = np.empty_like(vb)
    kb2[perm] = kb
    vb2[perm] = vb
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    out2 = attention.decode_paged(q, kb2, vb2, bt2, lens, 0.4, hkv, "f16")
    assert np.array_equal(out1, out2)
