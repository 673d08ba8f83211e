"""Pins of the oracle's reshape_and_cache scatter and pool interpretation (CPU only)."""
import numpy as np
import torch

from oracle import attention, cache, e4m3, paging


def _pools(rng, nb, hkv, d, elem):
    k = rng.integers(0, 256, (nb, hkv, 16, d * elem), dtype=np.uint8)
    v = rng.integers(0, 256, (nb, hkv, 16, d * elem), dtype=np.uint8)
    return k, v


def test_scatter_writes_only_the_slots_and_reads_back():
    rng = np.random.default_rng(0)
    nb, hkv, d = 12, 3, 8
    k0, v0 = _pools(rng, nb, hkv, d, 2)
    key = torch.randn(5, hkv, d, dtype=torch.float32).to(torch.float16)
    val = torch.randn(5, hkv, d, dtype=torch.float32).to(torch.float16)
    slots = np.array([37, -1, 0, 191, 100], dtype=np.int64)
    kb = key.view(torch.int16).numpy().view(np.uint16)
    vb = val.view(torch.int16).numpy().view(np.uint16)
    k1, v1 = cache.reshape_and_cache(kb, vb, slots, k0, v0, "f16")
    touched = np.zeros((nb, hkv, 16), dtype=bool)
    for t, s in enumerate(slots):
        if s < 0:
            continue
        blk, off = s // 16, s % 16
        touched[blk, :, off] = True
        assert np.array_equal(cache.pool_values(k1[blk, :, off], "f16"), key[t].double().numpy())
        assert np.array_equal(cache.pool_values(v1[blk, :, off], "f16"), val[t].double().numpy())
    assert np.array_equal(k1[~touched], k0[~touched])
    assert np.array_equal(v1[~touched], v0[~touched])


def test_bf16_pool_values_match_torch():
    x = torch.randn(4, 2, 16, 8).to(torch.bfloat16)
    b = x.view(torch.int16).numpy().view(np.uint8).reshape(4, 2, 16, 16)
    assert np.array_equal(cache.pool_values(b, "bf16"), x.double().numpy())


def test_e4m3_scatter_and_read_back_through_block_table():
    rng = np.random.default_rng(1)
    nb, hkv, d = 9, 2, 16
    k0, v0 = _pools(rng, nb, hkv, d, 1)
    n = 40
    bt = paging.build_block_tables([n], rng.permutation(nb), nb)
    src_k = torch.randn(n, hkv, d).to(torch.bfloat16).float().numpy()
    src_v = torch.randn(n, hkv, d).to(torch.bfloat16).float().numpy()
    slots = paging.slots_for_positions(bt, [0] * n, range(n))
    ks, vs = 0.0123, 0.02
    k1, v1 = cache.reshape_and_cache(src_k, src_v, slots, k0, v0, "e4m3", ks, vs)
    for hk in range(hkv):
        K = attention.gather_context(k1, bt[0], n, hk, "e4m3", ks)
        assert np.array_equal(K, e4m3.dequantize(e4m3.quantize(src_k[:, hk], ks), ks))
        V = attention.gather_context(v1, bt[0], n, hk, "e4m3", vs)
        assert np.array_equal(V, e4m3.dequantize(e4m3.quantize(src_v[:, hk], vs), vs))


def test_copy_blocks_copies_whole_blocks_only():
    rng = np.random.default_rng(9)
    k0, v0 = _pools(rng, 10, 3, 8, 2)
    mapping = [(2, 7), (5, 0), (9, 9)]
    k1, v1 = cache.copy_blocks(k0, v0, mapping)
    for src, dst in mapping:
        assert np.array_equal(k1[dst], k0[src]) and np.array_equal(v1[dst], v0[src])
    untouched = [b for b in range(10) if b not in (7, 0)]
    assert np.array_equal(k1[untouched], k0[untouched]) and np.array_equal(v1[untouched], v0[untouched])
