"""reshape_and_cache of the oracle: scatter new tokens' K/V into their slots (test infrastructure).

Source: vLLM pages, "PagedAttention / Cache Engine" (dingiv.github.io/ai/compute/engine/vllm):
the Cache Engine computes the page of a position and reads or writes that page's
data. The write side, for one token, is: find its slot, store its K and V there.

Readings taken where the pages are silent:
* pool layout [num_blocks, num_kv_heads, block_size, head_dim] per cache (K and
  V separate), so one (block, head) page is one contiguous run;
* slot -1 means "skip this token";
* 16-bit caches store the value bits unchanged; an e4m3 cache stores
  ``e4m3.quantize(x, scale)`` (see ``oracle.e4m3``);
* untouched slots keep their bytes.

The pools are numpy arrays of raw bytes [num_blocks, Hkv, block_size, D * elem],
so the comparison with the device pool is byte for byte.
"""
from __future__ import annotations

import numpy as np

from . import e4m3


def _token_bytes(x_row: np.ndarray, kv_dtype: str, scale: float) -> np.ndarray:
    """Bytes one token's [Hkv, D] row takes in the pool: [Hkv, D * elem] uint8."""
    if kv_dtype == "e4m3":
        assert x_row.dtype == np.float32
        return e4m3.quantize(x_row, scale)
    assert x_row.dtype == np.uint16
    return np.ascontiguousarray(x_row).view(np.uint8)


def reshape_and_cache(key_bits: np.ndarray, value_bits: np.ndarray, slots, k_pool: np.ndarray,
                      v_pool: np.ndarray, kv_dtype: str, k_scale: float = 1.0, v_scale: float = 1.0,
                      block_size: int = 16):
    """Return new (k_pool, v_pool) with token t's K/V stored at slot ``slots[t]``.

    ``key_bits``/``value_bits`` are [T, Hkv, D]. For a 16-bit cache they are the
    raw uint16 bit patterns of the f16/bf16 values (stored unchanged); for an
    e4m3 cache they are float32 arrays holding the source values exactly.
    """
    k_out = k_pool.copy()
    v_out = v_pool.copy()
    for t, slot in enumerate(np.asarray(slots, dtype=np.int64).tolist()):
        if slot < 0:
            continue
        blk, off = slot // block_size, slot % block_size
        k_out[blk, :, off, :] = _token_bytes(key_bits[t], kv_dtype, k_scale)
        v_out[blk, :, off, :] = _token_bytes(value_bits[t], kv_dtype, v_scale)
    return k_out, v_out


def pool_values(pool: np.ndarray, kv_dtype: str, scale: float = 1.0) -> np.ndarray:
    """Interpret a byte pool [NB, Hkv, BS, D * elem] as float64 values [NB, Hkv, BS, D]."""
    if kv_dtype == "f16":
        return pool.view(np.float16).astype(np.float64)
    if kv_dtype == "bf16":
        u16 = pool.view(np.uint16).astype(np.uint32) << 16
        return u16.view(np.float32).astype(np.float64)
    if kv_dtype == "e4m3":
        return e4m3.dequantize(pool, scale)
    raise ValueError(kv_dtype)


def copy_blocks(k_pool: np.ndarray, v_pool: np.ndarray, mapping):
    """Return new pools where block dst holds block src's bytes, for each (src, dst) pair.

    The pairs are applied to the pools as they were before the call (all sources read first), the
    reading the copy kernel implements for mappings whose destinations are distinct and are not
    also sources.
    """
    k_out = k_pool.copy()
    v_out = v_pool.copy()
    for src, dst in np.asarray(mapping, dtype=np.int64).reshape(-1, 2).tolist():
        k_out[dst] = k_pool[src]
        v_out[dst] = v_pool[src]
    return k_out, v_out
