"""Oracle-side view of a seeded workload: expected block tables, pools and outputs.

Everything here is computed by ``oracle/`` from the draws of ``workloads``; no
value comes from the CUDA path. The GPU tests compare the device's block
tables, pool bytes and outputs against these.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np
import torch

import workloads as W
from oracle import attention, cache, e4m3, paging


def bits16(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of an f16/bf16 tensor."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def values64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 values of an f16/bf16/f32 tensor."""
    return t.to(torch.float64).numpy()


@dataclasses.dataclass
class OracleCase:
    w: W.Workload
    lens: np.ndarray
    order: np.ndarray
    block_tables: np.ndarray
    q: np.ndarray  # float64 [B, Hq, D]
    k_scale: float
    v_scale: float
    k_logical: List[np.ndarray]  # float64 [ctx, Hkv, D] per sequence, as stored (dequantised for e4m3)
    v_logical: List[np.ndarray]
    k_pool: Optional[np.ndarray] = None  # expected bytes after the whole history + new token
    v_pool: Optional[np.ndarray] = None
    new_slots: Optional[np.ndarray] = None


def _stored_values(src: torch.Tensor, kv_dtype: str, scale: float) -> np.ndarray:
    if kv_dtype == "e4m3":
        return e4m3.dequantize(e4m3.quantize(src.float().numpy(), scale), scale)
    return values64(src)


def _src_bytes(src: torch.Tensor, kv_dtype: str):
    return src.float().numpy() if kv_dtype == "e4m3" else bits16(src)


def build(w: W.Workload, with_pools: bool = True) -> OracleCase:
    lens_t = W.context_lens(w)
    lens = lens_t.numpy().astype(np.int64)
    order = W.block_order(w).numpy()
    mb = W.max_blocks_per_seq(w, lens_t)
    bt = paging.build_block_tables(lens, order, w.num_blocks, w.block_size, w.shared_prefix_tokens, mb)
    q = values64(W.query(w))
    k_scale, v_scale = W.fp8_scales(w)
    k_src = [W.kv_source(w, s, "k", lens_t) for s in range(w.num_seqs)]
    v_src = [W.kv_source(w, s, "v", lens_t) for s in range(w.num_seqs)]
    case = OracleCase(w, lens, order, bt, q, k_scale, v_scale,
                      [_stored_values(k, w.kv_dtype, k_scale) for k in k_src],
                      [_stored_values(v, w.kv_dtype, v_scale) for v in v_src])
    if with_pools:
        sent = W.sentinel_pool(w, "sentinel/k").numpy()
        sent_v = W.sentinel_pool(w, "sentinel/v").numpy()
        seqs, poss, rows_k, rows_v = [], [], [], []
        for s in range(w.num_seqs):
            n = int(lens[s])
            # History rows 0..n-2, then the new token at n-1 (written last).
            # Shared-prefix rows are written once, by sequence 0.
            start = 0 if s == 0 else w.shared_prefix_tokens
            for p in range(start, n):
                seqs.append(s)
                poss.append(p)
            rows_k.append(_src_bytes(k_src[s][start:n], w.kv_dtype))
            rows_v.append(_src_bytes(v_src[s][start:n], w.kv_dtype))
        slots = paging.slots_for_positions(bt, seqs, poss, w.block_size)
        case.k_pool, case.v_pool = cache.reshape_and_cache(
            np.concatenate(rows_k), np.concatenate(rows_v), slots, sent, sent_v, w.kv_dtype, k_scale, v_scale,
            w.block_size)
        case.new_slots = paging.slots_for_positions(bt, range(w.num_seqs), [int(n) - 1 for n in lens],
                                                    w.block_size)
    return case


def expected_out(case: OracleCase) -> np.ndarray:
    """Path A: the definition over each sequence's logical rows."""
    return attention.decode_logical(case.q, case.k_logical, case.v_logical, case.w.scale, case.w.num_kv_heads)


def expected_out_paged(case: OracleCase) -> np.ndarray:
    """Path B: the same through the oracle's own pool and block tables."""
    w = case.w
    return attention.decode_paged(case.q, case.k_pool, case.v_pool, case.block_tables, case.lens, w.scale,
                                  w.num_kv_heads, w.kv_dtype, case.k_scale, case.v_scale, w.block_size)


def _all_bf16_values() -> np.ndarray:
    """Every bf16 bit pattern 0 .. 65535, as the float32 value it holds (index = bit pattern)."""
    bits = np.arange(65536, dtype=np.uint32) << 16
    return bits.view(np.float32)


_CODE_TABLES = {}


def e4m3_codes_of_bf16(src: torch.Tensor, scale: float) -> np.ndarray:
    """``oracle.e4m3.quantize(src, scale)`` for a bf16 source, looked up by the source's bits.

    quantize acts on each element alone, and a bf16 element holds one of 65536 bit patterns, so
    evaluating quantize once on every pattern and indexing that table by the source's bits gives
    exactly quantize's codes (``tests/test_oracle_e4m3.py`` checks the two agree). Full-size workloads
    hold ~10^9 elements, which the element-wise codec would take many minutes over.
    """
    assert src.dtype == torch.bfloat16
    key = float(scale)
    if key not in _CODE_TABLES:
        _CODE_TABLES[key] = e4m3.quantize(_all_bf16_values(), scale)
    return _CODE_TABLES[key][bits16(src)]


def e4m3_values(codes: np.ndarray, scale: float) -> np.ndarray:
    """``oracle.e4m3.dequantize(codes, scale)`` by lookup in its value at each of the 256 codes."""
    table = e4m3.dequantize(np.arange(256, dtype=np.uint8), scale)
    return table[codes]
