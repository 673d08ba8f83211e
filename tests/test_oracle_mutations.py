"""Plant plausible mistakes in copies of the oracle (on the CPU) and show the pins catch each one.

A pin that no plausible mistake can fail pins nothing; each case below swaps
one oracle function for a subtly wrong variant and expects a named check to
raise.
"""
import numpy as np
import pytest

from oracle import attention, cache, e4m3, paging
from tests import test_oracle_attention as TA
from tests import test_oracle_e4m3 as TE
from tests import test_oracle_paging as TP


def _decode_paged_with(attend=attention.attend, gather=attention.gather_context, kv_head_of=None):
    def decode(q, k_pool, v_pool, bt, lens, scale, hkv, kv_dtype, k_scale=1.0, v_scale=1.0, block_size=16):
        q = np.asarray(q, dtype=np.float64)
        B, Hq, D = q.shape
        out = np.zeros((B, Hq, D))
        for s in range(B):
            for h in range(Hq):
                hk = kv_head_of(h, Hq, hkv) if kv_head_of else h // (Hq // hkv)
                K = gather(k_pool, bt[s], int(lens[s]), hk, kv_dtype, k_scale, block_size)
                V = gather(v_pool, bt[s], int(lens[s]), hk, kv_dtype, v_scale, block_size)
                out[s, h] = attend(q[s, h], K, V, scale)
        return out
    return decode


def test_reference_decoder_passes():
    TA.check_vs_sdpa(_decode_paged_with())
    TA.check_gqa_mapping(_decode_paged_with())


def test_gqa_interleaved_mapping_is_caught():
    with pytest.raises(AssertionError):
        TA.check_gqa_mapping(_decode_paged_with(kv_head_of=lambda h, hq, hkv: h % hkv))


def test_dropped_scale_is_caught():
    with pytest.raises(AssertionError):
        TA.check_vs_sdpa(_decode_paged_with(attend=lambda q, K, V, s: attention.attend(q, K, V, 1.0)))


def test_swapped_k_and_v_is_caught():
    def swapped(q, K, V, s):
        return attention.attend(q, V, K, s)
    with pytest.raises(AssertionError):
        TA.check_bruteforce(swapped)


def test_transposed_score_product_is_caught(golden):
    def wrong(q, K, V, s):
        K = np.asarray(K, dtype=np.float64)
        V = np.asarray(V, dtype=np.float64)
        w = np.exp(s * (K @ q))
        return (V @ w) / w.sum()  # contracts V over the wrong axis (same shape when n == D)
    with pytest.raises(AssertionError):
        TA.check_hand_example(golden, wrong)


def test_off_by_one_page_is_caught():
    def gather(pool, row, n, hk, kv_dtype, scale=1.0, bs=16):
        t = np.arange(n)
        blocks = row[np.minimum((t + 1) // bs, len(row) - 1)].astype(np.int64)
        return cache.pool_values(pool[np.maximum(blocks, 0), hk, t % bs, :], kv_dtype, scale)
    with pytest.raises(AssertionError):
        TA.check_vs_sdpa(_decode_paged_with(gather=gather))


def test_offset_from_wrong_end_is_caught():
    def gather(pool, row, n, hk, kv_dtype, scale=1.0, bs=16):
        t = np.arange(n)
        return cache.pool_values(pool[row[t // bs].astype(np.int64), hk, bs - 1 - t % bs, :], kv_dtype, scale)
    with pytest.raises(AssertionError):
        TA.check_vs_sdpa(_decode_paged_with(gather=gather))


def test_page_index_rounding_up_is_caught(golden):
    with pytest.raises(AssertionError):
        TP.check_page_index(golden, lambda p, bs=16: -(-p // bs))


def test_slot_using_block_times_position_is_caught(golden):
    with pytest.raises(AssertionError):
        TP.check_slots(golden, lambda row, p, bs=16: int(row[p // bs]) * bs + p // bs)


def test_e4m3_bias_8_is_caught(golden):
    def decode(codes):
        return e4m3.decode(codes) / 2.0
    with pytest.raises(AssertionError):
        TE.check_spec_values(golden, decode=decode)


def test_e4m3_round_toward_zero_is_caught():
    def encode(x):
        v = np.asarray(x, dtype=np.float64)
        c = e4m3.encode(v)
        back = e4m3.decode(c)
        too_big = np.abs(back) > np.abs(v)
        return np.where(too_big & (c & 0x7F > 0), c - 1, c).astype(np.uint8)
    with pytest.raises(AssertionError):
        TE.check_encode_vs_torch(encode)


def test_e4m3_no_subnormals_is_caught():
    def decode(codes):
        c = np.asarray(codes, dtype=np.uint8)
        v = e4m3.decode(c)
        return np.where((c & 0x78) == 0, 0.0, v) * np.where(c & 0x80, -1, 1) * np.where(c & 0x80, -1, 1)
    with pytest.raises(AssertionError):
        TE.check_decode_vs_torch(decode)


def test_free_list_never_reusing_is_caught():
    class Leaky(paging.FreeListModel):
        def free(self, b):
            if not (0 <= b < self.num_blocks) or self._ref[b] == 0:
                return False
            self._ref[b] -= 1
            return True  # forgets to push the block back
    with pytest.raises(AssertionError):
        fl = Leaky(3)
        a = fl.alloc()
        fl.free(a)
        assert fl.num_free == 3


def test_prefill_without_causal_mask_is_caught():
    from tests import test_oracle_prefill as TPF

    def no_mask(q, k_pool, v_pool, bt, qs, lens, scale, hkv, kv_dtype, block_size=16):
        q = np.asarray(q, dtype=np.float64)
        out = np.zeros_like(q)
        G = q.shape[1] // hkv
        for s in range(len(lens)):
            n = int(lens[s])
            for hk in range(hkv):
                K = attention.gather_context(k_pool, bt[s], n, hk, kv_dtype)
                V = attention.gather_context(v_pool, bt[s], n, hk, kv_dtype)
                for r in range(int(qs[s]), int(qs[s + 1])):
                    for h in range(hk * G, (hk + 1) * G):
                        out[r, h] = attention.attend(q[r, h], K, V, scale)  # every key, no diagonal
        return out
    with pytest.raises(AssertionError):
        TPF.check_prefill_vs_sdpa(no_mask)


def test_prefill_excluding_the_diagonal_is_caught():
    from tests import test_oracle_prefill as TPF

    def strict(q, k_pool, v_pool, bt, qs, lens, scale, hkv, kv_dtype, block_size=16):
        q = np.asarray(q, dtype=np.float64)
        out = np.zeros_like(q)
        G = q.shape[1] // hkv
        for s in range(len(lens)):
            n = int(lens[s])
            start = n - (int(qs[s + 1]) - int(qs[s]))
            for hk in range(hkv):
                K = attention.gather_context(k_pool, bt[s], n, hk, kv_dtype)
                V = attention.gather_context(v_pool, bt[s], n, hk, kv_dtype)
                for i, r in enumerate(range(int(qs[s]), int(qs[s + 1]))):
                    p = max(start + i, 1)
                    for h in range(hk * G, (hk + 1) * G):
                        out[r, h] = attention.attend(q[r, h], K[:p], V[:p], scale)  # misses itself
        return out
    with pytest.raises(AssertionError):
        TPF.check_prefill_vs_sdpa(strict)
