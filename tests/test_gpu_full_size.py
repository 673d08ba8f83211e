"""Full-size parity: every output element and every pool byte of the four large workloads (GPU).

Each workload runs at its full size in the launch configuration the bench times: one
``pa_decode_step`` (the new token's write fused into the decode launch) with the workload's
partitioning (512-token partitions for the long-context e4m3 batch, the library's choice otherwise),
and for the shared-prefix batch also ``pa_decode_cascade`` with each prefix kernel. Then:

* every (sequence, query head, d) output is compared with the float64 oracle's plain definition over
  that sequence's logical rows, within the stated tolerance (e4m3: against the oracle's own
  dequantised values);
* every byte of both pools is compared with the oracle's scatter of the whole history and the new
  tokens onto the same seeded sentinel bytes (untouched slots included);
* the block tables equal the oracle's free-list model, and the device error word stays clear.

The oracle works one sequence at a time so host memory stays bounded. For the e4m3 cache the
oracle's codec is applied through a lookup on the bf16 source bits (``oracle_case.e4m3_codes_of_bf16``,
exact: see its docstring), and its codes reach the pool through the oracle's scatter as raw bytes.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_385_b200 as pa
import workloads as W
from oracle import attention, cache, paging
from tests import oracle_case
from tests.device_case import TOL, DeviceCase

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _stored(w, src, scale):
    """(pool bytes [n, Hkv, D * elem] as uint8, stored float64 values [n, Hkv, D]) of source rows."""
    if w.kv_dtype == "e4m3":
        codes = oracle_case.e4m3_codes_of_bf16(src, scale)
        return codes, oracle_case.e4m3_values(codes, scale)
    bits = oracle_case.bits16(src)
    return bits.view(np.uint8).reshape(src.shape[0], w.num_kv_heads, -1), oracle_case.values64(src)


def _oracle_sweep(w, dev):
    """Expected outputs [B, Hq, D] (float64) and expected pools, one sequence at a time."""
    lens = dev.lens_host
    q = oracle_case.values64(W.query(w))
    want = np.zeros(q.shape, dtype=np.float64)
    rows_k, rows_v, seqs, poss = [], [], [], []
    for s in range(w.num_seqs):
        n = int(lens[s])
        kb, K = _stored(w, W.kv_source(w, s, "k", lens), dev.k_scale)
        vb, V = _stored(w, W.kv_source(w, s, "v", lens), dev.v_scale)
        for h in range(w.num_q_heads):
            want[s, h] = attention.decode_logical_one(q[s, h], K, V, h, w.num_q_heads, w.num_kv_heads, w.scale)
        # Pool rows: history and new token of this sequence; shared-prefix rows once (sequence 0).
        start = 0 if s == 0 else w.shared_prefix_tokens
        rows_k.append(kb[start:n])
        rows_v.append(vb[start:n])
        seqs += [s] * (n - start)
        poss += list(range(start, n))
    slots = paging.slots_for_positions(dev.bt_host.numpy(), seqs, poss, w.block_size)
    # The oracle's scatter stores the bytes of a 16-bit row unchanged; e4m3 codes (already the
    # oracle's quantize) travel that path as byte pairs.
    as16 = lambda rows: np.ascontiguousarray(np.concatenate(rows)).view(np.uint16)  # noqa: E731
    sent_k = W.sentinel_pool(w, "sentinel/k").numpy()
    sent_v = W.sentinel_pool(w, "sentinel/v").numpy()
    k_pool, v_pool = cache.reshape_and_cache(as16(rows_k), as16(rows_v), slots, sent_k, sent_v, "f16", 1.0, 1.0,
                                             w.block_size)
    return want, k_pool, v_pool


def _check_out(out, want, w, what):
    got = out.double().cpu().numpy()
    err = np.abs(got - want)
    worst = float(err.max())
    assert np.isfinite(got).all(), what
    assert worst <= TOL[w.kv_dtype], f"{what}: max abs err {worst} at {np.unravel_index(err.argmax(), err.shape)}"


@pytest.mark.parametrize("name", ["llama7b_mha", "llama3_8b_gqa", "long70b_fp8"])
def test_full_size_step_every_output_and_pool_byte(name):
    w = W.FULL[name]
    dev = DeviceCase(w)  # history written by pa_reshape_and_cache onto the seeded sentinel bytes
    bt_o = paging.build_block_tables(dev.lens_host.numpy(), W.block_order(w).numpy(), w.num_blocks, w.block_size,
                                     w.shared_prefix_tokens, dev.max_blocks)
    assert np.array_equal(dev.bt_host.numpy(), bt_o)
    out = dev.step_fused().clone()  # the bench's launch: new-token write + decode (+ merge), w's partitioning
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    want, k_pool, v_pool = _oracle_sweep(w, dev)
    _check_out(out, want, w, name)
    k, v = dev.pool_bytes()
    assert np.array_equal(k, k_pool), f"K pool differs at {np.argwhere(k != k_pool)[:4]}"
    assert np.array_equal(v, v_pool), f"V pool differs at {np.argwhere(v != v_pool)[:4]}"


def test_full_size_prefix_workload_every_output_and_pool_byte():
    """The shared-prefix batch: plain fused step, and the cascade with each prefix kernel."""
    w = W.FULL["prefix_gqa"]
    dev = DeviceCase(w)
    bt_o = paging.build_block_tables(dev.lens_host.numpy(), W.block_order(w).numpy(), w.num_blocks, w.block_size,
                                     w.shared_prefix_tokens, dev.max_blocks)
    assert np.array_equal(dev.bt_host.numpy(), bt_o)
    outs = {"pa_decode_step": dev.step_fused().clone()}
    for pk in (1, 0):  # tcgen05, warp-level mma; the new token is rewritten with the same bytes
        outs[f"pa_decode_cascade prefix_kernel={pk}"] = dev.cascade(fused=True, prefix_kernel=pk).clone()
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    want, k_pool, v_pool = _oracle_sweep(w, dev)
    for what, out in outs.items():
        _check_out(out, want, w, what)
    k, v = dev.pool_bytes()
    assert np.array_equal(k, k_pool), f"K pool differs at {np.argwhere(k != k_pool)[:4]}"
    assert np.array_equal(v, v_pool), f"V pool differs at {np.argwhere(v != v_pool)[:4]}"


def test_full_size_prefill_sampled_rows():
    """The prefill the bench times (8 sequences x 2048-token prompts, Llama-3-8B heads 32/8, D=128,
    bf16, the library's kernel choice: the persistent tcgen05 kernel with 16 items per CTA) against the
    oracle's row definition on sampled rows: the first and last tokens of every sequence, tokens on
    either side of a 128-row tile edge and inside the causal diagonal block, for query heads at both
    ends of a KV group. The oracle reads the host K/V draws; every output is checked finite."""
    B, n, Hq, Hkv, D = 8, 2048, 32, 8, 128
    g = torch.Generator().manual_seed(4242)
    nb = B * n // 16 + 9
    order = torch.randperm(nb, generator=g)
    alloc = pa.BlockAllocator(nb, order.tolist())
    bt = pa.build_block_tables(alloc, [n] * B, n // 16)
    assert np.array_equal(bt.numpy(), paging.build_block_tables([n] * B, order.numpy(), nb, 16, 0, n // 16))
    K = torch.randn(B * n, Hkv, D, generator=g).to(torch.bfloat16)
    V = torch.randn(B * n, Hkv, D, generator=g).to(torch.bfloat16)
    q = torch.randn(B * n, Hq, D, generator=g).to(torch.bfloat16)
    kc = torch.randint(0, 256, (nb, Hkv, 16, 2 * D), generator=g, dtype=torch.uint8).view(torch.bfloat16)
    kc = kc.view(nb, Hkv, 16, D).cuda()
    vc = torch.randint(0, 256, (nb, Hkv, 16, 2 * D), generator=g, dtype=torch.uint8).view(torch.bfloat16)
    vc = vc.view(nb, Hkv, 16, D).cuda()
    seqs = [s for s in range(B) for _ in range(n)]
    poss = [t for _ in range(B) for t in range(n)]
    pa.pa_reshape_and_cache(K.cuda(), V.cuda(), pa.pa_slots_for_positions(bt, seqs, poss).cuda(), kc, vc)
    out = torch.full((B * n, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    qs = torch.arange(0, B * n + 1, n, dtype=torch.int32).cuda()
    lens = torch.full((B,), n, dtype=torch.int32).cuda()
    pa.pa_prefill(out, q.cuda(), kc, vc, bt.cuda(), qs, lens, n, D ** -0.5, Hkv)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    got = out.float().cpu()
    assert torch.isfinite(got).all()
    worst = 0.0
    for s in range(B):
        Kd = oracle_case.values64(K[s * n:(s + 1) * n])
        Vd = oracle_case.values64(V[s * n:(s + 1) * n])
        for t in (0, 1, 31, 32, 1023, 1024, 2015, 2047):  # 32 tokens x 4 heads = one 128-row tile
            qd = oracle_case.values64(q[s * n + t])
            for h in (0, 3, 4, 31):
                want = attention.decode_logical_one(qd[h], Kd[:t + 1], Vd[:t + 1], h, Hq, Hkv, D ** -0.5)
                worst = max(worst, float(np.max(np.abs(got[s * n + t, h].double().numpy() - want))))
    assert worst <= TOL["bf16"], worst
