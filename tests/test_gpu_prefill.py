"""GPU parity of chunked prefill (pa_prefill) against the float64 oracle's causal definition."""
import numpy as np
import pytest
import torch

import paged_kv_cache_385_b200 as pa
from oracle import attention, cache, paging
from tests import oracle_case
from tests.device_case import TOL

pytestmark = pytest.mark.gpu


def _build(ctxs, news, hq, hkv, d, dtype, seed, order_seed=None):
    """Device state through the library, and the oracle's pools from the same host draws.

    The oracle's block tables come from its own free-list model and its pools from its own scatter
    of the host K/V rows onto the host sentinel bytes; nothing the GPU wrote feeds the oracle.
    ``order_seed`` picks the free list's initial order (the physical placement) independently of
    the values, so two placements of the same logical data can be compared.
    """
    g = torch.Generator().manual_seed(seed)
    B = len(ctxs)
    nb = sum(-(-c // 16) for c in ctxs) + 11
    go = g if order_seed is None else torch.Generator().manual_seed(order_seed)
    order = torch.randperm(nb, generator=go)
    alloc = pa.BlockAllocator(nb, order.tolist())
    mb = max(-(-c // 16) for c in ctxs)
    bt = pa.build_block_tables(alloc, ctxs, mb)
    bt_oracle = paging.build_block_tables(ctxs, order.numpy(), nb, 16, 0, mb)
    assert np.array_equal(bt.numpy(), bt_oracle)
    # Pools start as random bytes (NaN patterns included) so unwritten slots are never read.
    kb = torch.randint(0, 256, (nb, hkv, 16, d * 2), generator=g, dtype=torch.uint8)
    vb = torch.randint(0, 256, (nb, hkv, 16, d * 2), generator=g, dtype=torch.uint8)
    K = [torch.randn(c, hkv, d, generator=g).to(dtype) for c in ctxs]
    V = [torch.randn(c, hkv, d, generator=g).to(dtype) for c in ctxs]
    seqs = [s for s in range(B) for _ in range(ctxs[s])]
    poss = [p for s in range(B) for p in range(ctxs[s])]
    kc = kb.clone().view(dtype).view(nb, hkv, 16, d).cuda()
    vc = vb.clone().view(dtype).view(nb, hkv, 16, d).cuda()
    pa.pa_reshape_and_cache(torch.cat(K).cuda(), torch.cat(V).cuda(), pa.pa_slots_for_positions(bt, seqs, poss).cuda(),
                            kc, vc)
    slots = paging.slots_for_positions(bt_oracle, seqs, poss)
    kvd = "bf16" if dtype == torch.bfloat16 else "f16"
    pools = cache.reshape_and_cache(oracle_case.bits16(torch.cat(K)), oracle_case.bits16(torch.cat(V)), slots,
                                    kb.numpy(), vb.numpy(), kvd)
    qs = torch.tensor([0] + np.cumsum(news).tolist(), dtype=torch.int32)
    q = torch.randn(int(qs[-1]), hq, d, generator=g).to(dtype)
    return bt, kc, vc, q, qs, (bt_oracle, pools)


def _oracle(host, q, qs, ctxs, scale, hkv, kvd):
    """The oracle's causal attention over its own block tables and pools (see _build)."""
    bt_oracle, (kp, vp) = host
    return attention.prefill_paged(q.double().numpy(), kp, vp, bt_oracle, qs.tolist(), ctxs, scale, hkv, kvd)


CASES = [
    ([37, 160, 90], [37, 16, 70], 8, 2, 128, torch.bfloat16),
    ([1, 64, 200, 33], [1, 64, 5, 33], 4, 4, 64, torch.float16),
    ([300, 129], [150, 129], 16, 2, 128, torch.float16),
    ([700, 5, 260], [400, 5, 131], 32, 8, 128, torch.bfloat16),
    ([129, 40], [129, 40], 4, 4, 128, torch.float16),
    # Long enough (24 key blocks) that the S / P buffers of the tcgen05 kernel are reused many times.
    ([1500, 300], [1500, 100], 8, 2, 128, torch.bfloat16),
    # 696 row tiles x KV heads: more items than the persistent grid's 2 x SMs CTAs, so each CTA walks
    # two or three items and hands Q, O and its rings from one to the next.
    ([900, 1200, 640], [900, 600, 640], 32, 8, 128, torch.bfloat16),
    # Groups of 16 query heads (the largest the tcgen05 kernel takes: 8 tokens x 16 heads per tile),
    # chunks that end mid-tile, one sequence with a single new token.
    ([333, 70, 1], [101, 70, 1], 32, 2, 128, torch.float16),
    # A sequence with no new tokens in the batch (its items have no rows).
    ([50, 300, 10], [0, 200, 10], 8, 2, 128, torch.bfloat16),
]


@pytest.mark.parametrize("kernel", [0, 1])
@pytest.mark.parametrize("ctxs,news,hq,hkv,d,dtype", CASES)
def test_prefill_matches_oracle(ctxs, news, hq, hkv, d, dtype, kernel):
    if kernel == 1 and d != 128:
        pytest.skip("the tcgen05 prefill takes head_dim 128")
    bt, kc, vc, q, qs, host = _build(ctxs, news, hq, hkv, d, dtype, seed=sum(ctxs))
    out = torch.full((q.shape[0], hq, d), float("nan"), dtype=dtype, device="cuda")
    pa.pa_prefill(out, q.cuda(), kc, vc, bt.cuda(), qs.cuda(), torch.tensor(ctxs, dtype=torch.int32).cuda(),
                  max(news), 1.0 / np.sqrt(d), hkv, kernel=kernel)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    want = _oracle(host, q, qs, ctxs, 1.0 / np.sqrt(d), hkv, "bf16" if dtype == torch.bfloat16 else "f16")
    err = float(np.max(np.abs(out.double().cpu().numpy() - want)))
    assert err <= TOL["bf16" if dtype == torch.bfloat16 else "f16"], err
    # The pools the kernels read hold exactly the oracle's bytes, sentinels included.
    _, (kp, vp) = host
    assert np.array_equal(kc.view(torch.uint8).reshape(kp.shape).cpu().numpy(), kp)
    assert np.array_equal(vc.view(torch.uint8).reshape(vp.shape).cpu().numpy(), vp)


@pytest.mark.parametrize("kernel", [0, 1])
@pytest.mark.parametrize("scale", [-0.11, 0.0, 1.5])
def test_prefill_scale_sign_and_size(scale, kernel):
    """Negative and zero scales (the softmax max comes from the raw min, or every weight is equal) and
    a large one (scores spanning hundreds in log2 units: many raises of the running reference)."""
    ctxs, news, hq, hkv, d, dtype = [200, 70], [136, 70], 8, 2, 128, torch.float16
    bt, kc, vc, q, qs, host = _build(ctxs, news, hq, hkv, d, dtype, seed=77)
    out = torch.full((q.shape[0], hq, d), float("nan"), dtype=dtype, device="cuda")
    pa.pa_prefill(out, q.cuda(), kc, vc, bt.cuda(), qs.cuda(), torch.tensor(ctxs, dtype=torch.int32).cuda(),
                  max(news), scale, hkv, kernel=kernel)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    want = _oracle(host, q, qs, ctxs, scale, hkv, "f16")
    err = float(np.max(np.abs(out.double().cpu().numpy() - want)))
    assert err <= TOL["f16"], err


@pytest.mark.parametrize("kernel", [0, 1])
def test_prefill_with_a_loose_max_query_len(kernel):
    """max_query_len is only a bound: twice the real one sizes a grid whose later row tiles have no rows
    in any sequence (the persistent kernel's CTAs skip those items, every role alike)."""
    ctxs, news, hq, hkv, d, dtype = [700, 260, 1300], [400, 131, 64], 32, 8, 128, torch.bfloat16
    bt, kc, vc, q, qs, host = _build(ctxs, news, hq, hkv, d, dtype, seed=88)
    out = torch.full((q.shape[0], hq, d), float("nan"), dtype=dtype, device="cuda")
    pa.pa_prefill(out, q.cuda(), kc, vc, bt.cuda(), qs.cuda(), torch.tensor(ctxs, dtype=torch.int32).cuda(),
                  2 * max(news), d ** -0.5, hkv, kernel=kernel)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    want = _oracle(host, q, qs, ctxs, d ** -0.5, hkv, "bf16")
    assert float(np.max(np.abs(out.double().cpu().numpy() - want))) <= TOL["bf16"]


def test_tcgen05_and_warp_mma_prefill_agree():
    ctxs, news, hq, hkv, d = [1000, 77], [1000, 77], 32, 8, 128
    bt, kc, vc, q, qs, _ = _build(ctxs, news, hq, hkv, d, torch.bfloat16, seed=31)
    outs = []
    for kernel in (0, 1):
        out = torch.empty(q.shape[0], hq, d, dtype=torch.bfloat16, device="cuda")
        pa.pa_prefill(out, q.cuda(), kc, vc, bt.cuda(), qs.cuda(), torch.tensor(ctxs, dtype=torch.int32).cuda(),
                      max(news), d ** -0.5, hkv, kernel=kernel)
        outs.append(out)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    # Each kernel is within TOL of the exact result, so they differ by at most 2 * TOL (one bf16 ulp
    # at |out| >= 2 is already 2^-6 > TOL).
    for o in outs[1:]:
        assert (outs[0].double() - o.double()).abs().max().item() <= 2 * TOL["bf16"]


def test_tcgen05_prefill_is_deterministic():
    """Repeated launches give bit-identical outputs: a pipeline race (a buffer reused before the MMA
    reading it finished) shows up as run-to-run differences, even where it stays within tolerance."""
    ctxs, news, hq, hkv, d = [2000, 1500, 333], [2000, 700, 333], 32, 8, 128
    bt, kc, vc, q, qs, _ = _build(ctxs, news, hq, hkv, d, torch.bfloat16, seed=41)
    lens = torch.tensor(ctxs, dtype=torch.int32).cuda()
    outs = []
    for _ in range(6):
        out = torch.empty(q.shape[0], hq, d, dtype=torch.bfloat16, device="cuda")
        pa.pa_prefill(out, q.cuda(), kc, vc, bt.cuda(), qs.cuda(), lens, max(news), d ** -0.5, hkv, kernel=1)
        outs.append(out)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))


def test_chunked_equals_whole_and_last_row_equals_decode():
    ctxs, hq, hkv, d = [100], 8, 2, 128
    bt, kc, vc, q, _, _ = _build(ctxs, [100], hq, hkv, d, torch.bfloat16, seed=5)
    lens = torch.tensor(ctxs, dtype=torch.int32).cuda()
    whole = torch.empty(100, hq, d, dtype=torch.bfloat16, device="cuda")
    pa.pa_prefill(whole, q.cuda(), kc, vc, bt.cuda(), torch.tensor([0, 100], dtype=torch.int32).cuda(), lens, 100,
                  0.09, hkv)
    first = torch.empty(40, hq, d, dtype=torch.bfloat16, device="cuda")
    second = torch.empty(60, hq, d, dtype=torch.bfloat16, device="cuda")
    pa.pa_prefill(first, q[:40].cuda(), kc, vc, bt.cuda(), torch.tensor([0, 40], dtype=torch.int32).cuda(),
                  torch.tensor([40], dtype=torch.int32).cuda(), 40, 0.09, hkv)
    pa.pa_prefill(second, q[40:].cuda(), kc, vc, bt.cuda(), torch.tensor([0, 60], dtype=torch.int32).cuda(), lens, 60,
                  0.09, hkv)
    dec = torch.empty(1, hq, d, dtype=torch.bfloat16, device="cuda")
    pa.pa_decode(dec, q[99:].cuda(), kc, vc, bt.cuda(), lens, 0.09, hkv)
    torch.cuda.synchronize()
    # Each result is within TOL of the exact one, so two of them differ by at most 2 * TOL.
    assert (whole.double() - torch.cat([first, second]).double()).abs().max().item() <= 2 * TOL["bf16"]
    assert (whole[99:].double() - dec.double()).abs().max().item() <= 2 * TOL["bf16"]


def test_prefill_reports_impossible_chunks():
    ctxs = [20]
    bt, kc, vc, q, qs, _ = _build(ctxs, [20], 4, 4, 64, torch.float16, seed=9)
    out = torch.empty(20, 4, 64, dtype=torch.float16, device="cuda")
    # 20 new tokens but a context of only 10: impossible, reported, nothing faults.
    pa.pa_prefill(out, q.cuda(), kc, vc, bt.cuda(), qs.cuda(), torch.tensor([10], dtype=torch.int32).cuda(), 20, 0.1, 4)
    assert pa.pa_read_device_error(clear=True) & pa.PA_DEVERR_CTX_RANGE


@pytest.mark.parametrize("kernel", [0, 1])
def test_permuted_physical_blocks_give_bit_identical_prefill(kernel):
    """The same logical K/V, q and chunks placed in two different sets of physical blocks."""
    ctxs, news, hq, hkv, d = [700, 5, 260, 1300], [400, 5, 131, 64], 32, 8, 128
    outs = []
    for order_seed in (3, 4):
        bt, kc, vc, q, qs, _ = _build(ctxs, news, hq, hkv, d, torch.bfloat16, seed=12, order_seed=order_seed)
        out = torch.empty(q.shape[0], hq, d, dtype=torch.bfloat16, device="cuda")
        pa.pa_prefill(out, q.cuda(), kc, vc, bt.cuda(), qs.cuda(), torch.tensor(ctxs, dtype=torch.int32).cuda(),
                      max(news), d ** -0.5, hkv, kernel=kernel)
        outs.append((bt, out))
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    assert not torch.equal(outs[0][0], outs[1][0])  # the placements really differ
    assert torch.equal(outs[0][1].view(torch.int16), outs[1][1].view(torch.int16))
