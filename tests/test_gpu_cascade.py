"""GPU parity of shared-prefix (cascade) decode against the float64 oracle.

pa_decode_cascade reads the prefix every sequence shares once per KV head (all B * G query rows as
one tensor-core contraction, by the tcgen05 kernel or the warp-level mma kernel), the rest of each
context with the decode kernel, and merges the two softmax partials; the oracle is the plain
definition over each sequence's whole context.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_385_b200 as pa
import workloads as W
from tests import oracle_case
from tests.device_case import TOL, DeviceCase

pytestmark = pytest.mark.gpu


def max_err(got, want):
    return float(np.max(np.abs(got.double().cpu().numpy() - want)))


PREFIX_KERNELS = [0, 1]  # warp-level mma, tcgen05


@pytest.mark.parametrize("prefix_kernel", PREFIX_KERNELS)
@pytest.mark.parametrize("fused", [True, False])
def test_cascade_matches_oracle(fused, prefix_kernel):
    w = W.ALL["prefix_gqa_small"]
    case = oracle_case.build(w)
    want = oracle_case.expected_out(case)
    dev = DeviceCase(w)
    if not fused:
        dev.write_new_token()
    for pt in (0, 16, 48):
        out = dev.cascade(fused=fused, partition_tokens=pt, prefix_kernel=prefix_kernel)
        torch.cuda.synchronize()
        assert max_err(out, want) <= TOL[w.kv_dtype], pt
    assert pa.pa_read_device_error(clear=True) == 0
    k, v = dev.pool_bytes()
    assert np.array_equal(k, case.k_pool) and np.array_equal(v, case.v_pool)


def test_cascade_equals_plain_decode_within_rounding():
    w = W.ALL["prefix_gqa_small"]
    dev = DeviceCase(w)
    dev.write_new_token()
    a = dev.decode(kernel=1).clone()
    b = dev.cascade(fused=False, prefix_kernel=0).clone()
    c = dev.cascade(fused=False, prefix_kernel=1).clone()
    torch.cuda.synchronize()
    # Each is within TOL of the exact result, so two of them differ by at most 2 * TOL.
    assert (a.double() - b.double()).abs().max().item() <= 2 * TOL[w.kv_dtype]
    assert (c.double() - b.double()).abs().max().item() <= 2 * TOL[w.kv_dtype]


def _shared_prefix_case(lens, hq, hkv, prefix, dtype, seed, nb_extra=0):
    """Block tables whose first prefix / 16 entries are blocks 0 .. prefix / 16 - 1 in every row."""
    B, D = len(lens), 128
    g = torch.Generator().manual_seed(seed)
    width = max(-(-max(lens) // 16), prefix // 16)
    own = sum(max(0, -(-n // 16) - prefix // 16) for n in lens)
    nb = prefix // 16 + own + nb_extra
    bt = torch.full((B, width), -1, dtype=torch.int32)
    order = (torch.randperm(own, generator=g) + prefix // 16).tolist()
    for s, n in enumerate(lens):
        for j in range(max(-(-n // 16), prefix // 16)):  # shorter sequences still list the prefix blocks
            bt[s, j] = j if j < prefix // 16 else order.pop()
    kc = torch.randn(nb, hkv, 16, D, generator=g).to(dtype)
    vc = torch.randn(nb, hkv, 16, D, generator=g).to(dtype)
    q = torch.randn(B, hq, D, generator=g).to(dtype)
    return q, kc, vc, bt


def _oracle_out(q, kc, vc, bt, lens, scale, hkv, kv):
    from oracle import attention
    nb, D = kc.shape[0], kc.shape[3]
    kb = kc.view(torch.int16).numpy().view(np.uint8).reshape(nb, hkv, 16, D * 2)
    vb = vc.view(torch.int16).numpy().view(np.uint8).reshape(nb, hkv, 16, D * 2)
    return attention.decode_paged(q.double().numpy(), kb, vb, bt.numpy(), lens, scale, hkv, kv)


@pytest.mark.parametrize("prefix_kernel", PREFIX_KERNELS)
@pytest.mark.parametrize("dtype,kv", [(torch.bfloat16, "bf16"), (torch.float16, "f16")])
def test_cascade_prefix_of_several_chunks(prefix_kernel, dtype, kv):
    """A 640-token prefix: two full 256-token chunks and a ragged one; 40 sequences x 4 group heads
    (two 128-row tiles, the second ragged); some contexts end inside the prefix, one exactly at it."""
    rng = np.random.default_rng(7)
    lens = [int(x) for x in 640 + rng.integers(1, 120, 40)]
    lens[3], lens[17], lens[30], lens[39] = 300, 640, 17, 641
    q, kc, vc, bt = _shared_prefix_case(lens, 8, 2, 640, dtype, seed=640)
    n = pa.pa_decode_cascade_workspace_bytes(len(lens), 8, 2, 128, max(lens), 640, 0)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    out = torch.empty(len(lens), 8, 128, dtype=dtype, device="cuda")
    pa.pa_decode_cascade(out, q.cuda(), None, None, None, kc.cuda(), vc.cuda(), bt.cuda(),
                         torch.tensor(lens, dtype=torch.int32).cuda(), 640, 0.0884, 2, workspace=ws,
                         max_context_len=max(lens), prefix_kernel=prefix_kernel)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    want = _oracle_out(q, kc, vc, bt, lens, 0.0884, 2, kv)
    assert max_err(out, want) <= TOL[kv]


@pytest.mark.parametrize("prefix_kernel", PREFIX_KERNELS)
@pytest.mark.parametrize("lens", [(5, 64, 100, 16, 129, 40), (64, 64, 65, 200, 1, 33)])
def test_cascade_with_sequences_shorter_than_the_prefix(lens, prefix_kernel):
    """Rows stop at their own context even inside the shared prefix; f16, G = 1 and G = 8 heads."""
    from oracle import attention
    for hq, hkv in ((4, 4), (16, 2)):
        B, D, P = len(lens), 128, 64
        g = torch.Generator().manual_seed(sum(lens) + hq)
        nb = 64
        # Prefix blocks 0..3 shared; each sequence's own blocks after that.
        bt = torch.full((B, 16), -1, dtype=torch.int32)
        nxt = 4
        for s, n in enumerate(lens):
            for j in range(-(-n // 16)):
                if j < P // 16:
                    bt[s, j] = j
                else:
                    bt[s, j] = nxt
                    nxt += 1
            for j in range(-(-n // 16), P // 16):  # shorter sequences still list the prefix blocks
                bt[s, j] = j
        kc = torch.randn(nb, hkv, 16, D, generator=g).to(torch.float16)
        vc = torch.randn(nb, hkv, 16, D, generator=g).to(torch.float16)
        q = torch.randn(B, hq, D, generator=g).to(torch.float16)
        lens_t = torch.tensor(lens, dtype=torch.int32)
        n = pa.pa_decode_cascade_workspace_bytes(B, hq, hkv, D, max(lens), P, 0)
        ws = torch.empty(n, dtype=torch.uint8, device="cuda")
        out = torch.empty(B, hq, D, dtype=torch.float16, device="cuda")
        pa.pa_decode_cascade(out, q.cuda(), None, None, None, kc.cuda(), vc.cuda(), bt.cuda(), lens_t.cuda(), P,
                             0.088, hkv, workspace=ws, prefix_kernel=prefix_kernel)
        torch.cuda.synchronize()
        assert pa.pa_read_device_error(clear=True) == 0
        kb = kc.view(torch.int16).numpy().view(np.uint8).reshape(nb, hkv, 16, D * 2)
        vb = vc.view(torch.int16).numpy().view(np.uint8).reshape(nb, hkv, 16, D * 2)
        want = attention.decode_paged(q.double().numpy(), kb, vb, bt.numpy(), lens, 0.088, hkv, "f16")
        assert max_err(out, want) <= TOL["f16"]


@pytest.mark.parametrize("prefix_kernel", PREFIX_KERNELS)
def test_cascade_reports_a_table_without_the_shared_prefix(prefix_kernel):
    w = W.ALL["prefix_gqa_small"]
    dev = DeviceCase(w)
    dev.write_new_token()
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt = dev.bt.clone()
    bt[2, 1] = int(bt[0, 1]) + 1 if int(bt[0, 1]) + 1 < w.num_blocks else 0
    old = dev.bt
    dev.bt = bt
    dev.cascade(fused=False, error_word=word, prefix_kernel=prefix_kernel)
    torch.cuda.synchronize()
    dev.bt = old
    assert int(word.item()) & pa.PA_DEVERR_PREFIX


@pytest.mark.parametrize("prefix_kernel", PREFIX_KERNELS)
@pytest.mark.parametrize("fused", [True, False])
def test_permuted_physical_blocks_give_bit_identical_cascade(fused, prefix_kernel):
    """Two free-list orders place the shared prefix and every suffix in different physical blocks;
    the cascade output (prefix kernel, suffix decode and merge) must not change by a bit."""
    w = W.ALL["prefix_gqa_small"]
    outs, tables = [], []
    for seed in (21, 22):
        order = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(seed)).to(torch.int32)
        dev = DeviceCase(w, order=order)
        if not fused:
            dev.write_new_token()
        for pt in (0, 16):
            outs.append((pt, dev.cascade(fused=fused, partition_tokens=pt, prefix_kernel=prefix_kernel).clone()))
        tables.append(dev.bt_host)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    assert not torch.equal(tables[0], tables[1])
    for pt in (0, 16):
        a, b = [o for p, o in outs if p == pt]
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), pt


@pytest.mark.parametrize("prefix_kernel", PREFIX_KERNELS)
def test_permuted_prefix_of_several_chunks_is_bit_identical(prefix_kernel):
    """The 640-token, two-row-tile case with its blocks renumbered by a random permutation."""
    rng = np.random.default_rng(8)
    lens = [int(x) for x in 640 + rng.integers(1, 120, 40)]
    lens[3], lens[30] = 300, 17
    q, kc, vc, bt = _shared_prefix_case(lens, 8, 2, 640, torch.bfloat16, seed=641)
    perm = torch.randperm(kc.shape[0], generator=torch.Generator().manual_seed(9))
    # Block b moves to perm[b]: the same logical data in other physical blocks.
    kc2, vc2 = torch.empty_like(kc), torch.empty_like(vc)
    kc2[perm], vc2[perm] = kc, vc
    bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0).long()].to(torch.int32), bt)
    n = pa.pa_decode_cascade_workspace_bytes(len(lens), 8, 2, 128, max(lens), 640, 0)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    outs = []
    for k_, v_, t_ in ((kc, vc, bt), (kc2, vc2, bt2)):
        out = torch.empty(len(lens), 8, 128, dtype=torch.bfloat16, device="cuda")
        pa.pa_decode_cascade(out, q.cuda(), None, None, None, k_.cuda(), v_.cuda(), t_.cuda(),
                             torch.tensor(lens, dtype=torch.int32).cuda(), 640, 0.0884, 2, workspace=ws,
                             max_context_len=max(lens), prefix_kernel=prefix_kernel)
        outs.append(out)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
