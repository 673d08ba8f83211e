"""GPU parity of shared-prefix (cascade) decode against the float64 oracle.

pa_decode_cascade reads the prefix every sequence shares once per KV head (all B * G query rows as
one tensor-core contraction), the rest of each context with the decode kernel, and merges the two
softmax partials; the oracle is the plain definition over each sequence's whole context.
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


@pytest.mark.parametrize("fused", [True, False])
def test_cascade_matches_oracle(fused):
    w = W.ALL["prefix_gqa_small"]
    case = oracle_case.build(w)
    want = oracle_case.expected_out(case)
    dev = DeviceCase(w)
    if not fused:
        dev.write_new_token()
    for pt in (0, 16, 48):
        out = dev.cascade(fused=fused, partition_tokens=pt)
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
    b = dev.cascade(fused=False).clone()
    torch.cuda.synchronize()
    assert (a.double() - b.double()).abs().max().item() <= TOL[w.kv_dtype]


@pytest.mark.parametrize("lens", [(5, 64, 100, 16, 129, 40), (64, 64, 65, 200, 1, 33)])
def test_cascade_with_sequences_shorter_than_the_prefix(lens):
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
                             0.088, hkv, workspace=ws)
        torch.cuda.synchronize()
        assert pa.pa_read_device_error(clear=True) == 0
        kb = kc.view(torch.int16).numpy().view(np.uint8).reshape(nb, hkv, 16, D * 2)
        vb = vc.view(torch.int16).numpy().view(np.uint8).reshape(nb, hkv, 16, D * 2)
        want = attention.decode_paged(q.double().numpy(), kb, vb, bt.numpy(), lens, 0.088, hkv, "f16")
        assert max_err(out, want) <= TOL["f16"]


def test_cascade_reports_a_table_without_the_shared_prefix():
    w = W.ALL["prefix_gqa_small"]
    dev = DeviceCase(w)
    dev.write_new_token()
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt = dev.bt.clone()
    bt[2, 1] = int(bt[0, 1]) + 1 if int(bt[0, 1]) + 1 < w.num_blocks else 0
    old = dev.bt
    dev.bt = bt
    dev.cascade(fused=False, error_word=word)
    torch.cuda.synchronize()
    dev.bt = old
    assert int(word.item()) & pa.PA_DEVERR_PREFIX


def test_full_size_prefix_workload_sampled():
    from oracle import attention
    w = W.FULL["prefix_gqa"]
    dev = DeviceCase(w, sentinel=False)
    out = dev.cascade(fused=True).cpu()
    assert pa.pa_read_device_error(clear=True) == 0
    lens = dev.lens_host
    rng = np.random.default_rng(11)
    worst = 0.0
    for s in sorted(set(rng.integers(0, w.num_seqs, 6).tolist())):
        K = W.kv_source(w, s, "k", lens).double().numpy()
        V = W.kv_source(w, s, "v", lens).double().numpy()
        q = W.query(w)[s].double().numpy()
        for h in (0, 5, 31):
            want = attention.decode_logical_one(q[h], K, V, h, w.num_q_heads, w.num_kv_heads, w.scale)
            worst = max(worst, float(np.max(np.abs(out[s, h].double().numpy() - want))))
    assert worst <= TOL[w.kv_dtype], worst
