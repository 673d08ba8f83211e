"""GPU parity of split-context decode in both forms against the float64 oracle.

Contexts split into partitions of at most 512 tokens run one persistent warp per partition (opts.kernel
1, the default); opts.kernel 2 keeps one CTA per partition. Both are checked here on batches built
for the split's edge cases: empty contexts, contexts of one token and of exact partition multiples,
many more partitions than resident warps, and more sequences than the persistent form takes (which
then falls back to one CTA per partition). The oracle's expected values come from the host draws
(its own block tables, its own e4m3 codec); nothing the GPU wrote feeds it.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_385_b200 as pa
from oracle import attention, e4m3, paging
from tests.device_case import TOL

pytestmark = pytest.mark.gpu

_DT = {"f16": torch.float16, "bf16": torch.bfloat16}


def _case(lens, hq, hkv, d, kv, seed):
    """Device state through the library, and the oracle's expected decode output.

    History positions 0 .. n - 2 of every sequence are written with pa_reshape_and_cache; the new
    token (position n - 1, none for an empty context) is returned for the caller to write.
    """
    g = torch.Generator().manual_seed(seed)
    B = len(lens)
    mb = max(1, max(-(-n // 16) for n in lens))
    nb = sum(-(-n // 16) for n in lens) + 7
    order = torch.randperm(nb, generator=g)
    alloc = pa.BlockAllocator(nb, order.tolist())
    bt = pa.build_block_tables(alloc, lens, mb)
    assert np.array_equal(bt.numpy(), paging.build_block_tables(lens, order.numpy(), nb, 16, 0, mb))
    src = torch.bfloat16 if kv == "e4m3" else _DT[kv]
    K = [torch.randn(n, hkv, d, generator=g).to(src) for n in lens]
    V = [torch.randn(n, hkv, d, generator=g).to(src) for n in lens]
    q = torch.randn(B, hq, d, generator=g).to(torch.bfloat16 if kv == "e4m3" else _DT[kv])
    ks = vs = 1.0
    if kv == "e4m3":
        c448 = torch.tensor(448.0)
        ks = float(torch.cat([k.float().abs().flatten() for k in K]).max() / c448)
        vs = float(torch.cat([v.float().abs().flatten() for v in V]).max() / c448)
        Ke = [e4m3.dequantize(e4m3.quantize(k.float().numpy(), ks), ks) for k in K]
        Ve = [e4m3.dequantize(e4m3.quantize(v.float().numpy(), vs), vs) for v in V]
    else:
        Ke = [k.double().numpy() for k in K]
        Ve = [v.double().numpy() for v in V]
    want = attention.decode_logical(q.double().numpy(), Ke, Ve, d ** -0.5, hkv)
    cdt = torch.float8_e4m3fn if kv == "e4m3" else _DT[kv]
    shape = (nb, hkv, 16, d)
    esz = 1 if kv == "e4m3" else 2
    kc = torch.randint(0, 256, (nb, hkv, 16, d * esz), generator=g, dtype=torch.uint8).view(cdt).view(shape).cuda()
    vc = torch.randint(0, 256, (nb, hkv, 16, d * esz), generator=g, dtype=torch.uint8).view(cdt).view(shape).cuda()
    seqs = [s for s in range(B) for _ in range(max(0, lens[s] - 1))]
    poss = [p for s in range(B) for p in range(max(0, lens[s] - 1))]
    if seqs:
        pa.pa_reshape_and_cache(torch.cat([k[:-1] for k in K if len(k)]).cuda(),
                                torch.cat([v[:-1] for v in V if len(v)]).cuda(),
                                pa.pa_slots_for_positions(bt, seqs, poss).cuda(), kc, vc, ks, vs)
    new_k = torch.stack([k[-1] if len(k) else torch.zeros(hkv, d, dtype=src) for k in K]).cuda()
    new_v = torch.stack([v[-1] if len(v) else torch.zeros(hkv, d, dtype=src) for v in V]).cuda()
    slots = torch.tensor([int(paging.slot_of(bt[s].numpy(), n - 1)) if n else -1 for s, n in enumerate(lens)],
                         dtype=torch.int64).cuda()
    dev = dict(q=q.cuda(), kc=kc, vc=vc, bt=bt.cuda(), lens=torch.tensor(lens, dtype=torch.int32).cuda(),
               new_k=new_k, new_v=new_v, slots=slots, ks=ks, vs=vs, hkv=hkv, d=d, max_ctx=max(max(lens), 1))
    return dev, want


def _decode(dev, kernel, pt, fused):
    B, hq = dev["q"].shape[0], dev["q"].shape[1]
    ws = pa.decode_workspace(B, hq, dev["hkv"], dev["d"], dev["max_ctx"], pt)
    out = torch.full_like(dev["q"], float("nan"))
    kw = dict(k_scale=dev["ks"], v_scale=dev["vs"], max_context_len=dev["max_ctx"], partition_tokens=pt,
              workspace=ws, kernel=kernel)
    if fused:
        pa.pa_decode_step(out, dev["q"], dev["new_k"], dev["new_v"], dev["slots"], dev["kc"], dev["vc"], dev["bt"],
                          dev["lens"], dev["d"] ** -0.5, dev["hkv"], **kw)
    else:
        pa.pa_reshape_and_cache(dev["new_k"], dev["new_v"], dev["slots"], dev["kc"], dev["vc"], dev["ks"], dev["vs"])
        pa.pa_decode(out, dev["q"], dev["kc"], dev["vc"], dev["bt"], dev["lens"], dev["d"] ** -0.5, dev["hkv"], **kw)
    return out


EDGE_LENS = [0, 1, 16, 17, 511, 512, 513, 1300, 0, 2047, 48, 47]


@pytest.mark.parametrize("kv,hq,hkv,d", [("f16", 8, 2, 128), ("bf16", 4, 4, 64), ("e4m3", 16, 2, 128),
                                         ("bf16", 32, 2, 128)])
@pytest.mark.parametrize("fused", [False, True])
def test_split_forms_match_oracle_on_edge_lengths(kv, hq, hkv, d, fused):
    dev, want = _case(EDGE_LENS, hq, hkv, d, kv, seed=hq * 7 + d + hkv)
    tol = TOL[kv]
    first = True
    for kernel in (1, 2):
        for pt in (16, 48, 256, 512):
            out = _decode(dev, kernel, pt, fused and first)
            first = False  # the new tokens are written once; later calls read them
            torch.cuda.synchronize()
            got = out.double().cpu().numpy()
            assert np.isfinite(got).all(), (kernel, pt)
            err = float(np.max(np.abs(got - want)))
            assert err <= tol, f"kernel {kernel} partition {pt}: max abs err {err}"
            for s, n in enumerate(EDGE_LENS):
                if n == 0:
                    assert not got[s].any(), (kernel, pt, s)
    assert pa.pa_read_device_error(clear=True) == 0


def test_split_with_many_more_partitions_than_warps():
    """16-token partitions of 1.5K-4K-token contexts: ~19K units for ~2.4K resident warps, so every
    warp runs its ring on through several partitions of different sequences and heads."""
    rng = np.random.default_rng(5)
    lens = [int(x) for x in rng.integers(1500, 4000, 12)]
    dev, want = _case(lens, 64, 8, 128, "e4m3", seed=9)
    out = _decode(dev, 1, 16, fused=True)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    assert float(np.max(np.abs(out.double().cpu().numpy() - want))) <= TOL["e4m3"]
    again = _decode(dev, 1, 16, fused=False)  # the same step again: bit-identical
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), again.view(torch.int16))


def test_split_beyond_the_persistent_form_sequence_limit():
    """More sequences than the persistent form's per-CTA tables hold: the split runs one CTA per
    partition, with the same results."""
    rng = np.random.default_rng(6)
    lens = [int(x) for x in rng.integers(0, 300, 600)]
    dev, want = _case(lens, 4, 2, 64, "f16", seed=10)
    for kernel in (1, 2):
        out = _decode(dev, kernel, 16, fused=kernel == 1)
        torch.cuda.synchronize()
        assert float(np.max(np.abs(out.double().cpu().numpy() - want))) <= TOL["f16"], kernel
    assert pa.pa_read_device_error(clear=True) == 0
