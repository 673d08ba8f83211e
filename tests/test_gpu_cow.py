"""GPU parity of copy-on-write: pa_copy_blocks bit-exact against the oracle, and a fork-then-append
decode where a child sequence shares its parent's blocks (parallel sampling / beam search, "vLLM
前世今生" §3.2) and each writes a different next token."""
import numpy as np
import pytest
import torch

import paged_kv_cache_385_b200 as pa
import workloads as W
from oracle import attention, cache, paging
from tests.device_case import TOL

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.float16, torch.float8_e4m3fn])
def test_copy_blocks_bit_exact(dtype):
    g = torch.Generator().manual_seed(3)
    nb, hkv, d = 64, 4, 128
    esz = 1 if dtype == torch.float8_e4m3fn else 2
    k0 = torch.randint(0, 256, (nb, hkv, 16, d * esz), generator=g, dtype=torch.uint8)
    v0 = torch.randint(0, 256, (nb, hkv, 16, d * esz), generator=g, dtype=torch.uint8)
    perm = torch.randperm(nb, generator=g)
    mapping = torch.stack([perm[:20], perm[20:40]], dim=1).to(torch.int64)  # distinct dsts, not sources
    mapping = torch.cat([mapping, torch.tensor([[perm[50], perm[50]]])])  # src == dst: no-op
    kc = k0.cuda().view(dtype).view(nb, hkv, 16, d)
    vc = v0.cuda().view(dtype).view(nb, hkv, 16, d)
    pa.pa_copy_blocks(kc, vc, mapping.cuda())
    torch.cuda.synchronize()
    ek, ev = cache.copy_blocks(k0.numpy(), v0.numpy(), mapping.numpy())
    assert np.array_equal(kc.view(torch.uint8).reshape(k0.shape).cpu().numpy(), ek)
    assert np.array_equal(vc.view(torch.uint8).reshape(v0.shape).cpu().numpy(), ev)
    assert pa.pa_read_device_error(clear=True) == 0
    bad = torch.tensor([[0, nb + 3]], dtype=torch.int64, device="cuda")
    pa.pa_copy_blocks(kc, vc, bad)
    assert pa.pa_read_device_error(clear=True) & pa.PA_DEVERR_BAD_BLOCK


def test_fork_then_append_with_copy_on_write():
    """B parents forked into B children; parent and child append different tokens at position ctx."""
    B, Hkv, G, D = 6, 2, 4, 128
    w = W.Workload("fork", B, Hkv * G, Hkv, D, "bf16", "bf16", 256, ("fixed", (33, 16, 47, 1, 64, 95)), seed=91)
    lens = W.context_lens(w)
    order = W.block_order(w)
    mb = 8
    alloc = pa.BlockAllocator(w.num_blocks, order.tolist())
    model = paging.FreeListModel(w.num_blocks, order.tolist())
    bt = pa.build_block_tables(alloc, lens.tolist(), mb)
    bt_model = paging.build_block_tables(lens.tolist(), order.tolist(), w.num_blocks, 16, 0, mb)
    for s in range(B):  # replay the same allocations on the model
        for b in bt_model[s][bt_model[s] >= 0]:
            assert model.alloc() == b
    assert np.array_equal(bt.numpy(), bt_model)
    # Fork: child s + B shares every block of parent s.
    child = bt.clone()
    for s in range(B):
        used = bt[s][bt[s] >= 0]
        alloc.incref_n(used)
        for b in used.tolist():
            assert model.incref(b)
    tables = torch.cat([bt, child]).clone()
    # Append position ctx to parent (first) and then child: copy-on-write if the block is shared.
    copies = []
    for s in range(2 * B):
        n = int(lens[s % B])
        j = n // 16
        if n % 16 == 0:  # a new block
            nbk = alloc.alloc()
            assert nbk == model.alloc()
        else:
            nbk, need_copy = alloc.cow(int(tables[s, j]))
            assert (nbk, need_copy) == model.cow(int(tables[s, j]))
            if need_copy:
                copies.append((int(tables[s, j]), nbk))
        tables[s, j] = nbk
    # Device: history in the pool, copies, then each sequence's own new token.
    dev = "cuda"
    kc = torch.zeros(w.num_blocks, Hkv, 16, D, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    ks = [W.kv_source(w, s, "k", lens) for s in range(B)]
    vs = [W.kv_source(w, s, "v", lens) for s in range(B)]
    seqs = [s for s in range(B) for _ in range(int(lens[s]))]
    poss = [p for s in range(B) for p in range(int(lens[s]))]
    pa.pa_reshape_and_cache(torch.cat(ks).to(dev), torch.cat(vs).to(dev),
                            pa.pa_slots_for_positions(bt, seqs, poss).to(dev), kc, vc)
    if copies:
        pa.pa_copy_blocks(kc, vc, torch.tensor(copies, dtype=torch.int64, device=dev))
    gen = torch.Generator().manual_seed(7)
    new_k = torch.randn(2 * B, Hkv, D, generator=gen).to(torch.bfloat16)
    new_v = torch.randn(2 * B, Hkv, D, generator=gen).to(torch.bfloat16)
    new_lens = torch.cat([lens, lens]) + 1
    slots = pa.pa_slots_for_positions(tables, list(range(2 * B)), [int(n) - 1 for n in new_lens])
    q = torch.randn(2 * B, Hkv * G, D, generator=gen).to(torch.bfloat16)
    out = torch.empty(2 * B, Hkv * G, D, dtype=torch.bfloat16, device=dev)
    pa.pa_decode_step(out, q.to(dev), new_k.to(dev), new_v.to(dev), slots.to(dev), kc, vc, tables.to(dev),
                      new_lens.to(dev), w.scale, Hkv)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error(clear=True) == 0
    for s in range(2 * B):
        K = torch.cat([ks[s % B], new_k[s:s + 1]]).double().numpy()
        V = torch.cat([vs[s % B], new_v[s:s + 1]]).double().numpy()
        for h in range(Hkv * G):
            want = attention.decode_logical_one(q[s, h].double().numpy(), K, V, h, Hkv * G, Hkv, w.scale)
            assert np.max(np.abs(out[s, h].double().cpu().numpy() - want)) <= TOL["bf16"]
    # Shared history blocks still hold the parent's rows; no sequence's write leaked into another's page.
    for s in range(B):
        n = int(lens[s])
        for t in range(n):
            blk = int(bt[s, t // 16])
            assert torch.equal(kc[blk, :, t % 16].cpu(), ks[s][t]) or t // 16 == n // 16
