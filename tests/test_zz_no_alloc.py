"""pa_decode_no_alloc against pa_decode (GPU).

pa_decode_no_alloc is for callers that cannot allocate device memory: a plugin whose host framework
owns all device memory and passes it only inputs and outputs, a process whose device-memory budget
is fixed at start-up, or a serving loop that cannot afford a cudaMalloc in the middle of a step.
Its split-partition scratch is a fixed array inside the library instead of a caller workspace.
These tests call it through the C ABI and check its outputs against pa_decode's (with a caller
workspace) on calls made back to back (the array is shared and keeps the previous call's contents).
Same kernels, same partition size, same inputs: only the scratch's address differs, so the outputs
must be bit-identical. A stale partial read from an earlier call's contents would show up here as a
difference even where it stayed within the oracle tolerance. They also check that a batch needing
more scratch than the array holds is refused before any device work.
"""
import pytest
import torch

import paged_kv_cache_385_b200 as pa
import workloads as W
from tests.device_case import DeviceCase

pytestmark = pytest.mark.gpu


def _no_alloc(dev: DeviceCase, pt: int) -> torch.Tensor:
    w = dev.w
    out = torch.full_like(dev.q, float("nan"))
    pa.pa_decode_no_alloc(out, dev.q, dev.k_cache, dev.v_cache, dev.bt, dev.lens, w.scale, w.num_kv_heads,
                          k_scale=dev.k_scale, v_scale=dev.v_scale, max_context_len=dev.max_ctx, partition_tokens=pt)
    return out


def test_matches_pa_decode_on_consecutive_calls():
    cases = [(W.ALL["long70b_fp8_small"], 512), (W.ALL["llama3_8b_gqa_small"], 256), (W.ALL["mqa_small"], 128)]
    devs, refs = [], []
    for w, pt in cases:
        dev = DeviceCase(w)
        dev.write_new_token()
        # The batch really splits, so the scratch is used.
        assert pa.pa_decode_workspace_bytes(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, dev.max_ctx,
                                            pt) > 0
        refs.append(dev.decode(partition_tokens=pt).clone())  # existing entry point, caller workspace
        devs.append((dev, pt))
    torch.cuda.synchronize()
    # Two rounds over three different batches: each call follows a call that left other contents.
    for _ in range(2):
        for (dev, pt), ref in zip(devs, refs):
            out = _no_alloc(dev, pt)
            torch.cuda.synchronize()
            assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), (dev.w.name, pt)
    assert pa.pa_read_device_error(clear=True) == 0


def test_same_batch_twice_in_a_row():
    w = W.ALL["long70b_fp8_small"]
    dev = DeviceCase(w)
    dev.write_new_token()
    ref = dev.decode(partition_tokens=512).clone()
    first = _no_alloc(dev, 512)
    second = _no_alloc(dev, 512)
    torch.cuda.synchronize()
    for out in (first, second):
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_library_partitioning_matches_pa_decode():
    """partition_tokens 0: the library picks the split for both calls (the array counts as a workspace)."""
    w = W.ALL["long70b_fp8_small"]
    dev = DeviceCase(w)
    dev.write_new_token()
    need = pa.pa_decode_workspace_bytes(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, dev.max_ctx, 0)
    assert 0 < need <= pa.NO_ALLOC_SCRATCH_BYTES
    ref = dev.decode(partition_tokens=0).clone()
    for _ in range(2):
        out = _no_alloc(dev, 0)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert pa.pa_read_device_error(clear=True) == 0


def test_rejects_batches_larger_than_the_array():
    B, Hkv, G, D = 64, 8, 8, 128
    q = torch.zeros(B, Hkv * G, D, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    kc = torch.zeros(16, Hkv, 16, D, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(B, 8192, dtype=torch.int32, device="cuda")
    lens = torch.ones(B, dtype=torch.int32, device="cuda")
    need = pa.pa_decode_workspace_bytes(B, Hkv * G, Hkv, D, 8192 * 16, 256)
    assert need > pa.NO_ALLOC_SCRATCH_BYTES
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_decode_no_alloc(out, q, kc, kc, bt, lens, 0.1, Hkv, max_context_len=8192 * 16, partition_tokens=256)
    assert e.value.status == pa.PA_ERR_WORKSPACE
    assert "scratch" in str(e.value)


def test_refuses_a_caller_workspace():
    w = W.TINY
    dev = DeviceCase(w, history=False)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_decode_no_alloc(dev.out, dev.q, dev.k_cache, dev.v_cache, dev.bt, dev.lens, w.scale, w.num_kv_heads,
                              workspace=ws)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
