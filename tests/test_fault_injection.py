"""Host-side fault injection (pa_debug_fail_next_launches): calls fail as a failed launch does,
with no device work, and argument errors still come first.

The descriptors point at host memory, so this runs only where no CUDA device is present (there the
calls that are not injected stop at the first CUDA call; on a GPU they would launch kernels on host
pointers). The hook itself never reaches a device.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_385_b200 as pa
from tests.host_buffers import aligned_zeros

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="host-pointer descriptors must never reach a GPU launch")


@pytest.fixture
def decode_args():
    B, Hq, Hkv, D, NB = 2, 8, 2, 128, 16
    q = aligned_zeros((B, Hq, D), torch.bfloat16)
    kc = aligned_zeros((NB, Hkv, 16, D), torch.bfloat16)
    bt = torch.zeros(B, 4, dtype=torch.int32)
    lens = torch.full((B,), 40, dtype=torch.int32)
    ts = [pa.as_pa_tensor(t, n, device=False) for t, n in ((q, "out"), (q, "q"), (kc, "k"), (kc, "v"), (bt, "bt"),
                                                            (lens, "lens"))]
    keep = (q, kc, bt, lens)

    def call(hkv=Hkv):
        return pa.lib().pa_decode(*[ctypes.byref(t) for t in ts], 0.088, hkv, None, None)
    call.keep = keep
    return call


def test_injected_failures_are_counted_and_host_only(decode_args):
    try:
        pa.pa_debug_fail_next_launches(2)
        assert decode_args() == pa.PA_ERR_CUDA and "injected" in pa.pa_last_error()
        # An argument error is reported as such and does not use up an injected failure.
        assert decode_args(hkv=3) == pa.PA_ERR_INVALID_ARG
        assert decode_args() == pa.PA_ERR_CUDA and "injected" in pa.pa_last_error()
        # Both used: the next call goes on to the device (none here: a real CUDA error).
        assert decode_args() == pa.PA_ERR_CUDA and "injected" not in pa.pa_last_error()
    finally:
        pa.pa_debug_fail_next_launches(0)


def test_every_enqueuing_entry_point_takes_the_hook():
    T, Hkv, D, NB = 3, 2, 64, 8
    key = aligned_zeros((T, Hkv, D), torch.float16)
    kc = aligned_zeros((NB, Hkv, 16, D), torch.float16)
    slots = torch.zeros(T, dtype=torch.int64)
    mapping = torch.tensor([[0, 1]], dtype=torch.int64)
    q = aligned_zeros((T, Hkv, D), torch.float16)
    bt = torch.zeros(1, 1, dtype=torch.int32)
    qs = torch.tensor([0, T], dtype=torch.int32)
    lens = torch.tensor([T], dtype=torch.int32)
    P = lambda t, n: ctypes.byref(pa.as_pa_tensor(t, n, device=False))  # noqa: E731
    lib = pa.lib()
    calls = {
        "pa_reshape_and_cache": lambda: lib.pa_reshape_and_cache(P(key, "k"), P(key, "v"), P(slots, "s"), P(kc, "kc"),
                                                                 P(kc, "vc"), 1.0, 1.0, None),
        "pa_copy_blocks": lambda: lib.pa_copy_blocks(P(kc, "kc"), P(kc, "vc"), P(mapping, "m"), None),
        "pa_prefill": lambda: lib.pa_prefill(P(q, "o"), P(q, "q"), P(kc, "kc"), P(kc, "vc"), P(bt, "bt"), P(qs, "qs"),
                                             P(lens, "l"), T, 0.125, Hkv, -1, None),
    }
    try:
        for name, call in calls.items():
            pa.pa_debug_fail_next_launches(1)
            assert call() == pa.PA_ERR_CUDA, name
            assert "injected" in pa.pa_last_error(), name
    finally:
        pa.pa_debug_fail_next_launches(0)


def test_negative_count_is_refused():
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_debug_fail_next_launches(-1)
    assert e.value.status == pa.PA_ERR_INVALID_ARG


@pytest.mark.parametrize("cascade", [False, True])
def test_queried_workspace_size_is_exactly_what_the_call_checks(cascade):
    """A workspace of the size the query function reports passes the entry point's checks (the
    armed failure is reached); one byte less is refused with PA_ERR_WORKSPACE when a split happens."""
    rng = np.random.default_rng(5 + cascade)
    lib = pa.lib()
    checked = 0
    for _ in range(150):
        Hkv = int(rng.choice([1, 2, 8]))
        G = int(rng.choice([1, 4, 8]))
        B, D = int(rng.integers(1, 40)), int(rng.choice([64, 128]))
        mb = int(rng.integers(1, 300))
        max_ctx = int(rng.integers(1, mb * 16 + 1))
        pt = int(rng.choice([0, 0, 16, 256, 512, 2048]))
        prefix = 16 * int(rng.integers(1, mb + 1)) if cascade else 0
        if cascade and D != 128:
            D = 128
        q = aligned_zeros((B, Hkv * G, D), torch.bfloat16)
        kc = aligned_zeros((4, Hkv, 16, D), torch.bfloat16)
        bt = torch.zeros(B, mb, dtype=torch.int32)
        lens = torch.ones(B, dtype=torch.int32)
        if cascade:
            need = pa.pa_decode_cascade_workspace_bytes(B, Hkv * G, Hkv, D, max_ctx, prefix, pt)
        else:
            need = pa.pa_decode_workspace_bytes(B, Hkv * G, Hkv, D, max_ctx, pt)
        ws = aligned_zeros((max(need, 1),), torch.uint8)
        ts = [pa.as_pa_tensor(t, n, device=False) for t, n in ((q, "out"), (q, "q"), (kc, "k"), (kc, "v"),
                                                                (bt, "bt"), (lens, "lens"))]

        def call(nbytes):
            opts = pa.PaDecodeOpts()
            lib.pa_decode_opts_init(ctypes.byref(opts))
            opts.max_context_len, opts.partition_tokens = max_ctx, pt
            if nbytes > 0:
                opts.workspace, opts.workspace_bytes = ws.data_ptr(), nbytes
            r = [ctypes.byref(t) for t in ts]
            pa.pa_debug_fail_next_launches(1)
            try:
                if cascade:
                    status = lib.pa_decode_cascade(r[0], r[1], None, None, None, r[2], r[3], r[4], r[5], prefix,
                                                   0.1, Hkv, ctypes.byref(opts), None)
                else:
                    status = lib.pa_decode(*r, 0.1, Hkv, ctypes.byref(opts), None)
                return status, pa.pa_last_error()  # read before the disarming call resets it
            finally:
                pa.pa_debug_fail_next_launches(0)

        st_, msg = call(need)
        assert st_ == pa.PA_ERR_CUDA and "injected" in msg, (msg, need)
        if need > 0:
            assert call(need - 1)[0] == pa.PA_ERR_WORKSPACE
            checked += 1
    assert checked > 20


def test_no_alloc_accepts_exactly_the_batches_its_array_holds():
    rng = np.random.default_rng(11)
    lib = pa.lib()
    seen = set()
    for _ in range(200):
        Hkv, G = int(rng.choice([1, 8])), int(rng.choice([1, 8]))
        B, D, mb = int(rng.integers(1, 64)), 128, int(rng.integers(1, 8192))
        max_ctx, pt = int(rng.integers(1, mb * 16 + 1)), int(rng.choice([0, 256, 512]))
        q = aligned_zeros((B, Hkv * G, D), torch.bfloat16)
        kc = aligned_zeros((4, Hkv, 16, D), torch.bfloat16)
        bt, lens = torch.zeros(B, mb, dtype=torch.int32), torch.ones(B, dtype=torch.int32)
        ts = [pa.as_pa_tensor(t, n, device=False) for t, n in ((q, "out"), (q, "q"), (kc, "k"), (kc, "v"),
                                                                (bt, "bt"), (lens, "lens"))]
        opts = pa.PaDecodeOpts()
        lib.pa_decode_opts_init(ctypes.byref(opts))
        opts.max_context_len, opts.partition_tokens = max_ctx, pt
        need = pa.pa_decode_workspace_bytes(B, Hkv * G, Hkv, D, max_ctx, pt)
        pa.pa_debug_fail_next_launches(1)
        try:
            st_ = lib.pa_decode_no_alloc(*[ctypes.byref(t) for t in ts], 0.1, Hkv, ctypes.byref(opts), None)
            msg = pa.pa_last_error()
        finally:
            pa.pa_debug_fail_next_launches(0)
        if need <= pa.NO_ALLOC_SCRATCH_BYTES:
            assert st_ == pa.PA_ERR_CUDA and "injected" in msg, (need, msg)
        else:
            assert st_ == pa.PA_ERR_WORKSPACE and "scratch" in msg, (need, msg)
        seen.add(need <= pa.NO_ALLOC_SCRATCH_BYTES)
    assert seen == {True, False}
