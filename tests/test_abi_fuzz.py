"""Malformed descriptors through every C-ABI entry point: a status comes back, nothing crashes.

Each case starts from a valid set of pa_tensor descriptors for one entry point and changes one to
three fields (dtype, ndim, a shape or stride entry, the data pointer's alignment) to values such as
0, -1, 2^31 or 2^62, together with random options. The library must answer with one of its
statuses; an integer overflow or a division by zero in its size arithmetic would end the process.

The descriptors point at host memory, so this runs only where no CUDA device is present: there a
case that passes every check stops at the first CUDA call with PA_ERR_CUDA, while on a GPU it
would launch kernels on host pointers.
"""
import ctypes
import random

import numpy as np
import pytest
import torch

import paged_kv_cache_385_b200 as pa

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="host-pointer descriptors must never reach a GPU launch")

STATUSES = {pa.PA_OK, pa.PA_ERR_INVALID_ARG, pa.PA_ERR_UNSUPPORTED, pa.PA_ERR_WORKSPACE, pa.PA_ERR_CUDA}
EXTREMES = [0, 1, -1, 2, 3, 7, 15, 17, 65535, 65536, (1 << 31) - 1, 1 << 31, 1 << 40, 1 << 62, -(1 << 62)]
KINDS = ["decode", "step", "cascade", "prefill", "cache", "copy", "no_alloc"]


class _Case:
    def __init__(self, rng: random.Random, base: int):
        self.rng, self.base = rng, base

    def tensor(self, dtype, shape):
        t = pa.PaTensor()
        t.data, t.dtype, t.ndim = self.base, dtype, len(shape)
        acc = 1
        for i in reversed(range(len(shape))):
            t.shape[i], t.stride[i] = shape[i], acc
            acc *= shape[i]
        return t

    def valid(self, kind):
        r = self.rng
        B, Hkv, G, D = r.choice([1, 3, 32]), r.choice([1, 2, 8]), r.choice([1, 2, 4, 8, 16]), r.choice([64, 128])
        NB, mb, Hq = r.choice([16, 64, 1000]), r.choice([1, 4, 128]), Hkv * r.choice([1, 2, 4, 8, 16])
        dt = r.choice([pa.PA_F16, pa.PA_BF16])
        cd = dt if kind in ("prefill", "copy") else r.choice([dt, dt, pa.PA_E4M3])
        q, out = self.tensor(dt, [B, Hq, D]), self.tensor(dt, [B, Hq, D])
        kc, vc = self.tensor(cd, [NB, Hkv, 16, D]), self.tensor(cd, [NB, Hkv, 16, D])
        bt, lens = self.tensor(pa.PA_I32, [B, mb]), self.tensor(pa.PA_I32, [B])
        new = [self.tensor(dt, [B, Hkv, D]), self.tensor(dt, [B, Hkv, D]), self.tensor(pa.PA_I64, [B])]
        if kind in ("decode", "no_alloc"):
            return [out, q, kc, vc, bt, lens]
        if kind in ("step", "cascade"):
            return [out, q] + new + [kc, vc, bt, lens]
        if kind == "prefill":
            return [out, q, kc, vc, bt, self.tensor(pa.PA_I32, [B + 1]), lens]
        if kind == "cache":
            T = r.choice([1, 5, 64])
            return [self.tensor(dt, [T, Hkv, D]), self.tensor(dt, [T, Hkv, D]), self.tensor(pa.PA_I64, [T]), kc, vc]
        return [kc, vc, self.tensor(pa.PA_I64, [r.choice([0, 1, 9]), 2])]

    def mutate(self, ts):
        r = self.rng
        t, field = r.choice(ts), r.randrange(5)
        if field == 0:
            t.dtype = r.choice([0, 1, 2, 3, 4, 5, 6, -1])
        elif field == 1:
            t.shape[r.randrange(4)] = r.choice(EXTREMES)
        elif field == 2:
            t.stride[r.randrange(4)] = r.choice(EXTREMES + [8, 16, 128])
        elif field == 3:
            t.data = r.choice([0, self.base + 2, self.base + 8, self.base + 16, self.base + 64])
        else:
            t.ndim = r.randint(-1, 5)


def _call(lib, kind, case, ts, opts):
    r = case.rng
    refs = [ctypes.byref(t) for t in ts]
    hkv = ts[2].shape[1] if kind in ("decode", "prefill", "no_alloc") else ts[5].shape[1] if kind in (
        "step", "cascade") else 0
    if r.random() < 0.1:
        hkv = r.choice([0, -1, 3, 1 << 30])
    scale = 0.1 if r.random() < 0.9 else r.choice([float("nan"), float("inf")])
    o = ctypes.byref(opts)
    if kind == "decode":
        return lib.pa_decode(*refs, scale, hkv, o, None)
    if kind == "step":
        return lib.pa_decode_step(*refs, scale, hkv, o, None)
    if kind == "cascade":
        if r.random() < 0.2:
            refs[2] = refs[3] = refs[4] = None
        return lib.pa_decode_cascade(*refs, r.choice([16, 32, 64, 24, 1 << 20, 0]), scale, hkv, o, None)
    if kind == "prefill":
        return lib.pa_prefill(*refs, r.choice([1, 16, 1 << 30, 0]), scale, hkv, r.choice([-1, 0, 1]), None)
    if kind == "cache":
        return lib.pa_reshape_and_cache(*refs, opts.k_scale, opts.v_scale, None)
    if kind == "copy":
        return lib.pa_copy_blocks(*refs, None)
    if r.random() < 0.8:
        opts.workspace, opts.workspace_bytes = None, 0
    return lib.pa_decode_no_alloc(*refs, scale, hkv, o, None)


@pytest.mark.parametrize("seed", range(4))
def test_malformed_descriptors_return_a_status(seed):
    lib = pa.lib()
    buf = np.zeros(1 << 16, dtype=np.uint8)
    base = (buf.ctypes.data + 255) // 256 * 256
    case = _Case(random.Random(seed), base)
    seen = set()
    for _ in range(5000):
        kind = case.rng.choice(KINDS)
        ts = case.valid(kind)
        for _ in range(case.rng.choice([0, 1, 1, 1, 2, 3])):
            case.mutate(ts)
        opts = pa.PaDecodeOpts()
        lib.pa_decode_opts_init(ctypes.byref(opts))
        r = case.rng
        if r.random() < 0.4:
            opts.partition_tokens = r.choice([0, 16, 24, 512, 2048, 4096, -16])
            opts.max_context_len = r.choice([0, 1, 100, 1 << 20, -5, (1 << 31) - 1])
            opts.kernel, opts.prefix_kernel = r.choice([-1, 0, 1, 2]), r.choice([-1, 0, 1, 5])
            opts.k_scale, opts.v_scale = r.choice([1.0, 0.0, float("nan"), 0.01]), r.choice([1.0, 0.5, float("inf")])
        if r.random() < 0.3:
            opts.workspace, opts.workspace_bytes = r.choice([base, base + 8]), r.choice([0, 1024, 1 << 20, 1 << 62])
        status = _call(lib, kind, case, ts, opts)
        assert status in STATUSES, (kind, status)
        seen.add(status)
    # The cases reach past the argument checks (PA_ERR_CUDA: no device here) as well as fail them.
    assert {pa.PA_ERR_INVALID_ARG, pa.PA_ERR_CUDA} <= seen


def test_block_table_wider_than_any_context():
    """A table claiming 2^62 columns: once a division by zero (the token count of a row overflowed)."""
    buf = np.zeros(1 << 16, dtype=np.uint8)
    case = _Case(random.Random(0), (buf.ctypes.data + 255) // 256 * 256)
    q, out = case.tensor(pa.PA_BF16, [3, 4, 64]), case.tensor(pa.PA_BF16, [3, 4, 64])
    kc, vc = case.tensor(pa.PA_BF16, [1000, 1, 16, 64]), case.tensor(pa.PA_BF16, [1000, 1, 16, 64])
    bt, lens = case.tensor(pa.PA_I32, [3, 1 << 62]), case.tensor(pa.PA_I32, [3])
    bt.stride[0] = 4
    opts = pa.PaDecodeOpts()
    pa.lib().pa_decode_opts_init(ctypes.byref(opts))
    refs = [ctypes.byref(t) for t in (out, q, kc, vc, bt, lens)]
    assert pa.lib().pa_decode(*refs, 0.1, 1, ctypes.byref(opts), None) in STATUSES
    assert pa.pa_decode_workspace_bytes(65535, 1 << 20, 65535, 128, (1 << 31) - 1, 16) == 2 ** 64 - 1
