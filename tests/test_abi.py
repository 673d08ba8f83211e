"""CPU checks of the C-ABI library: it loads, exports every declared entry point, and its host-side
allocator and slot helper agree with the oracle's models. No GPU and no device compute here."""
import copy
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import paged_kv_cache_385_b200 as pa
import workloads as W
from oracle import paging
from tests.host_buffers import aligned_zeros

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if not hdr.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", hdr)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("pa_reshape_and_cache", "pa_decode", "pa_decode_workspace_bytes", "pa_allocator_create",
                     "pa_block_alloc", "pa_block_incref", "pa_block_free", "pa_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(pa.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (pa_[a-z0-9_]+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported


def test_status_strings_and_version():
    assert pa.pa_status_string(pa.PA_OK) == "ok"
    assert pa.pa_status_string(pa.PA_ERR_WORKSPACE).startswith("workspace")
    assert re.match(r"^\d+\.\d+\.\d+$", pa.pa_version())


def test_workspace_sizing():
    assert pa.pa_decode_workspace_bytes(4, 4, 4, 64, 100, 0) == 0  # fits one partition
    assert pa.pa_decode_partition_tokens(32, 32, 2048) == 0  # 1024 units fill the GPU unsplit
    assert pa.pa_decode_partition_tokens(8, 8, 131072) == 2048
    assert pa.pa_decode_partition_tokens(64, 8, 8192) == 2048
    assert pa.pa_decode_partition_tokens(1, 8, 32768) == 256
    assert pa.pa_decode_partition_tokens(4, 8, 4096) == 256
    n = pa.pa_decode_workspace_bytes(8, 64, 8, 128, 131072, 512)
    P = 131072 // 512
    assert n >= 8 * 64 * P * (128 + 2) * 4


def test_null_tensor_is_rejected_without_a_gpu():
    lib = pa.lib()
    st_ = lib.pa_decode(None, None, None, None, None, None, 1.0, 1, None, None)
    assert st_ == pa.PA_ERR_INVALID_ARG
    assert "NULL" in pa.pa_last_error()


@settings(max_examples=150, deadline=None)
@given(n=st.integers(1, 40), ops=st.lists(st.tuples(st.sampled_from("aifc"), st.integers(-2, 42)), max_size=150),
       seed=st.integers(0, 2**31 - 1))
def test_allocator_matches_oracle_model(n, ops, seed):
    order = np.random.default_rng(seed).permutation(n).tolist()
    model = paging.FreeListModel(n, order)
    a = pa.BlockAllocator(n, order)
    lib = pa.lib()
    for op, b in ops:
        if op == "a":
            want = model.alloc()
            got = lib.pa_block_alloc(a._h)
            assert got == (pa.PA_ERR_EXHAUSTED if want is None else want)
        elif op == "i":
            assert (lib.pa_block_incref(a._h, b) == pa.PA_OK) == model.incref(b)
        elif op == "c":
            want = model.cow(b)
            out = ctypes.c_int32(-7)
            r = lib.pa_block_cow(a._h, b, ctypes.byref(out))
            if want is None:
                assert r in (pa.PA_ERR_BAD_BLOCK, pa.PA_ERR_EXHAUSTED)
            else:
                assert (out.value, r == 1) == want
        else:
            assert (lib.pa_block_free(a._h, b) == pa.PA_OK) == model.free(b)
        assert a.num_free == model.num_free
    for blk in range(n):
        assert a.refcount(blk) == model.refcount(blk)
    assert lib.pa_block_refcount(a._h, n) == pa.PA_ERR_BAD_BLOCK


def test_allocator_rejects_bad_orders():
    with pytest.raises(ValueError):
        pa.BlockAllocator(4, [0, 1, 1, 2])
    with pytest.raises(ValueError):
        pa.BlockAllocator(4, [0, 1, 2, 4])
    with pytest.raises(ValueError):
        pa.BlockAllocator(0)


def test_alloc_n_is_all_or_nothing():
    a = pa.BlockAllocator(5)
    a.alloc_n(3)
    with pytest.raises(pa.PagedAttentionError) as e:
        a.alloc_n(3)
    assert e.value.status == pa.PA_ERR_EXHAUSTED
    assert a.num_free == 2


@pytest.mark.parametrize("name", ["tiny", "llama3_8b_gqa_small", "prefix_gqa_small", "long70b_fp8_small",
                                  "llama3_8b_gqa", "prefix_gqa", "long70b_fp8"])
def test_block_tables_and_slots_match_oracle(name):
    w = W.ALL[name]
    lens = W.context_lens(w)
    order = W.block_order(w)
    mb = W.max_blocks_per_seq(w, lens)
    bt = pa.build_block_tables(pa.BlockAllocator(w.num_blocks, order.tolist()), lens.tolist(), mb,
                               w.shared_prefix_tokens)
    bt_o = paging.build_block_tables(lens.numpy(), order.numpy(), w.num_blocks, 16, w.shared_prefix_tokens, mb)
    assert np.array_equal(bt.numpy(), bt_o)
    rng = np.random.default_rng(3)
    seqs = rng.integers(0, w.num_seqs, 200)
    poss = [int(rng.integers(0, int(lens[s]))) for s in seqs]
    got = pa.pa_slots_for_positions(bt, seqs.tolist(), poss).numpy()
    want = paging.slots_for_positions(bt_o, seqs.tolist(), poss)
    assert np.array_equal(got, want)


def test_slot_helper_rejects_out_of_range():
    bt = torch.tensor([[3, -1]], dtype=torch.int32)
    with pytest.raises(pa.PagedAttentionError):
        pa.pa_slots_for_positions(bt, [0], [16])  # entry -1
    with pytest.raises(pa.PagedAttentionError):
        pa.pa_slots_for_positions(bt, [0], [40])  # beyond the table
    assert pa.pa_slots_for_positions(bt, [0], [5]).tolist() == [53]


def test_cascade_option_validation_happens_on_the_host():
    """A bad opts.prefix_kernel or an unaligned prefix length is refused before any device work (the
    tensors here are host memory, which no kernel could read)."""
    B, Hq, Hkv, D, NB = 2, 8, 2, 128, 16
    q = aligned_zeros((B, Hq, D), torch.bfloat16)
    kc = aligned_zeros((NB, Hkv, 16, D), torch.bfloat16)
    bt = torch.zeros(B, 4, dtype=torch.int32)
    lens = torch.full((B,), 40, dtype=torch.int32)
    ts = [pa.as_pa_tensor(t, n, device=False) for t, n in ((q, "out"), (q, "q"), (kc, "k"), (kc, "v"), (bt, "bt"),
                                                            (lens, "lens"))]
    lib = pa.lib()

    def call(prefix_tokens, **kw):
        opts = pa.PaDecodeOpts()
        lib.pa_decode_opts_init(ctypes.byref(opts))
        for k, v in kw.items():
            setattr(opts, k, v)
        out, qq, k, v, b, n = [ctypes.byref(t) for t in ts]
        return lib.pa_decode_cascade(out, qq, None, None, None, k, v, b, n, prefix_tokens, 0.088, Hkv,
                                     ctypes.byref(opts), None)

    assert call(32, prefix_kernel=7) == pa.PA_ERR_INVALID_ARG
    assert "prefix_kernel" in pa.pa_last_error()
    assert call(24) == pa.PA_ERR_INVALID_ARG  # not a multiple of 16
    assert "multiple of 16" in pa.pa_last_error()


def test_prefill_kernel_choice_is_checked_on_the_host():
    """The tcgen05 prefill takes head_dim 128 and a group dividing 128: asking for it with D = 64 is
    refused before any device work; an unknown kernel number too."""
    T, Hq, Hkv, D, NB, B = 8, 4, 4, 64, 4, 1
    q = aligned_zeros((T, Hq, D), torch.float16)
    kc = aligned_zeros((NB, Hkv, 16, D), torch.float16)
    bt = torch.zeros(B, 1, dtype=torch.int32)
    qs = torch.tensor([0, T], dtype=torch.int32)
    lens = torch.tensor([T], dtype=torch.int32)
    ts = [pa.as_pa_tensor(t, n, device=False) for t, n in ((q, "out"), (q, "q"), (kc, "k"), (kc, "v"), (bt, "bt"),
                                                            (qs, "qs"), (lens, "lens"))]
    lib = pa.lib()
    args = [ctypes.byref(t) for t in ts]
    assert lib.pa_prefill(*args, T, 0.125, Hkv, 1, None) == pa.PA_ERR_UNSUPPORTED
    assert "tcgen05" in pa.pa_last_error()
    for kernel in (2, -2):
        assert lib.pa_prefill(*args, T, 0.125, Hkv, kernel, None) == pa.PA_ERR_INVALID_ARG


def test_bounded_wait_selftest_checks_its_timeout_on_the_host():
    assert pa.lib().pa_selftest_bounded_wait(0, None, None) == pa.PA_ERR_INVALID_ARG
    assert pa.lib().pa_selftest_bounded_wait(2000000, None, None) == pa.PA_ERR_INVALID_ARG


def test_decode_argument_errors_are_reported_before_device_work():
    """Every argument error of pa_decode is found on the host, the workspace check included: the
    tensors here are host memory, so a call that reached the device would not return these codes."""
    B, Hq, Hkv, D, NB = 2, 8, 2, 128, 16
    q = aligned_zeros((B, Hq, D), torch.bfloat16)
    kc = aligned_zeros((NB, Hkv, 16, D), torch.bfloat16)
    kc16 = aligned_zeros((NB, Hkv, 16, D), torch.float16)
    bt = torch.zeros(B, 64, dtype=torch.int32)
    lens = torch.full((B,), 1000, dtype=torch.int32)
    lib = pa.lib()

    def call(kcache=kc, tables=bt, hkv=Hkv, **kw):
        ts = [pa.as_pa_tensor(t, n, device=False) for t, n in ((q, "out"), (q, "q"), (kcache, "k"), (kcache, "v"),
                                                                (tables, "bt"), (lens, "lens"))]
        opts = pa.PaDecodeOpts()
        lib.pa_decode_opts_init(ctypes.byref(opts))
        for k, v in kw.items():
            setattr(opts, k, v)
        return lib.pa_decode(*[ctypes.byref(t) for t in ts], 0.088, hkv, ctypes.byref(opts), None)

    assert call(kcache=kc16) == pa.PA_ERR_INVALID_ARG  # f16 cache with a bf16 query
    assert call(hkv=4) == pa.PA_ERR_INVALID_ARG  # does not match the cache's head count
    assert call(tables=bt.to(torch.int64)) == pa.PA_ERR_INVALID_ARG
    assert call(partition_tokens=24) == pa.PA_ERR_INVALID_ARG
    assert call(kernel=3) == pa.PA_ERR_INVALID_ARG
    # A split into 1024 / 256 = 4 partitions needs a workspace; none given.
    assert call(partition_tokens=256) == pa.PA_ERR_WORKSPACE
    assert "workspace" in pa.pa_last_error()
    small = aligned_zeros((64,), torch.uint8)
    assert call(partition_tokens=256, workspace=small.data_ptr(), workspace_bytes=64) == pa.PA_ERR_WORKSPACE
    kc3 = aligned_zeros((NB, 3, 16, D), torch.bfloat16)
    assert call(kcache=kc3, hkv=3) == pa.PA_ERR_INVALID_ARG  # 8 query heads over 3 KV heads
    assert "multiple" in pa.pa_last_error()
    # Misaligned pointers: q / out rows, the pool, the workspace.
    for i, off in ((1, 2), (2, 64)):
        ts = [pa.as_pa_tensor(t, n, device=False) for t, n in ((q, "out"), (q, "q"), (kc, "k"), (kc, "v"),
                                                                (bt, "bt"), (lens, "lens"))]
        ts[i].data += off
        opts = pa.PaDecodeOpts()
        lib.pa_decode_opts_init(ctypes.byref(opts))
        assert lib.pa_decode(*[ctypes.byref(t) for t in ts], 0.088, Hkv, ctypes.byref(opts), None) == \
            pa.PA_ERR_INVALID_ARG
        assert "aligned" in pa.pa_last_error()
    big = aligned_zeros((1 << 20,), torch.uint8)
    assert call(partition_tokens=256, workspace=big.data_ptr() + 8, workspace_bytes=(1 << 20) - 8) == \
        pa.PA_ERR_INVALID_ARG
    assert "aligned" in pa.pa_last_error()


def test_shared_prefix_blocks_come_from_the_first_sequence_reaching_them():
    """Sequences shorter than the shared prefix: prefix block j is allocated by the first sequence
    that needs it and referenced by every later one, as the oracle's free-list model builds it."""
    lens, npre, nb = [20, 70, 5, 0, 100, 33], 4, 64
    order = np.random.default_rng(8).permutation(nb)
    alloc = pa.BlockAllocator(nb, order.tolist())
    bt = pa.build_block_tables(alloc, lens, 7, shared_prefix_tokens=16 * npre)
    want = paging.build_block_tables(lens, order, nb, 16, 16 * npre, 7)
    assert np.array_equal(bt.numpy(), want)
    need = [-(-n // 16) for n in lens]
    for j in range(npre):
        holders = [s for s in range(len(lens)) if need[s] > j]
        assert len({int(bt[s, j]) for s in holders}) == 1
        assert alloc.refcount(int(bt[holders[0], j])) == len(holders)
    distinct = {int(b) for b in bt.flatten().tolist() if b >= 0}
    assert alloc.num_free == nb - len(distinct)


@settings(max_examples=120, deadline=None)
@given(lens=st.lists(st.integers(0, 90), min_size=0, max_size=9), npre=st.integers(0, 5),
       spare=st.integers(-3, 4), seed=st.integers(0, 2**31 - 1))
def test_build_block_tables_through_the_c_abi(lens, npre, spare, seed):
    """pa_build_block_tables called through ctypes with host arrays: the oracle's tables when the pool
    suffices; otherwise PA_ERR_EXHAUSTED with the allocator and the output untouched."""
    need = [-(-n // 16) for n in lens]
    fresh = sum(max(0, b - npre) for b in need) + max([min(npre, b) for b in need] or [0])
    nb = max(1, fresh + spare)
    mb = max(need or [0]) + 1
    order = np.random.default_rng(seed).permutation(nb).astype(np.int32)
    alloc = pa.BlockAllocator(nb, order.tolist())
    lens_a = np.ascontiguousarray(lens, dtype=np.int32)
    out = np.full((len(lens), mb), 12345, dtype=np.int32)
    i32p = ctypes.POINTER(ctypes.c_int32)
    r = pa.lib().pa_build_block_tables(alloc._h, lens_a.ctypes.data_as(i32p), len(lens), mb, 16 * npre,
                                       out.ctypes.data_as(i32p))
    if fresh <= nb:
        assert r == pa.PA_OK
        want = paging.build_block_tables(lens, order, nb, 16, 16 * npre, mb) if lens else out[:0]
        assert np.array_equal(out, want)
        assert alloc.num_free == nb - fresh
    else:
        assert r == pa.PA_ERR_EXHAUSTED and "free" in pa.pa_last_error()
        assert alloc.num_free == nb and (out == 12345).all()


def test_build_block_tables_rejects_bad_arguments():
    alloc = pa.BlockAllocator(64)
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.build_block_tables(alloc, [10, 40], 2)  # 40 tokens need 3 blocks
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.build_block_tables(alloc, [10, -1], 2)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.build_block_tables(alloc, [10], 2, shared_prefix_tokens=8)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    assert alloc.num_free == 64  # nothing was allocated by the refused calls


def test_no_alloc_decode_checks_arguments_before_the_scratch_lookup():
    """pa_decode_no_alloc finds argument errors, the scratch capacity included, before its first CUDA
    call (the lookup of the built-in array): with host tensors it returns them, not PA_ERR_CUDA."""
    B, Hkv, G, D = 64, 8, 8, 128
    q = aligned_zeros((B, Hkv * G, D), torch.bfloat16)
    kc = aligned_zeros((16, Hkv, 16, D), torch.bfloat16)
    kc16 = aligned_zeros((16, Hkv, 16, D), torch.float16)
    bt = torch.zeros(B, 8192, dtype=torch.int32)
    lens = torch.ones(B, dtype=torch.int32)
    lib = pa.lib()

    def call(kcache=kc, **kw):
        ts = [pa.as_pa_tensor(t, n, device=False) for t, n in ((q, "out"), (q, "q"), (kcache, "k"), (kcache, "v"),
                                                                (bt, "bt"), (lens, "lens"))]
        opts = pa.PaDecodeOpts()
        lib.pa_decode_opts_init(ctypes.byref(opts))
        for k, v in kw.items():
            setattr(opts, k, v)
        return lib.pa_decode_no_alloc(*[ctypes.byref(t) for t in ts], 0.1, Hkv, ctypes.byref(opts), None)

    assert call(kcache=kc16) == pa.PA_ERR_INVALID_ARG
    assert call(partition_tokens=24) == pa.PA_ERR_INVALID_ARG
    # 64 sequences x 64 heads x 512 partitions of 256 tokens: far more than the built-in array.
    assert call(max_context_len=8192 * 16, partition_tokens=256) == pa.PA_ERR_WORKSPACE
    assert "scratch" in pa.pa_last_error()
    small = aligned_zeros((256,), torch.uint8)
    assert call(workspace=small.data_ptr(), workspace_bytes=256) == pa.PA_ERR_INVALID_ARG


@settings(max_examples=120, deadline=None)
@given(n=st.integers(1, 12), pre=st.lists(st.tuples(st.sampled_from("ai"), st.integers(0, 11)), max_size=30),
       batch=st.lists(st.integers(-1, 12), max_size=10), free=st.booleans())
def test_batch_incref_and_free_are_all_or_nothing(n, pre, batch, free):
    """A batch call equals the same single calls in list order when every one of them would succeed,
    and otherwise fails and changes nothing (counts, free list and its order)."""
    a = pa.BlockAllocator(n)
    model = paging.FreeListModel(n, list(range(n)))
    for op, b in pre:  # some state: allocated blocks, some shared
        if op == "a":
            if model.alloc() is not None:
                a.alloc()
        elif model.incref(b):
            a.incref(b)
    trial = copy.deepcopy(model)  # the single calls, applied to a copy
    ok = all((trial.free if free else trial.incref)(b) for b in batch)
    arr = torch.tensor(batch, dtype=torch.int32)
    lib = pa.lib()
    r = (lib.pa_blocks_free_n if free else lib.pa_blocks_incref_n)(a._h, len(batch), pa._i32_ptr(arr))
    want = trial if ok else model
    assert (r == pa.PA_OK) == ok
    if not ok:
        assert r == pa.PA_ERR_BAD_BLOCK
    assert [a.refcount(b) for b in range(n)] == [want.refcount(b) for b in range(n)]
    # The free lists agree in content and order: n allocations drain them identically.
    got = [lib.pa_block_alloc(a._h) for _ in range(a.num_free)]
    assert got == [want.alloc() for _ in range(want.num_free)]


def _partition_rule(B, Hkv, ctx):
    """The partition rule as pa.h states it, restated for the test."""
    units = B * Hkv
    if ctx <= 2048 and units >= 592:
        return 0
    for size in (2048, 1024, 512):
        if ctx > size and units * -(-ctx // size) >= 592:
            return size
    return 256 if ctx > 256 else 0


@settings(max_examples=400, deadline=None)
@given(B=st.integers(1, 300), Hkv=st.sampled_from([1, 2, 4, 8, 32]), ctx=st.integers(1, 200000),
       G=st.sampled_from([1, 4, 8]), D=st.sampled_from([64, 128]))
def test_partition_rule_and_workspace_size(B, Hkv, ctx, G, D):
    pt = pa.pa_decode_partition_tokens(B, Hkv, ctx)
    assert pt == _partition_rule(B, Hkv, ctx)
    P = -(-ctx // pt) if pt else 1
    want = 0 if P <= 1 else -(-(B * Hkv * G * P * D * 4) // 256) * 256 + -(-(B * Hkv * G * P * 2 * 4) // 256) * 256
    assert pa.pa_decode_workspace_bytes(B, Hkv * G, Hkv, D, ctx, 0) == want


def test_allocator_errors_carry_a_reason():
    lib = pa.lib()
    assert not lib.pa_allocator_create(0, None)
    assert "num_blocks" in pa.pa_last_error()
    bad = torch.tensor([0, 2, 2], dtype=torch.int32)
    assert not lib.pa_allocator_create(3, pa._i32_ptr(bad))
    assert "permutation" in pa.pa_last_error()
    a = pa.BlockAllocator(2)
    a.alloc_n(2)
    with pytest.raises(pa.PagedAttentionError, match="2 blocks are in use"):
        a.alloc()
    with pytest.raises(pa.PagedAttentionError, match="block 7 is not allocated"):
        a.incref(7)
    with pytest.raises(pa.PagedAttentionError, match="listed 2 times but referenced 1"):
        a.free_n(torch.tensor([1, 1], dtype=torch.int32))
    with pytest.raises(pa.PagedAttentionError, match="past the table"):
        pa.pa_slots_for_positions(torch.tensor([[0, 1]], dtype=torch.int32), [0], [40])


def test_binding_declares_every_entry_point():
    """The ctypes binding gives every function of the header its argument and result types (a call
    through an undeclared signature would pass Python ints as C ints and truncate pointers)."""
    lib = pa.lib()
    undeclared = [n for n in declared_functions() if getattr(lib, n).argtypes is None]
    assert not undeclared, undeclared


def test_binding_signatures_match_the_header_arity():
    """Each ctypes signature has as many arguments as the header's prototype."""
    protos = {}
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if hdr.endswith(".h"):
            text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", hdr)).read(), flags=re.S)
            for name, params in re.findall(r"\b(pa_[a-z0-9_]+)\s*\(([^;{}]*?)\)\s*;", text):
                p = " ".join(params.split())
                protos[name] = 0 if p in ("", "void") else p.count(",") + 1
    lib = pa.lib()
    assert set(protos) == set(declared_functions())
    wrong = {n: (k, len(getattr(lib, n).argtypes)) for n, k in protos.items() if len(getattr(lib, n).argtypes) != k}
    assert not wrong, wrong


def test_struct_layouts_match_the_header(tmp_path):
    """The ctypes mirrors of pa_tensor and pa_decode_opts have the C structs' sizes and field offsets
    (compiled from include/pa.h with the host C compiler)."""
    import shutil
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    fields = {"pa_tensor": [f[0] for f in pa.PaTensor._fields_],
              "pa_decode_opts": [f[0] for f in pa.PaDecodeOpts._fields_]}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "pa.h"', "int main(void) {"]
    for st_, names in fields.items():
        lines.append(f'  printf("{st_} size %zu\\n", sizeof({st_}));')
        lines += [f'  printf("{st_} {n} %zu\\n", offsetof({st_}, {n}));' for n in names]
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = dict(ln.rsplit(" ", 1) for ln in subprocess.run([str(exe)], capture_output=True, text=True,
                                                          check=True).stdout.splitlines())
    for st_, cls in (("pa_tensor", pa.PaTensor), ("pa_decode_opts", pa.PaDecodeOpts)):
        assert int(got[f"{st_} size"]) == ctypes.sizeof(cls)
        for n in fields[st_]:
            assert int(got[f"{st_} {n}"]) == getattr(cls, n).offset, (st_, n)


def test_no_alloc_scratch_size_matches_the_header():
    """The binding's NO_ALLOC_SCRATCH_BYTES is the header's PA_NO_ALLOC_SCRATCH_BYTES."""
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    m = re.search(r"#define PA_NO_ALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert m, "PA_NO_ALLOC_SCRATCH_BYTES is not defined as ((size_t)a << b)"
    assert pa.NO_ALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
