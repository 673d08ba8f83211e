"""B200-native paged-KV-cache decode: Python binding over the C ABI of ``libpagedattn.so``.

The functions here carry the C names (``include/pa.h``) and only marshal arguments: torch tensors
become ``pa_tensor`` views, the current CUDA stream is passed through, a non-OK status raises
``PagedAttentionError``. Every step of the hot path runs in the library's CUDA kernels; there is no
CPU fallback. Device arguments must be CUDA tensors.

Build the library first (``python paged_kv_cache_385_b200/build.py``); importing this package
without it raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# PAGED_KV_CACHE_LIB points the binding at another build of the library (e.g. a tuning variant).
LIB_PATH = os.environ.get("PAGED_KV_CACHE_LIB") or os.path.join(_HERE, "libpagedattn.so")

PA_OK = 0
PA_ERR_INVALID_ARG = -1
PA_ERR_UNSUPPORTED = -2
PA_ERR_WORKSPACE = -3
PA_ERR_CUDA = -4
PA_ERR_EXHAUSTED = -5
PA_ERR_BAD_BLOCK = -6

PA_F16, PA_BF16, PA_E4M3, PA_I32, PA_I64, PA_F32 = range(6)

PA_DEVERR_BAD_BLOCK = 1
PA_DEVERR_BAD_SLOT = 2
PA_DEVERR_TIMEOUT = 4
PA_DEVERR_CTX_RANGE = 8
PA_DEVERR_PREFIX = 16

BLOCK_SIZE = 16

_DTYPES = {
    torch.float16: PA_F16,
    torch.bfloat16: PA_BF16,
    torch.float8_e4m3fn: PA_E4M3,
    torch.int32: PA_I32,
    torch.int64: PA_I64,
    torch.float32: PA_F32,
}


class PaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class PaDecodeOpts(ctypes.Structure):
    _fields_ = [("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float), ("max_context_len", ctypes.c_int32),
                ("partition_tokens", ctypes.c_int32), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t), ("kernel", ctypes.c_int32),
                ("error_word", ctypes.c_void_p), ("prefix_kernel", ctypes.c_int32)]


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {status_string(status)} ({status}): {detail}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python paged_kv_cache_385_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, F32, SZ, VP = (ctypes.POINTER(PaTensor), ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                ctypes.c_size_t, ctypes.c_void_p)
    i32p = ctypes.POINTER(ctypes.c_int32)
    sig = {
        "pa_decode_opts_init": (None, [ctypes.POINTER(PaDecodeOpts)]),
        "pa_reshape_and_cache": (ctypes.c_int, [P, P, P, P, P, F32, F32, VP]),
        "pa_decode": (ctypes.c_int, [P, P, P, P, P, P, F32, I32, ctypes.POINTER(PaDecodeOpts), VP]),
        "pa_decode_step": (ctypes.c_int, [P, P, P, P, P, P, P, P, P, F32, I32, ctypes.POINTER(PaDecodeOpts), VP]),
        "pa_decode_cascade": (ctypes.c_int, [P, P, P, P, P, P, P, P, P, I32, F32, I32,
                                             ctypes.POINTER(PaDecodeOpts), VP]),
        "pa_decode_cascade_workspace_bytes": (SZ, [I32, I32, I32, I32, I32, I32, I32]),
        "pa_prefill": (ctypes.c_int, [P, P, P, P, P, P, P, I32, F32, I32, I32, VP]),
        "pa_decode_no_alloc": (ctypes.c_int, [P, P, P, P, P, P, F32, I32, ctypes.POINTER(PaDecodeOpts), VP]),
        "pa_decode_partition_tokens": (I32, [I32, I32, I32]),
        "pa_decode_workspace_bytes": (SZ, [I32, I32, I32, I32, I32, I32]),
        "pa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "pa_last_error": (ctypes.c_char_p, []),
        "pa_read_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]),
        "pa_version": (ctypes.c_char_p, []),
        "pa_debug_fail_next_launches": (ctypes.c_int, [I32]),
        "pa_selftest_bounded_wait": (ctypes.c_int, [I32, ctypes.c_void_p, VP]),
        "pa_allocator_create": (VP, [I32, i32p]),
        "pa_allocator_destroy": (None, [VP]),
        "pa_block_alloc": (I32, [VP]),
        "pa_block_incref": (ctypes.c_int, [VP, I32]),
        "pa_block_free": (ctypes.c_int, [VP, I32]),
        "pa_block_refcount": (I32, [VP, I32]),
        "pa_block_cow": (ctypes.c_int, [VP, I32, i32p]),
        "pa_copy_blocks": (ctypes.c_int, [P, P, P, VP]),
        "pa_allocator_num_free": (I32, [VP]),
        "pa_allocator_num_blocks": (I32, [VP]),
        "pa_blocks_alloc_n": (ctypes.c_int, [VP, I32, i32p]),
        "pa_blocks_incref_n": (ctypes.c_int, [VP, I32, i32p]),
        "pa_blocks_free_n": (ctypes.c_int, [VP, I32, i32p]),
        "pa_build_block_tables": (ctypes.c_int, [VP, i32p, I32, I32, I32, i32p]),
        "pa_slots_for_positions": (ctypes.c_int, [i32p, I64, I32, I32, i32p, i32p, I64,
                                                  ctypes.POINTER(ctypes.c_int64)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def lib() -> ctypes.CDLL:
    """The loaded ``libpagedattn.so`` handle."""
    return _lib


def status_string(status: int) -> str:
    return _lib.pa_status_string(status).decode()


def _check(status: int, where: str) -> None:
    if status != PA_OK:
        raise PagedAttentionError(status, where, _lib.pa_last_error().decode())


def as_pa_tensor(t: Optional[torch.Tensor], name: str, device: bool = True) -> PaTensor:
    """A pa_tensor view of a torch tensor (no copy)."""
    if t is None:
        raise ValueError(f"{name} is None")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype not in _DTYPES:
        raise TypeError(f"{name}: unsupported dtype {t.dtype}")
    if t.dim() > 4:
        raise ValueError(f"{name}: more than 4 dimensions")
    pt = PaTensor()
    pt.data = t.data_ptr()
    pt.dtype = _DTYPES[t.dtype]
    pt.ndim = t.dim()
    for i in range(t.dim()):
        pt.shape[i] = t.shape[i]
        pt.stride[i] = t.stride(i)
    return pt


def _stream_handle(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def pa_reshape_and_cache(key: torch.Tensor, value: torch.Tensor, slot_mapping: torch.Tensor, k_cache: torch.Tensor,
                         v_cache: torch.Tensor, k_scale: float = 1.0, v_scale: float = 1.0, stream=None) -> None:
    """Write new tokens' K/V into their slots (see ``pa_reshape_and_cache`` in include/pa.h)."""
    args = [as_pa_tensor(key, "key"), as_pa_tensor(value, "value"), as_pa_tensor(slot_mapping, "slot_mapping"),
            as_pa_tensor(k_cache, "k_cache"), as_pa_tensor(v_cache, "v_cache")]
    _check(_lib.pa_reshape_and_cache(*[ctypes.byref(a) for a in args], float(k_scale), float(v_scale),
                                     ctypes.c_void_p(_stream_handle(stream))), "pa_reshape_and_cache")


def pa_copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, block_mapping: torch.Tensor, stream=None) -> None:
    """Copy whole blocks (src, dst) of both caches for copy-on-write (see include/pa.h)."""
    args = [as_pa_tensor(k_cache, "k_cache"), as_pa_tensor(v_cache, "v_cache"),
            as_pa_tensor(block_mapping, "block_mapping")]
    _check(_lib.pa_copy_blocks(*[ctypes.byref(a) for a in args], ctypes.c_void_p(_stream_handle(stream))),
           "pa_copy_blocks")


def decode_opts(k_scale: float = 1.0, v_scale: float = 1.0, max_context_len: int = 0, partition_tokens: int = 0,
                workspace: Optional[torch.Tensor] = None, kernel: int = -1,
                error_word: Optional[torch.Tensor] = None, prefix_kernel: int = -1) -> PaDecodeOpts:
    o = PaDecodeOpts()
    _lib.pa_decode_opts_init(ctypes.byref(o))
    o.k_scale = k_scale
    o.v_scale = v_scale
    o.max_context_len = int(max_context_len)
    o.partition_tokens = int(partition_tokens)
    if workspace is not None:
        if not workspace.is_cuda:
            raise ValueError("workspace must be a CUDA tensor")
        o.workspace = workspace.data_ptr()
        o.workspace_bytes = workspace.numel() * workspace.element_size()
    o.kernel = int(kernel)
    o.prefix_kernel = int(prefix_kernel)
    if error_word is not None:
        if not error_word.is_cuda or error_word.dtype != torch.int32:
            raise ValueError("error_word must be a CUDA int32 tensor")
        o.error_word = error_word.data_ptr()
    return o


def pa_decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float, num_kv_heads: int,
              opts: Optional[PaDecodeOpts] = None, stream=None, **kw) -> None:
    """One paged-attention decode step (see ``pa_decode`` in include/pa.h). ``kw`` builds ``opts``."""
    if opts is None:
        opts = decode_opts(**kw)
    elif kw:
        raise TypeError("pass either opts or keyword options, not both")
    args = [as_pa_tensor(out, "out"), as_pa_tensor(q, "q"), as_pa_tensor(k_cache, "k_cache"),
            as_pa_tensor(v_cache, "v_cache"), as_pa_tensor(block_tables, "block_tables"),
            as_pa_tensor(context_lens, "context_lens")]
    _check(_lib.pa_decode(*[ctypes.byref(a) for a in args], float(scale), int(num_kv_heads), ctypes.byref(opts),
                          ctypes.c_void_p(_stream_handle(stream))), "pa_decode")


def pa_decode_step(out: torch.Tensor, q: torch.Tensor, key: torch.Tensor, value: torch.Tensor,
                   slot_mapping: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                   block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float, num_kv_heads: int,
                   opts: Optional[PaDecodeOpts] = None, stream=None, **kw) -> None:
    """pa_reshape_and_cache of one new token per sequence + pa_decode in one launch (include/pa.h)."""
    if opts is None:
        opts = decode_opts(**kw)
    elif kw:
        raise TypeError("pass either opts or keyword options, not both")
    args = [as_pa_tensor(out, "out"), as_pa_tensor(q, "q"), as_pa_tensor(key, "key"), as_pa_tensor(value, "value"),
            as_pa_tensor(slot_mapping, "slot_mapping"), as_pa_tensor(k_cache, "k_cache"),
            as_pa_tensor(v_cache, "v_cache"), as_pa_tensor(block_tables, "block_tables"),
            as_pa_tensor(context_lens, "context_lens")]
    _check(_lib.pa_decode_step(*[ctypes.byref(a) for a in args], float(scale), int(num_kv_heads), ctypes.byref(opts),
                               ctypes.c_void_p(_stream_handle(stream))), "pa_decode_step")


def pa_decode_cascade(out: torch.Tensor, q: torch.Tensor, key: Optional[torch.Tensor], value: Optional[torch.Tensor],
                      slot_mapping: Optional[torch.Tensor], k_cache: torch.Tensor, v_cache: torch.Tensor,
                      block_tables: torch.Tensor, context_lens: torch.Tensor, shared_prefix_tokens: int, scale: float,
                      num_kv_heads: int, opts: Optional[PaDecodeOpts] = None, stream=None, **kw) -> None:
    """Decode with a prefix shared by every sequence read once per KV head (see include/pa.h)."""
    if opts is None:
        opts = decode_opts(**kw)
    elif kw:
        raise TypeError("pass either opts or keyword options, not both")
    nk = [None if t is None else ctypes.byref(as_pa_tensor(t, n)) for t, n in
          ((key, "key"), (value, "value"), (slot_mapping, "slot_mapping"))]
    args = [as_pa_tensor(out, "out"), as_pa_tensor(q, "q")]
    rest = [as_pa_tensor(k_cache, "k_cache"), as_pa_tensor(v_cache, "v_cache"),
            as_pa_tensor(block_tables, "block_tables"), as_pa_tensor(context_lens, "context_lens")]
    _check(_lib.pa_decode_cascade(*[ctypes.byref(a) for a in args], *nk, *[ctypes.byref(a) for a in rest],
                                  int(shared_prefix_tokens), float(scale), int(num_kv_heads), ctypes.byref(opts),
                                  ctypes.c_void_p(_stream_handle(stream))), "pa_decode_cascade")


def pa_decode_cascade_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                                      max_context_len: int, shared_prefix_tokens: int, partition_tokens: int = 0) -> int:
    return int(_lib.pa_decode_cascade_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                                      shared_prefix_tokens, partition_tokens))


def pa_prefill(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
               block_tables: torch.Tensor, query_start: torch.Tensor, context_lens: torch.Tensor, max_query_len: int,
               scale: float, num_kv_heads: int, kernel: int = -1, stream=None) -> None:
    """Causal attention of each sequence's new tokens over its paged context (see include/pa.h)."""
    args = [as_pa_tensor(out, "out"), as_pa_tensor(q, "q"), as_pa_tensor(k_cache, "k_cache"),
            as_pa_tensor(v_cache, "v_cache"), as_pa_tensor(block_tables, "block_tables"),
            as_pa_tensor(query_start, "query_start"), as_pa_tensor(context_lens, "context_lens")]
    _check(_lib.pa_prefill(*[ctypes.byref(a) for a in args], int(max_query_len), float(scale), int(num_kv_heads),
                           int(kernel), ctypes.c_void_p(_stream_handle(stream))), "pa_prefill")


def pa_selftest_bounded_wait(timeout_us: int, error_word: Optional[torch.Tensor] = None, stream=None) -> None:
    """Run the library's bounded barrier wait against a barrier nothing arrives on (see include/pa.h):
    it gives up after timeout_us and sets PA_DEVERR_TIMEOUT in error_word (or the library's word)."""
    ptr = None
    if error_word is not None:
        if not error_word.is_cuda or error_word.dtype != torch.int32:
            raise ValueError("error_word must be a CUDA int32 tensor")
        ptr = error_word.data_ptr()
    _check(_lib.pa_selftest_bounded_wait(int(timeout_us), ctypes.c_void_p(ptr), ctypes.c_void_p(_stream_handle(stream))),
           "pa_selftest_bounded_wait")


# Size of the library's built-in scratch array used by pa_decode_no_alloc (PA_NO_ALLOC_SCRATCH_BYTES).
NO_ALLOC_SCRATCH_BYTES = 32 << 20


def pa_decode_no_alloc(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                       block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float, num_kv_heads: int,
                       opts: Optional[PaDecodeOpts] = None, stream=None, **kw) -> None:
    """pa_decode for callers that cannot allocate device memory (see ``pa_decode_no_alloc`` in include/pa.h).

    The split-partition scratch comes from a fixed array inside the library, so no ``workspace``
    may be passed. Batches needing more than ``NO_ALLOC_SCRATCH_BYTES`` of scratch are rejected.
    """
    if opts is None:
        opts = decode_opts(**kw)
    elif kw:
        raise TypeError("pass either opts or keyword options, not both")
    args = [as_pa_tensor(out, "out"), as_pa_tensor(q, "q"), as_pa_tensor(k_cache, "k_cache"),
            as_pa_tensor(v_cache, "v_cache"), as_pa_tensor(block_tables, "block_tables"),
            as_pa_tensor(context_lens, "context_lens")]
    _check(_lib.pa_decode_no_alloc(*[ctypes.byref(a) for a in args], float(scale), int(num_kv_heads),
                                   ctypes.byref(opts), ctypes.c_void_p(_stream_handle(stream))),
           "pa_decode_no_alloc")


def pa_decode_partition_tokens(num_seqs: int, num_kv_heads: int, max_context_len: int) -> int:
    return int(_lib.pa_decode_partition_tokens(num_seqs, num_kv_heads, max_context_len))


def pa_decode_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                              max_context_len: int, partition_tokens: int = 0) -> int:
    return int(_lib.pa_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                              partition_tokens))


def decode_workspace(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int, max_context_len: int,
                     partition_tokens: int = 0, device=None) -> Optional[torch.Tensor]:
    """A device workspace big enough for these sizes (None when no split happens)."""
    n = pa_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, partition_tokens)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def pa_read_device_error(clear: bool = True) -> int:
    bits = ctypes.c_uint32(0)
    _check(_lib.pa_read_device_error(ctypes.byref(bits), int(clear)), "pa_read_device_error")
    return bits.value


def pa_status_string(status: int) -> str:
    return status_string(status)


def pa_last_error() -> str:
    return _lib.pa_last_error().decode()


def pa_version() -> str:
    return _lib.pa_version().decode()


def pa_debug_fail_next_launches(count: int) -> None:
    """Host-side fault injection: the next ``count`` calls that pass their argument checks raise
    PagedAttentionError(PA_ERR_CUDA) without device work, as a failed launch does (see include/pa.h)."""
    _check(_lib.pa_debug_fail_next_launches(int(count)), "pa_debug_fail_next_launches")


def _i32_ptr(t: torch.Tensor):
    return ctypes.cast(t.data_ptr(), ctypes.POINTER(ctypes.c_int32))


def pa_slots_for_positions(block_tables: torch.Tensor, token_seq: Sequence[int], token_pos: Sequence[int]) -> torch.Tensor:
    """Host helper: int64 slots of (sequence, position) pairs through a host int32 block table."""
    bt = block_tables.to("cpu", torch.int32).contiguous()
    seq = torch.as_tensor(token_seq, dtype=torch.int32).contiguous()
    pos = torch.as_tensor(token_pos, dtype=torch.int32).contiguous()
    out = torch.empty(seq.numel(), dtype=torch.int64)
    _check(_lib.pa_slots_for_positions(_i32_ptr(bt), bt.shape[1], bt.shape[0], bt.shape[1], _i32_ptr(seq),
                                       _i32_ptr(pos), seq.numel(),
                                       ctypes.cast(out.data_ptr(), ctypes.POINTER(ctypes.c_int64))),
           "pa_slots_for_positions")
    return out


class BlockAllocator:
    """Host free-list block allocator with reference counts (``pa_allocator_*`` in include/pa.h)."""

    def __init__(self, num_blocks: int, initial_order: Optional[Sequence[int]] = None):
        order = None
        if initial_order is not None:
            order = torch.as_tensor(initial_order, dtype=torch.int32).contiguous()
            if order.numel() != num_blocks:
                raise ValueError("initial_order must hold num_blocks ids")
        self._order = order  # keep alive during create
        h = _lib.pa_allocator_create(int(num_blocks), _i32_ptr(order) if order is not None else None)
        if not h:
            raise ValueError(f"pa_allocator_create: {pa_last_error()}")
        self._h = ctypes.c_void_p(h)
        self._destroy = _lib.pa_allocator_destroy  # still reachable during interpreter shutdown

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._destroy(h)
            self._h = None

    def alloc(self) -> int:
        b = int(_lib.pa_block_alloc(self._h))
        if b < 0:
            _check(b, "pa_block_alloc")
        return b

    def alloc_n(self, n: int) -> torch.Tensor:
        out = torch.empty(n, dtype=torch.int32)
        _check(_lib.pa_blocks_alloc_n(self._h, int(n), _i32_ptr(out)), "pa_blocks_alloc_n")
        return out

    def incref(self, block: int) -> None:
        _check(_lib.pa_block_incref(self._h, int(block)), "pa_block_incref")

    def incref_n(self, blocks: torch.Tensor) -> None:
        b = blocks.to(torch.int32).contiguous()
        _check(_lib.pa_blocks_incref_n(self._h, b.numel(), _i32_ptr(b)), "pa_blocks_incref_n")

    def free(self, block: int) -> None:
        _check(_lib.pa_block_free(self._h, int(block)), "pa_block_free")

    def free_n(self, blocks: torch.Tensor) -> None:
        b = blocks.to(torch.int32).contiguous()
        _check(_lib.pa_blocks_free_n(self._h, b.numel(), _i32_ptr(b)), "pa_blocks_free_n")

    def cow(self, block: int):
        """Copy-on-write before writing into ``block``: returns (block_to_write, needs_copy)."""
        out = ctypes.c_int32(-1)
        r = int(_lib.pa_block_cow(self._h, int(block), ctypes.byref(out)))
        if r < 0:
            _check(r, "pa_block_cow")
        return int(out.value), r == 1

    def refcount(self, block: int) -> int:
        return int(_lib.pa_block_refcount(self._h, int(block)))

    @property
    def num_free(self) -> int:
        return int(_lib.pa_allocator_num_free(self._h))

    @property
    def num_blocks(self) -> int:
        return int(_lib.pa_allocator_num_blocks(self._h))


def build_block_tables(alloc: BlockAllocator, context_lens: Sequence[int], max_blocks: int,
                       shared_prefix_tokens: int = 0) -> torch.Tensor:
    """Host int32 block tables [num_seqs, max_blocks] (-1 padded) from the allocator
    (``pa_build_block_tables`` in include/pa.h: sequences in order, one allocation per logical block,
    shared-prefix blocks allocated by the first sequence reaching them and referenced by later ones)."""
    lens = torch.as_tensor([int(c) for c in context_lens], dtype=torch.int32).contiguous()
    bt = torch.empty((lens.numel(), int(max_blocks)), dtype=torch.int32)
    _check(_lib.pa_build_block_tables(alloc._h, _i32_ptr(lens), lens.numel(), int(max_blocks),
                                      int(shared_prefix_tokens), _i32_ptr(bt)), "pa_build_block_tables")
    return bt
