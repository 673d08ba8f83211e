"""Device-side view of a seeded workload, built only through the library's public API.

Block tables come from the library's allocator, slots from its slot helper, the pool from
``pa_reshape_and_cache`` (history in batches, then the step's new token), outputs from
``pa_decode``. Tests compare each of these against ``tests/oracle_case.py``.
"""
from __future__ import annotations

from typing import Optional

import torch

import paged_kv_cache_385_b200 as pa
import workloads as W

TORCH_KV = {"f16": torch.float16, "bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn}
TOL = {"f16": 5e-3, "bf16": 1.5e-2, "e4m3": 3e-2}  # max abs error vs the float64 oracle


class DeviceCase:
    def __init__(self, w: W.Workload, order: Optional[torch.Tensor] = None, sentinel: bool = True,
                 device: str = "cuda", fill_batch_tokens: int = 1 << 16, history: bool = True):
        self.w = w
        self.device = device
        self.lens_host = W.context_lens(w)
        order = W.block_order(w) if order is None else order
        self.alloc = pa.BlockAllocator(w.num_blocks, order.tolist())
        self.max_blocks = W.max_blocks_per_seq(w, self.lens_host)
        self.bt_host = pa.build_block_tables(self.alloc, self.lens_host.tolist(), self.max_blocks,
                                             w.shared_prefix_tokens)
        self.k_scale, self.v_scale = W.fp8_scales(w)
        kv_dt = TORCH_KV[w.kv_dtype]
        shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
        if sentinel:
            self.k_cache = W.sentinel_pool(w, "sentinel/k").to(device).view(kv_dt).view(shape)
            self.v_cache = W.sentinel_pool(w, "sentinel/v").to(device).view(kv_dt).view(shape)
        else:
            self.k_cache = torch.zeros(shape, dtype=kv_dt, device=device)
            self.v_cache = torch.zeros(shape, dtype=kv_dt, device=device)
        self.q = W.query(w).to(device)
        self.bt = self.bt_host.to(device)
        self.lens = self.lens_host.to(device)
        self.out = torch.empty_like(self.q)
        if history:
            self._fill_history(fill_batch_tokens)
        # The step's new token: position ctx - 1 of every sequence.
        B = w.num_seqs
        keys, vals = [], []
        for s in range(B):
            n = int(self.lens_host[s])
            k = W.kv_source(w, s, "k", self.lens_host)
            v = W.kv_source(w, s, "v", self.lens_host)
            keys.append(k[n - 1:n])
            vals.append(v[n - 1:n])
        self.new_k = torch.cat(keys).to(device)
        self.new_v = torch.cat(vals).to(device)
        self.new_slots = pa.pa_slots_for_positions(self.bt_host, list(range(B)),
                                                   [int(n) - 1 for n in self.lens_host]).to(device)
        self.max_ctx = int(self.lens_host.max())

    def _fill_history(self, batch_tokens: int) -> None:
        """Write positions [start, ctx - 1) of every sequence; shared-prefix rows once (sequence 0)."""
        w = self.w
        pend_k, pend_v, pend_s, pend_p = [], [], [], []
        count = 0

        def flush():
            nonlocal pend_k, pend_v, pend_s, pend_p, count
            if not pend_k:
                return
            k = torch.cat(pend_k).to(self.device)
            v = torch.cat(pend_v).to(self.device)
            slots = pa.pa_slots_for_positions(self.bt_host, pend_s, pend_p).to(self.device)
            pa.pa_reshape_and_cache(k, v, slots, self.k_cache, self.v_cache, self.k_scale, self.v_scale)
            pend_k, pend_v, pend_s, pend_p, count = [], [], [], [], 0

        for s in range(w.num_seqs):
            n = int(self.lens_host[s])
            start = 0 if s == 0 else min(w.shared_prefix_tokens, n - 1)
            if n - 1 <= start:
                continue
            k = W.kv_source(w, s, "k", self.lens_host)[start:n - 1]
            v = W.kv_source(w, s, "v", self.lens_host)[start:n - 1]
            pend_k.append(k)
            pend_v.append(v)
            pend_s += [s] * (n - 1 - start)
            pend_p += list(range(start, n - 1))
            count += n - 1 - start
            if count >= batch_tokens:
                flush()
        flush()

    def write_new_token(self) -> None:
        pa.pa_reshape_and_cache(self.new_k, self.new_v, self.new_slots, self.k_cache, self.v_cache, self.k_scale,
                                self.v_scale)

    def workspace(self, partition_tokens: int = 0) -> Optional[torch.Tensor]:
        w = self.w
        return pa.decode_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, self.max_ctx, partition_tokens)

    def decode(self, kernel: int = -1, partition_tokens: Optional[int] = None, out: Optional[torch.Tensor] = None,
               error_word: Optional[torch.Tensor] = None) -> torch.Tensor:
        w = self.w
        pt = w.partition_tokens if partition_tokens is None else partition_tokens
        out = self.out if out is None else out
        pa.pa_decode(out, self.q, self.k_cache, self.v_cache, self.bt, self.lens, w.scale, w.num_kv_heads,
                     k_scale=self.k_scale, v_scale=self.v_scale, max_context_len=self.max_ctx, partition_tokens=pt,
                     workspace=self.workspace(pt), kernel=kernel, error_word=error_word)
        return out

    def step(self, **kw) -> torch.Tensor:
        self.write_new_token()
        return self.decode(**kw)

    def step_fused(self, kernel: int = -1, partition_tokens: Optional[int] = None,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """pa_decode_step: the new-token write and the decode in one launch."""
        w = self.w
        pt = w.partition_tokens if partition_tokens is None else partition_tokens
        out = self.out if out is None else out
        pa.pa_decode_step(out, self.q, self.new_k, self.new_v, self.new_slots, self.k_cache, self.v_cache, self.bt,
                          self.lens, w.scale, w.num_kv_heads, k_scale=self.k_scale, v_scale=self.v_scale,
                          max_context_len=self.max_ctx, partition_tokens=pt, workspace=self.workspace(pt),
                          kernel=kernel)
        return out

    def cascade(self, fused: bool = True, partition_tokens: int = 0, out: Optional[torch.Tensor] = None,
                error_word: Optional[torch.Tensor] = None, prefix_kernel: int = -1) -> torch.Tensor:
        """pa_decode_cascade over the workload's shared prefix (with the new-token write if fused)."""
        w = self.w
        out = self.out if out is None else out
        n = pa.pa_decode_cascade_workspace_bytes(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, self.max_ctx,
                                                 w.shared_prefix_tokens, partition_tokens)
        ws = torch.empty(n, dtype=torch.uint8, device=self.device)
        nk = (self.new_k, self.new_v, self.new_slots) if fused else (None, None, None)
        pa.pa_decode_cascade(out, self.q, *nk, self.k_cache, self.v_cache, self.bt, self.lens,
                             w.shared_prefix_tokens, w.scale, w.num_kv_heads, max_context_len=self.max_ctx,
                             partition_tokens=partition_tokens, workspace=ws, error_word=error_word,
                             prefix_kernel=prefix_kernel)
        return out

    def pool_bytes(self):
        """(k, v) pools as host uint8 [NB, Hkv, 16, D * elem]."""
        w = self.w
        shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim * w.kv_elem_bytes)
        return (self.k_cache.view(torch.uint8).reshape(shape).cpu().numpy(),
                self.v_cache.view(torch.uint8).reshape(shape).cpu().numpy())
