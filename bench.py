"""Benchmark of one paged-attention decode step on B200: KV-read HBM GB/s and microseconds per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is the whole hot path for one batch: the write of the batch's new tokens into their slots
and the decode attention over every sequence's pages (plus the partition merge when the context is
split). By default (``--step fused``) both run in one launch, ``pa_decode_step``; ``--step separate``
calls ``pa_reshape_and_cache`` then ``pa_decode``; ``--step cascade`` calls ``pa_decode_cascade``.
The default workload is the Llama-7B-shaped MHA batch: 32 sequences x 2048 tokens, 32 query = 32 KV
heads, head_dim 128, fp16, 16-token blocks scattered through a 5120-block pool. Its KV cache
(1.07 GB per step) is far larger than L2 (126 MB), so no L2 flush is needed between steps.

value = algorithmic KV bytes read per step (sum_s ctx_s * Hkv * D * 2 B * 2) x ranks / step time.
Under torchrun every rank runs the same batch on its own GPU (replicas; the path has no exchange
step), so scaling is weak. ``--impl reference`` times the float64 CPU oracle on a bounded sample of
the same workload on this host's cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "paged decode attention: KV-read HBM GB/s (% of B200 peak) and µs/decode step"
TORCH_KV = {"f16": torch.float16, "bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn}
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama7b_mha", choices=sorted(W.FULL))
    ap.add_argument("--kernel", type=int, default=-1,
                    help="-1 library choice, 0 CUDA-core, 1 tensor-core, 2 tensor-core with one CTA per partition")
    ap.add_argument("--partition-tokens", type=int, default=None)
    ap.add_argument("--step", choices=["fused", "separate", "cascade"], default="fused",
                    help="fused: pa_decode_step (new-token write inside the decode launch); "
                         "separate: pa_reshape_and_cache then pa_decode; "
                         "cascade: pa_decode_cascade over the workload's shared prefix (prefix_gqa)")
    ap.add_argument("--op", choices=["step", "copy_blocks", "kv_utilization", "prefill"], default="step",
                    help="step: the decode step (the headline); copy_blocks: copy-on-write block copies; "
                         "kv_utilization: KV memory utilisation of the block allocator (host only)")
    ap.add_argument("--prefix-kernel", type=int, default=-1,
                    help="--step cascade: shared-prefix kernel, -1 library choice, 0 warp-level mma, 1 tcgen05")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(value_ms: float, device=None) -> float:
    """The slowest rank's time: every rank passes its own device time, all get the maximum.

    Replicas run the same batch on every GPU with no exchange step, so the job's throughput is the
    units all ranks processed over the slowest rank's time.
    """
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value_ms
    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank_step: int, world: int, max_ms_per_step: float) -> float:
    """Whole-job GB/s: all ranks' bytes per step over the slowest rank's step time."""
    return bytes_per_rank_step * world / (max_ms_per_step / 1e3) / 1e9


# ---------------------------------------------------------------------------------------------
# Clock sampling during the timed region (NVML, every 20 ms).
# ---------------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h, self.matched_by = self.nvml_handle(pynvml, device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.error = f"{type(e).__name__}: {e}"

    @staticmethod
    def nvml_handle(nv, device_index: int):
        """NVML handle of the GPU torch calls cuda:device_index. NVML numbers every GPU of the machine
        while CUDA numbers only the visible ones (CUDA_VISIBLE_DEVICES), so match by UUID; fall back
        to the index when the UUID is not available."""
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            return nv.nvmlDeviceGetHandleByUUID("GPU-" + uuid), "uuid"
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(device_index), "index"

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            self._stop.wait(0.02)

    def sample(self):
        if not self._ok:
            return
        try:
            self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
            self.reasons |= self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        except Exception:
            pass

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self.sample()
        self._stop.set()
        self._t.join()

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.error}
        names = [n for n, bit in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples), "nvml_device_matched_by": self.matched_by}


# ---------------------------------------------------------------------------------------------
# Our implementation: setup through the C ABI, device-timed steps, e2e with host buffers.
# ---------------------------------------------------------------------------------------------
class Setup:
    """Device state of one workload, built through the library (history written by pa_reshape_and_cache)."""

    def __init__(self, w: W.Workload, device: torch.device, kernel: int, partition_tokens):
        import paged_kv_cache_385_b200 as pa
        self.pa = pa
        self.w = w
        self.device = device
        self.kernel = kernel
        lens = W.context_lens(w)
        self.lens_host = lens
        self.max_ctx = int(lens.max())
        alloc = pa.BlockAllocator(w.num_blocks, W.block_order(w).tolist())
        self.max_blocks = W.max_blocks_per_seq(w, lens)
        self.bt_host = pa.build_block_tables(alloc, lens.tolist(), self.max_blocks, w.shared_prefix_tokens)
        self.alloc = alloc
        kv_dt = TORCH_KV[w.kv_dtype]
        shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
        self.k_cache = torch.zeros(shape, dtype=kv_dt, device=device)
        self.v_cache = torch.zeros(shape, dtype=kv_dt, device=device)
        g = torch.Generator(device=device)
        g.manual_seed(w.seed)
        src = w.source_dtype
        self.k_scale = self.v_scale = 1.0
        if w.kv_dtype == "e4m3":
            # N(0, 1) sources: per-tensor scale from the amax of a large draw of the same distribution.
            self.k_scale = self.v_scale = float(torch.tensor(5.5 / 448.0, dtype=torch.float32))
        # History: positions [start, ctx - 1) of each sequence, written in batches of <= 16K tokens.
        seqs, poss = [], []
        for s in range(w.num_seqs):
            n = int(lens[s])
            start = 0 if s == 0 else min(w.shared_prefix_tokens, n - 1)
            seqs += [s] * max(0, n - 1 - start)
            poss += list(range(start, n - 1))
        slots = pa.pa_slots_for_positions(self.bt_host, seqs, poss)
        chunk = 16384
        for i in range(0, len(seqs), chunk):
            sl = slots[i:i + chunk].to(device)
            k = torch.randn(sl.numel(), w.num_kv_heads, w.head_dim, generator=g, device=device).to(src)
            v = torch.randn(sl.numel(), w.num_kv_heads, w.head_dim, generator=g, device=device).to(src)
            pa.pa_reshape_and_cache(k, v, sl, self.k_cache, self.v_cache, self.k_scale, self.v_scale)
        B = w.num_seqs
        self.new_k = torch.randn(B, w.num_kv_heads, w.head_dim, generator=g, device=device).to(src)
        self.new_v = torch.randn(B, w.num_kv_heads, w.head_dim, generator=g, device=device).to(src)
        self.new_slots = pa.pa_slots_for_positions(self.bt_host, list(range(B)),
                                                   [int(n) - 1 for n in lens]).to(device)
        self.q = torch.randn(B, w.num_q_heads, w.head_dim, generator=g, device=device).to(w.q_torch_dtype)
        self.out = torch.empty_like(self.q)
        self.bt = self.bt_host.to(device)
        self.lens = lens.to(device)
        pt = w.partition_tokens if partition_tokens is None else partition_tokens
        self.pt = pt
        self.ws = pa.decode_workspace(B, w.num_q_heads, w.num_kv_heads, w.head_dim, self.max_ctx, pt, device=device)
        self.opts = pa.decode_opts(k_scale=self.k_scale, v_scale=self.v_scale, max_context_len=self.max_ctx,
                                   partition_tokens=pt, workspace=self.ws, kernel=kernel)
        eff_pt = pt if pt else pa.pa_decode_partition_tokens(B, w.num_kv_heads, self.max_ctx)
        if self.ws is None:
            eff_pt = 0
        self.split = eff_pt > 0 and -(-self.max_ctx // eff_pt) > 1
        self.partition_tokens_used = eff_pt if self.split else 0
        self.fused_step = True
        self.cascade_step = False
        self.prefix_kernel = -1
        self.launches_per_step = 2 + (1 if self.split else 0)
        torch.cuda.synchronize(device)

    def k1(self, stream=None):
        self.pa.pa_reshape_and_cache(self.new_k, self.new_v, self.new_slots, self.k_cache, self.v_cache,
                                     self.k_scale, self.v_scale, stream=stream)

    def decode(self, stream=None):
        w = self.w
        self.pa.pa_decode(self.out, self.q, self.k_cache, self.v_cache, self.bt, self.lens, w.scale, w.num_kv_heads,
                          opts=self.opts, stream=stream)

    def cascade(self, stream=None):
        w = self.w
        if not hasattr(self, "_casc_opts"):
            n = self.pa.pa_decode_cascade_workspace_bytes(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                                          self.max_ctx, w.shared_prefix_tokens, 0)
            self._casc_ws = torch.empty(n, dtype=torch.uint8, device=self.device)
            self._casc_opts = self.pa.decode_opts(max_context_len=self.max_ctx, workspace=self._casc_ws,
                                                  kernel=self.kernel, prefix_kernel=self.prefix_kernel)
        self.pa.pa_decode_cascade(self.out, self.q, self.new_k, self.new_v, self.new_slots, self.k_cache,
                                  self.v_cache, self.bt, self.lens, w.shared_prefix_tokens, w.scale, w.num_kv_heads,
                                  opts=self._casc_opts, stream=stream)

    def fused(self, stream=None):
        w = self.w
        self.pa.pa_decode_step(self.out, self.q, self.new_k, self.new_v, self.new_slots, self.k_cache, self.v_cache,
                               self.bt, self.lens, w.scale, w.num_kv_heads, opts=self.opts, stream=stream)

    def step(self):
        if self.cascade_step:
            self.cascade()
        elif self.fused_step:
            self.fused()
        else:
            self.k1()
            self.decode()


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (no MEASURED_PEAKS.json)"


# The sources of the decode kernels whose DRAM traffic profiles/decode_traffic.json records.
DECODE_SOURCES = ("decode.cu", "decode_math.cuh", "decode_units.cu", "pa_device.cuh", "internal.h")


def decode_source_hash() -> str:
    """Hash of the decode kernel's sources with comments, blank lines and line-edge whitespace removed:
    the recorded DRAM traffic stays valid across comment edits and is dropped by any code change."""
    h = hashlib.sha256()
    for f in DECODE_SOURCES:
        with open(os.path.join(ROOT, "paged_kv_cache_385_b200", "csrc", f), encoding="utf-8") as fh:
            text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        lines = [re.sub(r"//.*$", "", ln).strip() for ln in text.splitlines()]
        h.update("\n".join(ln for ln in lines if ln).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """Per-launch DRAM bytes of the decode kernel from the committed ncu summary, if it matches this source."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[workload]
        if e.get("source_hash") != decode_source_hash():
            return None
        return int(e["dram_bytes_per_launch"])
    except Exception:
        return None


def cpu_baseline_sample(w: W.Workload, budget_s: float = 15.0, min_s: float = 10.0):
    """Time the float64 oracle (as it stands) on whole sequences of the workload: at least min_s of
    oracle time (passing over the batch again when it finishes sooner), and no new sequence after
    budget_s once every sequence has run once."""
    import numpy as np
    from oracle import attention
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    lens = W.context_lens(w)
    rng = np.random.default_rng(w.seed)
    D, Hkv, Hq = w.head_dim, w.num_kv_heads, w.num_q_heads
    esz = w.kv_elem_bytes
    done_bytes, t_total, nseq, done_tokens = 0, 0.0, 0, 0
    kept, kept_bytes = [], 0  # the first pass's inputs (up to 256 MB of pools) for the repeat passes

    def timed(args):
        nonlocal done_bytes, t_total, nseq, done_tokens
        q, kp, vp, bt, n = args
        t0 = time.perf_counter()
        attention.decode_paged(q, kp, vp, bt, [n], w.scale, Hkv, w.kv_dtype, 0.0123, 0.0123)
        t_total += time.perf_counter() - t0
        done_bytes += n * Hkv * D * esz * 2
        done_tokens += n
        nseq += 1

    while nseq == 0 or (t_total < budget_s and nseq < w.num_seqs):
        n = int(lens[nseq])
        nb = -(-n // 16)
        if w.kv_dtype == "e4m3":
            kp = rng.integers(0, 0x7E, (nb, Hkv, 16, D), dtype=np.uint8)
            vp = rng.integers(0, 0x7E, (nb, Hkv, 16, D), dtype=np.uint8)
        else:
            tdt = TORCH_KV[w.kv_dtype]
            kp = torch.randn(nb, Hkv, 16, D).to(tdt).view(torch.int16).numpy().view(np.uint8)
            vp = torch.randn(nb, Hkv, 16, D).to(tdt).view(torch.int16).numpy().view(np.uint8)
        bt = rng.permutation(nb).astype(np.int32)[None, :]
        q = rng.standard_normal((1, Hq, D))
        if kept_bytes + 2 * kp.nbytes <= (256 << 20):
            kept.append((q, kp, vp, bt, n))
            kept_bytes += 2 * kp.nbytes
        timed((q, kp, vp, bt, n))
    while t_total < min_s and kept:  # repeat passes over the kept sequences until min_s of oracle time
        for args in kept:
            timed(args)
    what = (f"{nseq} of {w.num_seqs} sequences" if nseq <= w.num_seqs else
            f"{nseq} sequence runs (each of the {w.num_seqs} sequences once, then repeats over the first "
            f"{len(kept)} until {min_s:.0f} s of oracle time)")
    return {"value": done_bytes / t_total / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{what} (all {Hq} query heads, {done_tokens} tokens), "
                      f"float64 numpy oracle (gather through the block table + softmax(qK^T)V), "
                      f"{t_total:.1f} s wall"}


def run_ours(args, rank, world, local_rank):
    import paged_kv_cache_385_b200 as pa
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    w = W.FULL[args.workload]
    st = Setup(w, device, args.kernel, args.partition_tokens)
    st.fused_step = args.step in ("fused", "cascade")
    st.cascade_step = args.step == "cascade"
    if st.cascade_step and not w.shared_prefix_tokens:
        raise SystemExit("--step cascade needs a workload with a shared prefix (prefix_gqa)")
    st.prefix_kernel = args.prefix_kernel
    if st.cascade_step:
        # prefix kernel + suffix decode (+ the partition merge when the suffix itself splits)
        span = max(st.max_ctx - w.shared_prefix_tokens, 1)
        spt = st.pa.pa_decode_partition_tokens(w.num_seqs, w.num_kv_heads, span)
        st.launches_per_step = 2 + (1 if spt > 0 and -(-span // spt) > 1 else 0)
    else:
        st.launches_per_step = (1 if st.fused_step else 2) + (1 if st.split else 0)
    kv_bytes = W.kv_bytes_read(w, st.lens_host)
    K, Wm = args.steps, max(3, args.warmup)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(Wm):
        st.step()
    torch.cuda.synchronize(device)
    pa.pa_read_device_error(clear=True)

    # ---- device-timed steps ------------------------------------------------------------------
    # Only the region is bracketed by events: an event between two launches serialises them (the
    # next launch can no longer overlap the previous one's tail) and adds ~9 us per step. A fused
    # step is one decode launch (plus the partition merge when the context is split), so the
    # per-launch duration of the decode call is the region's time over K. In "separate" mode a
    # second pass of K steps brackets each pa_decode with events to isolate it.
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(local_rank) as clocks:
        start.record()
        for _ in range(K):
            st.step()
        end.record()
        torch.cuda.synchronize(device)
    barrier()
    total_ms = start.elapsed_time(end)
    k1_ms = []
    if st.fused_step:
        dec_ms = [total_ms / K]
    else:
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
        for k in range(K):
            ev[k][0].record()
            st.k1()
            ev[k][1].record()
            st.decode()
            ev[k][2].record()
        torch.cuda.synchronize(device)
        dec_ms = [ev[k][1].elapsed_time(ev[k][2]) for k in range(K)]
        k1_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in range(K)]
    dev_err = pa.pa_read_device_error(clear=True)
    total_ms = max_over_ranks(total_ms, device)
    ms_per_step = total_ms / K

    # ---- end to end through the C ABI with host buffers --------------------------------------
    # The step's inputs (q, new K/V, slots, block tables, context lengths) are packed into one pinned
    # host buffer and copied with one H2D copy into a device buffer the step's tensors view; the
    # output comes back with one D2H copy. The KV pool is the resident cache and is not copied.
    # Inputs and outputs are double-buffered: a copy stream moves step k + 2's inputs in and step k's
    # output out while the kernels of step k + 1 run, so every step's copies are inside the timed
    # region without stalling the kernels. The last output read back is checked bit for bit against
    # the device-timed run's output (same inputs, so the same result).
    e2e = None
    if not args.no_e2e:
        ref_out = st.out.clone()
        parts = [st.q, st.new_k, st.new_v, st.new_slots, st.bt, st.lens]
        offs, total = [], 0
        for t in parts:
            offs.append(total)
            total += -(-(t.numel() * t.element_size()) // 256) * 256
        hbuf = torch.empty(total, dtype=torch.uint8).pin_memory()
        dbufs = [torch.empty(total, dtype=torch.uint8, device=device) for _ in range(2)]
        views = [[], []]
        for t, o in zip(parts, offs):
            n = t.numel() * t.element_size()
            hbuf[o:o + n].view(t.dtype).view(t.shape).copy_(t.cpu())
            for b in range(2):
                views[b].append(dbufs[b][o:o + n].view(t.dtype).view(t.shape))
        outs = [torch.empty_like(st.out) for _ in range(2)]
        houts = [torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory() for _ in range(2)]
        h2d, d2h = total, houts[0].numel() * houts[0].element_size()
        Ke = max(10, min(K, 500))
        comp = torch.cuda.current_stream(device)
        copy = torch.cuda.Stream(device)
        ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer b landed
        ev_done = [torch.cuda.Event() for _ in range(2)]  # kernels that used buffer b finished
        ev_out = [torch.cuda.Event() for _ in range(2)]   # output b read back

        def h2d_into(b):
            with torch.cuda.stream(copy):
                dbufs[b].copy_(hbuf, non_blocking=True)
                ev_in[b].record(copy)

        def run(n_steps, start_ev=None):
            copy.wait_stream(comp)  # start after everything queued so far (and the start event)
            h2d_into(0)
            h2d_into(1)
            for k in range(n_steps):
                b = k & 1
                comp.wait_event(ev_in[b])
                if k >= 2:
                    comp.wait_event(ev_out[b])  # output b of step k - 2 has been read back
                st.q, st.new_k, st.new_v, st.new_slots, st.bt, st.lens = views[b]
                st.out = outs[b]
                st.step()
                ev_done[b].record(comp)
                with torch.cuda.stream(copy):
                    copy.wait_event(ev_done[b])
                    houts[b].copy_(outs[b], non_blocking=True)
                    ev_out[b].record(copy)
                    if k + 2 < n_steps:
                        dbufs[b].copy_(hbuf, non_blocking=True)  # step k + 2's inputs (buffer b is free)
                        ev_in[b].record(copy)
            comp.wait_stream(copy)  # the last read-backs are part of the region

        run(3)
        barrier()
        torch.cuda.synchronize(device)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(comp)
        run(Ke)
        s1.record(comp)
        torch.cuda.synchronize(device)
        barrier()
        e_ms = max_over_ranks(s0.elapsed_time(s1), device)
        same = torch.equal(houts[(Ke - 1) & 1].view(torch.int16), ref_out.cpu().view(torch.int16))
        e2e = {"value": round(job_throughput(kv_bytes, world, e_ms / Ke), 1), "unit": "GB/s",
               "ms_per_step": round(e_ms / Ke, 5), "steps": Ke, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "output_matches_device_run": bool(same),
               "note": "per step: one pinned H2D copy of the packed inputs (q, new K/V, slots, block tables, "
                       "context lens), the decode step through the C ABI, one D2H copy of out; inputs and "
                       "outputs double-buffered so the copies of neighbouring steps overlap the kernels; the "
                       "KV pool is the resident cache"}

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return

    peak, peak_src = measured_hbm_peak()
    dec_avg_s = statistics.mean(dec_ms) / 1e3
    achieved = kv_bytes / dec_avg_s / 1e9
    traffic = ncu_traffic(args.workload)
    value = job_throughput(kv_bytes, world, ms_per_step)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_sample(w)
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": Wm,
        "ms_per_step": round(ms_per_step, 5),
        "us_per_step": round(ms_per_step * 1e3, 2),
        "us_decode": round(dec_avg_s * 1e6, 2),
        "us_reshape_and_cache": round(statistics.mean(k1_ms) * 1e3, 2) if k1_ms else None,
        "step": ("pa_decode_cascade (shared prefix once per KV head + suffix decode + merge; new-token write fused)"
                 if st.cascade_step else "pa_decode_step (new-token write fused into the decode launch)"
                 if st.fused_step else "pa_reshape_and_cache + pa_decode"),
        "pct_of_8TBps": round(100.0 * value / world / 8000.0, 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.kv_dtype,
        "data": "synthetic",
        "config": {"workload": w.name, "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads,
                   "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
                   "context_lens": "fixed 2048" if w.name == "llama7b_mha" else str(w.ctx),
                   "pool_blocks": w.num_blocks, "kv_bytes_per_step": kv_bytes,
                   "partition_tokens": st.partition_tokens_used, "kernel": {0: "cuda-core", 2: "tensor-core, one CTA per partition"}.get(args.kernel, "tensor-core"),
                   **({"prefix_kernel": "warp-level mma" if args.prefix_kernel == 0 else "tcgen05"}
                      if st.cascade_step else {}),
                   "l2": f"inputs larger than L2: {kv_bytes / 1e9:.2f} GB of KV per step vs 126 MB L2, no flush",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": ("pa_decode_cascade (prefix + suffix decode + merge kernels)"
                                                if st.cascade_step else
                                                ("pa_decode_step" if st.fused_step else "pa_decode")
                                                + (" (decode kernel + partition merge)" if st.split else " (decode kernel)")),
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": peak_src,
                     "launch_us": round(dec_avg_s * 1e6, 2),
                     "launch_timing": ("CUDA events around the K-step timed region / K (one decode call per step)"
                                       if st.fused_step else "CUDA events around each pa_decode, second pass of K steps"),
                     "algorithmic_bytes_per_launch": kv_bytes},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": K * st.launches_per_step,
        "clocks": clocks.summary(),
        "device_error_bits": dev_err,
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------
# Reference arm: the float64 CPU oracle, as it stands, on bounded samples of the same workload.
# ---------------------------------------------------------------------------------------------
def run_reference(args, rank, world):
    if rank != 0:
        return
    w = W.FULL[args.workload]
    per_step = []
    cpu = None
    for i in range(max(3, args.warmup) + args.steps):
        r = cpu_baseline_sample(w, budget_s=0.0, min_s=0.0)  # one sequence per step
        if i >= max(3, args.warmup):
            per_step.append(r)
        cpu = r
    value = statistics.mean(r["value"] for r in per_step)
    lens = W.context_lens(w)
    kv_seq = int(lens[0]) * w.num_kv_heads * w.head_dim * w.kv_elem_bytes * 2
    ms = kv_seq / (value * 1e9) * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "num_seqs_per_step": 1, "num_q_heads": w.num_q_heads,
                   "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "parallelism": "host cores, rank 0"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cpu["cores"], "kind": "oracle",
                         "sample": "one sequence per step: " + cpu["sample"]},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_prefill(args, rank, world, local_rank):
    """Chunked-prefill attention: 8 sequences x 2048-token prompts, Llama-3-8B heads (32/8, D=128), bf16."""
    import paged_kv_cache_385_b200 as pa
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    B, n, Hq, Hkv, D = 8, 2048, 32, 8, 128
    nb = B * n // 16 + 64
    g = torch.Generator(device=device)
    g.manual_seed(77)
    alloc = pa.BlockAllocator(nb, torch.randperm(nb, generator=torch.Generator().manual_seed(77)).tolist())
    bt = pa.build_block_tables(alloc, [n] * B, n // 16)
    kc = torch.randn(nb, Hkv, 16, D, generator=g, device=device).to(torch.bfloat16)
    vc = torch.randn(nb, Hkv, 16, D, generator=g, device=device).to(torch.bfloat16)
    q = torch.randn(B * n, Hq, D, generator=g, device=device).to(torch.bfloat16)
    out = torch.empty_like(q)
    qs = torch.arange(0, B * n + 1, n, dtype=torch.int32, device=device)
    lens = torch.full((B,), n, dtype=torch.int32, device=device)
    btd = bt.to(device)
    # Causal FLOPs: QK^T and PV, 2 flops per MAC, position i sees i + 1 keys.
    flops = B * Hq * 2 * 2 * D * (n * (n + 1) // 2)
    K, Wm = max(20, args.steps // 100), max(3, args.warmup)

    kernel = 1 if args.kernel == -1 else args.kernel  # -1: the library's choice (tcgen05 here)

    def call():
        pa.pa_prefill(out, q, kc, vc, btd, qs, lens, n, D ** -0.5, Hkv, kernel=kernel)

    for _ in range(Wm):
        call()
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        a.record()
        for _ in range(K):
            call()
        b.record()
        torch.cuda.synchronize(device)
    ms = a.elapsed_time(b) / K
    tflops = flops / (ms / 1e3) / 1e12
    peak_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(peak_path) as f:
            peak, src = float(json.load(f)["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, cuBLAS burst)"
    except Exception:
        peak, src = 1590.0, "fallback"
    if rank == 0:
        print(json.dumps({
            "metric": "chunked prefill attention over paged KV: TFLOP/s (causal, QK^T + PV)", "value": round(tflops, 1),
            "unit": "TFLOP/s", "n_gpus": 1, "steps": K, "warmup": Wm, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"num_seqs": B, "prompt_tokens": n, "num_q_heads": Hq, "num_kv_heads": Hkv, "head_dim": D,
                       "flops_per_call": flops},
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(tflops / peak, 4), "traffic": None, "peak_source": src,
                         "kernel": "tcgen05 (tensor memory accumulators)" if kernel == 1 else "warp-level mma.sync"},
            "gpu_launches": K, "clocks": clocks.summary()}), flush=True)


def run_copy_blocks(args, rank, world, local_rank):
    """Throughput of pa_copy_blocks on the workload's pool: 1024 distinct (src, dst) block pairs per call."""
    import paged_kv_cache_385_b200 as pa
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    w = W.FULL[args.workload]
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    kc = torch.zeros(shape, dtype=TORCH_KV[w.kv_dtype], device=device)
    vc = torch.zeros_like(kc)
    n = min(1024, w.num_blocks // 2)
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(w.seed))
    mapping = torch.stack([perm[:n], perm[n:2 * n]], dim=1).to(torch.int64).to(device)
    block_bytes = w.num_kv_heads * w.block_size * w.head_dim * w.kv_elem_bytes
    moved = n * block_bytes * 2 * 2  # K and V, read + write
    K, Wm = args.steps, max(3, args.warmup)
    for _ in range(Wm):
        pa.pa_copy_blocks(kc, vc, mapping)
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        a.record()
        for _ in range(K):
            pa.pa_copy_blocks(kc, vc, mapping)
        b.record()
        torch.cuda.synchronize(device)
    ms = a.elapsed_time(b) / K
    peak, peak_src = measured_hbm_peak()
    gbs = moved / (ms / 1e3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": "pa_copy_blocks (copy-on-write block copies): HBM GB/s read+write", "value": round(gbs, 1),
            "unit": "GB/s", "n_gpus": 1, "steps": K, "warmup": Wm, "ms_per_step": round(ms, 5),
            "higher_is_better": True, "dtype": w.kv_dtype, "data": "synthetic",
            "config": {"workload": w.name, "pairs_per_call": n, "block_bytes_per_cache": block_bytes,
                       "bytes_moved_per_call": moved},
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(gbs / peak, 4), "traffic": None, "peak_source": peak_src},
            "gpu_launches": K, "clocks": clocks.summary()}), flush=True)


def kv_utilization_sim(num_blocks: int = 65536, slots: int = 256, num_requests: int = 4000, seed: int = 7,
                       reserve_tokens: int = 2048, sample_every: int = 16):
    """Continuous batching over a synthetic request stream with the library's allocator.

    Up to `slots` sequences run at once; each step every running sequence appends one token (a new
    block when it crosses a 16-token boundary); finished sequences free their blocks and the next
    request takes the slot (its prompt blocks allocated at once). Every `sample_every` steps the
    live token counts and the allocator's blocks in use are recorded. Returns the samples as
    (live token counts, blocks in use) pairs.
    """
    import paged_kv_cache_385_b200 as pa
    prompts, outs = W.request_stream(seed, num_requests, reserve_tokens)
    alloc = pa.BlockAllocator(num_blocks)
    nxt = 0
    running = []  # [tokens, remaining, blocks]
    samples = []
    step = 0
    while nxt < num_requests or running:
        while len(running) < slots and nxt < num_requests:
            n = prompts[nxt]
            blocks = alloc.alloc_n(-(-n // 16)).tolist()
            running.append([n, outs[nxt], blocks])
            nxt += 1
        for r in running:
            if r[0] % 16 == 0:
                r[2].append(alloc.alloc())
            r[0] += 1
            r[1] -= 1
        done = [r for r in running if r[1] <= 0]
        for r in done:
            alloc.free_n(torch.tensor(r[2], dtype=torch.int32))
        running = [r for r in running if r[1] > 0]
        if step % sample_every == 0 and running:
            samples.append(([r[0] for r in running], num_blocks - alloc.num_free))
        step += 1
    return samples


def run_kv_utilization(args, rank):
    if rank != 0:
        return
    t0 = time.perf_counter()
    samples = kv_utilization_sim()
    wall = time.perf_counter() - t0
    tokens = sum(sum(n) for n, _ in samples)
    held = sum(b * 16 for _, b in samples)
    reserved = sum(len(n) * 2048 for n, _ in samples)
    print(json.dumps({
        "metric": "KV memory utilisation: tokens stored / KV slots held (paged, blocks of 16 on demand)",
        "value": round(100.0 * tokens / held, 2), "unit": "%", "higher_is_better": True, "data": "synthetic",
        "contiguous_reservation_pct": round(100.0 * tokens / reserved, 2),
        "config": {"requests": 4000, "concurrent_slots": 256, "prompt": "U[16,1024]", "output": "exp(mean 256)",
                   "reserve_tokens_contiguous": 2048, "samples": len(samples)},
        "wall_s": round(wall, 2)}), flush=True)


def main():
    args = parse()
    rank, world, local_rank = dist_env()
    if args.gpus != world and rank == 0:
        # Ranks come from the launcher (torch.distributed.run); the line reports the ranks that ran.
        print(f"bench.py: --gpus {args.gpus} but {world} rank(s) launched; measuring {world} "
              f"(launch N ranks with python -m torch.distributed.run --nproc-per-node N)", file=sys.stderr)
    if args.op == "kv_utilization":
        run_kv_utilization(args, rank)
        return 0
    if args.op == "copy_blocks":
        run_copy_blocks(args, rank, world, local_rank)
        return 0
    if args.op == "prefill":
        run_prefill(args, rank, world, local_rank)
        return 0
    if args.impl == "reference":
        run_reference(args, rank, world)
        return 0
    run_ours(args, rank, world, local_rank)
    return 0


if __name__ == "__main__":
    sys.exit(main())
