"""Step time of the decode step launched eagerly, with CUDA events around every step, and from a
CUDA graph; and the host time to submit one step through the Python binding.

Why: the bench brackets only its whole timed region with events. An event between two launches
serialises them (the next launch can no longer overlap the previous one's tail), and a CUDA graph
is the usual cure for launch-bound loops; this measures both on the bench's own workloads.

    python paged_kv_cache_385_b200/measure/launch_overheads.py [events | graphs]

events: llama7b_mha and llama3_8b_gqa, fused (pa_decode_step) and separate (pa_reshape_and_cache +
        pa_decode) steps: no events, an event pair around every step (and the mean inside the
        pairs), and a graph of 50 steps replayed.
graphs: prefix_gqa (cascade), llama7b_mha and llama3_8b_gqa (fused): host submit time per call,
        eager device time per step, a graph of one step and a graph of ten steps replayed.
One GPU; 1000 or 2000 timed steps after 20 warm-up steps.
"""
import os
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import paged_kv_cache_385_b200 as pa  # noqa: E402
import workloads as W  # noqa: E402


def _ms(a, b):
    return a.elapsed_time(b)


def _timed(fn, n):
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(n):
        fn()
    b.record()
    torch.cuda.synchronize()
    return _ms(a, b)


def _graph(fn, steps):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(3):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(steps):
            fn()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    return g


def events(dev):
    K = 1000
    for name in ("llama7b_mha", "llama3_8b_gqa"):
        st = bench.Setup(W.FULL[name], dev, -1, None)
        for mode in ("fused", "separate"):
            fn = st.fused if mode == "fused" else (lambda: (st.k1(), st.decode()))
            for _ in range(20):
                fn()
            torch.cuda.synchronize()
            no_ev = _timed(fn, K) / K * 1e3
            pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]

            def with_events():
                for x, y in pairs:
                    x.record()
                    fn()
                    y.record()
            with_ev = _timed(with_events, 1) / K * 1e3
            inner = statistics.mean(_ms(x, y) for x, y in pairs) * 1e3
            g = _graph(fn, 50)
            graph_us = _timed(g.replay, K // 50) / K * 1e3
            print(f"{name} {mode}: no events {no_ev:.2f} us/step, with events {with_ev:.2f} (inner {inner:.2f}), "
                  f"graph {graph_us:.2f}", flush=True)
        del st
        torch.cuda.empty_cache()


def graphs(dev):
    K = 2000
    for name, step in (("prefix_gqa", "cascade"), ("llama7b_mha", "fused"), ("llama3_8b_gqa", "fused")):
        st = bench.Setup(W.FULL[name], dev, -1, None)
        st.cascade_step = step == "cascade"
        for _ in range(20):
            st.step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        a.record()
        for _ in range(K):
            st.step()
        b.record()
        host_us = (time.perf_counter() - t0) / K * 1e6
        torch.cuda.synchronize()
        dev_us = _ms(a, b) / K * 1e3
        g1 = _graph(st.step, 1)
        graph1_us = _timed(g1.replay, K) / K * 1e3
        g10 = _graph(st.step, 10)
        graph10_us = _timed(g10.replay, K // 10) / (K // 10 * 10) * 1e3
        err = pa.pa_read_device_error(clear=True)
        print(f"{name} {step}: host submit {host_us:.1f} us/call, eager device {dev_us:.2f} us/step, "
              f"graph(1) {graph1_us:.2f}, graph(10) {graph10_us:.2f}, err {err}", flush=True)
        del st, g1, g10
        torch.cuda.empty_cache()


if __name__ == "__main__":
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    which = sys.argv[1] if len(sys.argv) > 1 else "events"
    {"events": events, "graphs": graphs}[which](dev)
