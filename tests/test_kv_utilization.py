"""KV-memory utilisation measured with the library's allocator, pinned to the closed form (CPU only).

The pages report that earlier systems used 20-40% of KV memory for real tokens while paged,
on-demand 16-token blocks reach >90% ("vLLM 前世今生" §1, §3.1-3.2). The measurement runs
continuous batching over a synthetic request stream through pa_allocator; at every sample the
blocks the allocator has handed out must equal sum ceil(n / 16) over the live sequences (no leaks,
no over-allocation), so the measured utilisation is exactly the oracle's closed form.
"""
import bench
from oracle import paging


def test_blocks_in_use_match_closed_form_at_every_sample():
    samples = bench.kv_utilization_sim(num_blocks=8192, slots=48, num_requests=300, seed=3, sample_every=4)
    assert len(samples) > 50
    for counts, blocks in samples:
        assert blocks == sum(-(-n // 16) for n in counts)
        paged, contiguous = paging.utilization(counts, 16, 2048)
        assert abs(paged - sum(counts) / (16 * blocks)) < 1e-12
        # Internal waste is below one block per sequence.
        assert 16 * blocks - sum(counts) < 16 * len(counts)
        assert contiguous < paged


def test_closed_form_examples():
    assert paging.utilization([16, 32], 16, 64) == (1.0, 48 / 128)
    paged, _ = paging.utilization([1], 16, 16)
    assert paged == 1 / 16
    paged, contiguous = paging.utilization([17, 100], 16, 2048)
    assert paged == 117 / (32 + 112)
    assert contiguous == 117 / 4096
