"""CPU checks of bench.py's bookkeeping: the decode-source hash that keys the recorded DRAM traffic
ignores comments and blank lines but not code, and the recorded traffic is used only on a match."""
import json
import os
import shutil

import bench

SRC = bench.DECODE_SOURCES


def _tree(tmp_path, edit=None):
    root = tmp_path / "repo"
    csrc = root / "paged_kv_cache_385_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in SRC:
        shutil.copy(os.path.join(bench.ROOT, "paged_kv_cache_385_b200", "csrc", f), csrc / f)
    if edit:
        p = csrc / "decode.cu"
        p.write_text(edit(p.read_text()))
    return str(root)


def test_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path / "a"))
    h0 = bench.decode_source_hash()
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path / "b", lambda t: "// a new comment\n\n" + t.replace(
        "namespace pa {", "/* block\n comment */ namespace pa {  // trailing", 1)))
    assert bench.decode_source_hash() == h0
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path / "c", lambda t: t.replace("kLog2e", "kLog2E")))
    assert bench.decode_source_hash() != h0


def test_recorded_traffic_needs_a_matching_hash(tmp_path, monkeypatch):
    root = _tree(tmp_path)
    (tmp_path / "repo" / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", root)
    rec = {"w": {"source_hash": bench.decode_source_hash(), "dram_bytes_per_launch": 123}}
    (tmp_path / "repo" / "profiles" / "decode_traffic.json").write_text(json.dumps(rec))
    assert bench.ncu_traffic("w") == 123
    rec["w"]["source_hash"] = "0" * 16
    (tmp_path / "repo" / "profiles" / "decode_traffic.json").write_text(json.dumps(rec))
    assert bench.ncu_traffic("w") is None
    assert bench.ncu_traffic("missing") is None


class _FakeNvml:
    """Stands in for pynvml: two GPUs, the visible one is the second of the machine."""
    NVML_CLOCK_SM = 0

    def __init__(self):
        self.calls = []

    def nvmlDeviceGetHandleByUUID(self, uuid):
        self.calls.append(("uuid", uuid))
        return {"GPU-bbbb": "gpu1"}[uuid]

    def nvmlDeviceGetHandleByIndex(self, i):
        self.calls.append(("index", i))
        return ["gpu0", "gpu1"][i]


def test_clock_sampler_reads_the_timed_gpu_by_uuid(monkeypatch):
    """cuda:0 is the machine's second GPU when CUDA_VISIBLE_DEVICES hides the first: NVML index 0
    would sample the wrong GPU, its UUID does not."""
    import types
    nv = _FakeNvml()
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", lambda i: types.SimpleNamespace(uuid="bbbb"))
    assert bench.ClockSampler.nvml_handle(nv, 0) == ("gpu1", "uuid")

    def no_props(i):
        raise RuntimeError("no CUDA")
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", no_props)
    assert bench.ClockSampler.nvml_handle(nv, 0) == ("gpu0", "index")
