"""Host-side pieces of bench.py that decide what a measurement means: which
workloads get an L2 flush, the config the JSON line reports, and when an ncu
traffic figure still belongs to the kernel source it was taken from."""

import os

import pytest
import torch

import bench
from paged_kv_cache_382_b200 import workloads as W


@pytest.fixture(scope="module")
def steps():
    """The decode suite's batches (lengths, tables, sharing) without their
    K/V data: the pools are left as empty meta tensors, which none of the
    functions under test reads."""
    mp = pytest.MonkeyPatch()
    mp.setattr(W, "_generator", lambda device, seed: None)
    mp.setattr(W, "_normal", lambda shape, dtype, device, gen: torch.empty(shape, dtype=dtype, device="meta"))
    try:
        out = {}
        for name in bench.DECODE_SUITE:
            P = bench.CONFIGS[name].get("partition_size", 512)
            out[name] = bench.build_step(name, 0, "cpu", P)
    finally:
        mp.undo()
    return out


def test_only_workloads_that_fit_l2_are_flushed(steps):
    """A workload whose unique bytes per step fit the 126 MB L2 is flushed before
    every timed step; the others are larger than L2 and run back to back."""
    flushed = {n for n, s in steps.items() if bench.needs_flush(s)}
    assert flushed == {"shared_prefix_cow"}
    for n, s in steps.items():
        alg = W.algorithmic_bytes(s, unique=True)
        assert (alg < bench.L2_BYTES) == (n in flushed), n


def test_config_names_the_workload_and_its_l2_policy(steps):
    """`config` (one function builds it for the GPU arm and the reference arm)
    names the workload by its description and sizes and says which L2 policy
    its timing used."""
    for n, s in steps.items():
        P = bench.CONFIGS[n].get("partition_size", 512)
        a = bench.config_dict(n, s, 1, P, bench.needs_flush(s))
        assert set(a) == {"workload", "name", "num_seqs_per_gpu", "context_tokens_per_gpu", "partition_size",
                          "parallelism", "l2"}
        assert a["workload"] == bench.CONFIGS[n]["desc"] and a["name"] == n
        assert a["num_seqs_per_gpu"] == s.num_seqs and a["context_tokens_per_gpu"] == int(s.context_lens.sum())
        assert ("flushed" in a["l2"]) == bench.needs_flush(s)


def test_profiled_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    """The ncu traffic figure is reported only while the kernel sources hash to
    the value recorded beside it; any change to them makes it null."""
    src = tmp_path / "kernel.cu"
    src.write_text("// one kernel\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "attend", ["kernel.cu"])
    h = bench.kernel_source_hash("attend")
    (prof / "attend_gqa.ncu.md").write_text(f"# x\n\n- dram_bytes_per_launch: 1234\n- kernel_source_sha256: {h}\n")
    assert bench.profiled_traffic("gqa") == 1234
    assert bench.profiled_traffic("llama7b") is None           # no summary for this workload
    src.write_text("// one kernel, changed\n")
    assert bench.profiled_traffic("gqa") is None               # the source moved on


def test_committed_profiles_name_their_workloads():
    """Every committed attend summary belongs to a suite workload and carries
    the two fields the bench reads."""
    root = os.path.join(os.path.dirname(bench.__file__), "profiles")
    names = [f for f in os.listdir(root) if f.startswith("attend_") and f.endswith(".ncu.md")]
    assert names
    for f in names:
        config = f[len("attend_"):-len(".ncu.md")]
        assert config in bench.DECODE_SUITE, f
        text = open(os.path.join(root, f)).read()
        assert "- dram_bytes_per_launch:" in text and "- kernel_source_sha256:" in text, f
