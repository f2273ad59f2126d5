"""Host-side logic of bench.py (CPU only): the kernel-launch count each
workload's step claims, the DRAM-traffic record keyed to the source of the
kernel it was captured on, and the source hash that ignores comments."""
import importlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def load_bench(monkeypatch, **env):
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    import bench
    return importlib.reload(bench)


def test_launch_counts_per_workload(monkeypatch):
    monkeypatch.delenv("MOE_FUSE_ALIGN", raising=False)
    monkeypatch.delenv("MOE_FUSED_FFN", raising=False)
    b = load_bench(monkeypatch)
    from mixture_experts_layer_counts_b200.inputs import WORKLOADS
    got = {n: b.launches_per_step(w, w["T"]) for n, w in WORKLOADS.items()}
    # logits, top-k, align, gather, GEMMs, combine
    assert got["tiny"] == got["decode"] == got["decode-zipf"] == 6        # one fused FFN launch
    assert got["decode-fp8"] == 7                                          # w13 and w2 (swap-AB only)
    assert got["prefill-zipf"] == 10                                       # two align grids, 2 x 2 GEMMs


def test_launch_counts_follow_the_switches(monkeypatch):
    b = load_bench(monkeypatch, MOE_FUSE_ALIGN="1", MOE_FUSED_FFN="0")
    from mixture_experts_layer_counts_b200.inputs import WORKLOADS
    w = WORKLOADS["decode"]
    assert b.launches_per_step(w, w["T"]) == 6        # align folded (-1), two GEMM launches (+1)
    w = WORKLOADS["prefill-zipf"]
    assert b.launches_per_step(w, w["T"]) == 10       # T*k >= 8192: the align is never folded


def test_traffic_record_is_keyed_to_its_kernel_source(monkeypatch):
    """An entry is reported while its kernel's source hash matches, else
    None (a changed kernel needs new counters); no entry gives None."""
    import json
    b = load_bench(monkeypatch)
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    assert {"decode-fp8", "decode", "prefill-zipf"} <= set(rec)
    for name, e in rec.items():
        src = os.path.join(ROOT, "mixture_experts_layer_counts_b200", "csrc", e["code_file"])
        assert os.path.exists(src), e["code_file"]
        want = e["dram_bytes_per_launch"] if b.code_sha(src) == e["code_sha"] else None
        assert b.kernel_traffic(name) == want, name
        assert 0.9 < e["dram_bytes_per_launch"] / e["algorithmic_bytes_per_launch"] < 1.5, name
    assert b.kernel_traffic("tiny") is None


def test_source_hash_ignores_comments(tmp_path, monkeypatch):
    b = load_bench(monkeypatch)
    a = tmp_path / "a.cu"
    c = tmp_path / "c.cu"
    d = tmp_path / "d.cu"
    a.write_text("int f() {\n  return 1;  // one\n}\n")
    c.write_text("// header\nint f() {\n\n  return 1;  // another comment\n}\n")
    d.write_text("int f() {\n  return 2;\n}\n")
    assert b.code_sha(str(a)) == b.code_sha(str(c))
    assert b.code_sha(str(a)) != b.code_sha(str(d))
