"""Host-side logic of bench.py (no GPU): how many input sets rotate, and when
the committed DRAM-traffic record may be reported."""

import json
import os

import bench
from tiled_attention_13_b200.inputs import WORKLOADS


def test_input_sets_exceed_twice_l2():
    for name, wl in WORKLOADS.items():
        n = bench.n_input_sets(wl)
        assert n >= 2, name
        assert n * wl.bytes_min >= 2 * bench.L2_BYTES, name
        # no more sets than needed
        assert n == 2 or (n - 1) * wl.bytes_min < 2 * bench.L2_BYTES, name


def test_config_names_the_rotation():
    cfg = bench._config(WORKLOADS["cross"], 1)
    assert "16 input sets" in cfg["l2"] and cfg["workload"] == "cross"


def test_traffic_record_follows_kernel_source():
    """The committed record is used only while the kernel source hash matches
    (else the bench reports null), and only for its own workload."""
    import hashlib

    path = os.path.join(bench.ROOT, "profiles", "fa_fwd_tc_llama13b_8k.json")
    rec = json.load(open(path))
    csrc = os.path.join(bench.ROOT, "tiled_attention_13_b200", "csrc")
    sha = hashlib.sha256(b"".join(open(os.path.join(csrc, f), "rb").read()
                                  for f in ("fa_fwd_tc.cuh", "ptx.cuh"))).hexdigest()
    t = bench.captured_traffic("llama13b-8k")
    if sha == rec["kernel_source_sha256"]:
        assert t == float(rec["dram_bytes_per_launch"])
    else:
        assert t is None
    assert 0.5 < rec["dram_bytes_per_launch"] / rec["algorithmic_bytes_per_launch"] < 2
    assert bench.captured_traffic("b4-8k-causal") is None  # no record for that workload


def test_every_traffic_record_is_keyed_by_its_sources():
    """Each committed record names its workload, the kernel's source files
    (each of which exists) and a hash; the bench reports its traffic only
    while those files hash to the recorded value."""
    import glob
    import hashlib

    csrc = os.path.join(bench.ROOT, "tiled_attention_13_b200", "csrc")
    recs = sorted(glob.glob(os.path.join(bench.ROOT, "profiles", "*.json")))
    assert len(recs) >= 7
    for path in recs:
        rec = json.load(open(path))
        assert rec["workload"] in WORKLOADS, path
        files = rec.get("source_files", ["fa_fwd_tc.cuh", "ptx.cuh"])
        assert all(os.path.exists(os.path.join(csrc, f)) for f in files), path
        sha = hashlib.sha256(b"".join(open(os.path.join(csrc, f), "rb").read() for f in files)).hexdigest()
        t = bench.captured_traffic(rec["workload"])
        if sha == rec["kernel_source_sha256"]:
            assert t == float(rec["dram_bytes_per_launch"]), path
        assert rec["dram_bytes_per_launch"] > 0


def test_traffic_record_rejected_when_source_changes(tmp_path, monkeypatch):
    root = tmp_path
    (root / "profiles").mkdir()
    csrc = root / "tiled_attention_13_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "fa_fwd_tc.cuh").write_text("kernel v2\n")
    (csrc / "ptx.cuh").write_text("helpers\n")
    rec = {"workload": "llama13b-8k", "kernel_source_sha256": "0" * 64, "dram_bytes_per_launch": 1.0}
    (root / "profiles" / "fa_fwd_tc_llama13b_8k.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.captured_traffic("llama13b-8k") is None


def test_roofline_bound_follows_arithmetic_intensity():
    """Self-attention is tensor-bound at every configured length (intensity
    about N/2 FLOP per byte against a ridge near 257); the 77-key
    cross-attention (74 FLOP/B) and a decoding step (1 FLOP/B) are HBM-bound."""
    peaks = {"bf16_tflops": 1686.0, "hbm_gbs": 6549.1}
    for name, wl in WORKLOADS.items():
        want = "hbm" if name in ("cross", "llama13b-decode-8k", "llama13b-decode-8k-paged16") or wl.dtype == "fp32" \
            else "tensor"
        assert bench.roofline_bound(wl, peaks) == want, name


def test_step_percentiles():
    """Nearest-rank p10 / median / p90 of the per-step kernel times."""
    ms = [float(x) for x in range(1, 12)]  # 1 .. 11
    assert bench.step_percentiles(ms) == {"p10": 2.0, "median": 6.0, "p90": 10.0}
    assert bench.step_percentiles([3.5]) == {"p10": 3.5, "median": 3.5, "p90": 3.5}


def test_traffic_record_names_its_kernel_sources(tmp_path, monkeypatch):
    """A record lists the source files of the kernel it captured; it is used
    while their hash matches, whatever the file name of the record."""
    import hashlib

    root = tmp_path
    (root / "profiles").mkdir()
    csrc = root / "tiled_attention_13_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "fa_fwd_short.cuh").write_text("short kernel\n")
    (csrc / "ptx.cuh").write_text("helpers\n")
    sha = hashlib.sha256(b"short kernel\nhelpers\n").hexdigest()
    rec = {"workload": "cross", "source_files": ["fa_fwd_short.cuh", "ptx.cuh"], "kernel_source_sha256": sha,
           "dram_bytes_per_launch": 17.0e6}
    (root / "profiles" / "fa_fwd_short_cross.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.captured_traffic("cross") == 17.0e6
    (csrc / "ptx.cuh").write_text("helpers v2\n")
    assert bench.captured_traffic("cross") is None
