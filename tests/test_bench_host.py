"""bench.py's host-side accounting (no GPU): the algorithmic bytes and flops
the roofline divides by, the kernel family each workload runs, the keying of
recorded DRAM traffic to the kernel sources, and the CPU-baseline record."""
import json
import os

import pytest

import bench
from gated_delta_rule_147_b200.inputs import WORKLOADS


@pytest.mark.parametrize("name,mb,gf", [
    ("gdn", 273.7, 47.96),    # 1028 B per token-head + S_T; 182,955 flop per token-head
    ("kda", 680.5, 95.92),    # + channel alpha, random S0 read
    ("gdn2", 940.6, 147.46),  # + channel b, w; 281,259 flop per token-head
])
def test_algorithmic_work(name, mb, gf):
    wl = WORKLOADS[name]
    assert bench.workload_bytes(wl) / 1e6 == pytest.approx(mb, abs=0.05)
    assert bench.workload_flops(wl) / 1e9 == pytest.approx(gf, abs=0.005)


def test_kernel_families():
    fam = {n: bench.kernel_family(w) for n, w in WORKLOADS.items()}
    assert fam == {"tiny": "general", "gdn": "twopass", "kda": "twopass_general",
                   "gdn2": "twopass_general", "gla": "erasefree", "gdn_gqa": "twopass",
                   "gdn256": "twopass256"}
    assert set(bench.LAUNCHES_PER_CALL) == set(bench.KERNEL_SOURCES) == set(bench.KERNEL_NAMES)


def test_recorded_traffic_is_keyed_to_the_kernel_sources(monkeypatch, tmp_path):
    rec = {"workloads": {"gla": {"source_sha256": bench.kernel_source_hash("erasefree"),
                                 "dram_bytes_per_launch": 123}}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "chunk_fwd_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the recorded figure needs the sources it was taken on: here they are absent
    with pytest.raises(OSError):
        bench.kernel_source_hash("erasefree")
    monkeypatch.setattr(bench, "kernel_source_hash", lambda fam: rec["workloads"]["gla"]["source_sha256"])
    assert bench.measured_traffic("gla") == 123
    monkeypatch.setattr(bench, "kernel_source_hash", lambda fam: "0" * 64)
    assert bench.measured_traffic("gla") is None
    assert bench.measured_traffic("kda") is None


def test_backward_flop_counts():
    # state-gradient pass per token-head: 3 C d_k + C^2 (first pass), C d_v + 3 d_k d_v
    # (state pass) multiply-adds, the solve C^2 / 3 flop
    assert bench.BWD_GRAD_FLOPS_PER_TOKEN_HEAD == 174763
    # chunk kernel: one 128x256x128, one 128x64x128 and three 128x128x128 products
    assert bench.BWD_TC_FLOPS_PER_CHUNK == 2 * (128 * 256 * 128 + 128 * 64 * 128 + 3 * 128 ** 3)


def test_cpu_baseline_record():
    wl = WORKLOADS["gdn"].with_(B=1, H=2, T=64)
    rec = bench.cpu_baseline(wl, budget_s=0.2)
    assert rec["kind"] == "oracle" and rec["unit"] == "tokens/s"
    assert rec["value"] > 0 and rec["cores"] >= 1
    assert rec["single_core"]["value"] > 0
    assert "heads" in rec["sample"]


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one
    JSON line with the contract's keys and the reference marker."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                         timeout=300, check=True, cwd=root)
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_tied_flops_follow_the_head_dims():
    """The tied (Gated DeltaNet) count at d = 128 is 182,955 flops per
    token-head; at d = 256 each d_k d_v term grows 4x, each C d term 2x."""
    per = lambda wl: bench.workload_flops(wl) / (wl.B * wl.T * wl.H)
    assert per(WORKLOADS["gdn"]) == 182955
    C = 64
    assert per(WORKLOADS["gdn256"]) == round(2 * (3 * 256 * 256 + C * 5 * 256 + C * C / 3))
