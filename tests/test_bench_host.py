"""The bench's host-side pieces on the CPU: the clock sampler against a
stand-in nvidia-smi, the peak and traffic records it reads.

The stand-in accepts only the ids it is told to (as nvidia-smi refuses an id it
does not know), answers the one-shot id query, and in loop mode prints sample
lines in the format of the sampler's query until it is terminated.
"""
import json
import os
import stat
import sys
import time

import pytest

import bench

FAKE = """#!{python}
import sys, time
args = sys.argv[1:]
gid = next(a.split("=", 1)[1] for a in args if a.startswith("--id="))
if gid not in {accepted!r}:
    print("No devices were found", file=sys.stderr)
    sys.exit(6)
query = next(a.split("=", 1)[1] for a in args if a.startswith("--query-gpu="))
if query == "index":
    print("0")
    sys.exit(0)
rows = {rows!r}
i = 0
while True:
    print(rows[i % len(rows)], flush=True)
    i += 1
    time.sleep(0.05)
"""

ROWS = [
    "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
    "0, 1950, 1965, 980.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
    "0, 1965, 1965, 650.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
]


@pytest.fixture
def fake_smi(tmp_path, monkeypatch):
    def make(accepted):
        path = tmp_path / "nvidia-smi"
        path.write_text(FAKE.format(python=sys.executable, accepted=list(accepted), rows=ROWS))
        path.chmod(path.stat().st_mode | stat.S_IXUSR)
        monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    return make


def test_sampler_reads_clocks_and_reasons(fake_smi):
    fake_smi(["0"])
    c = bench.ClockSampler(0)
    c.start()
    assert c.proc is not None
    time.sleep(0.5)
    clk = c.stop()
    assert clk is not None and clk["samples"] >= 3
    assert clk["sm_max_mhz"] == 1965.0
    assert 1950.0 <= clk["sm_mhz"] <= 1965.0
    assert clk["reasons"] == ["sw_power_cap"]
    assert not os.path.exists(c.path)  # the sample file is removed


def test_sampler_prefers_the_device_uuid(fake_smi, monkeypatch):
    """With CUDA_VISIBLE_DEVICES remapping, the CUDA index is not nvidia-smi's:
    the UUID is tried first."""
    fake_smi(["GPU-1234"])
    c = bench.ClockSampler(0)
    monkeypatch.setattr(c, "_ids", lambda: ["GPU-1234", "0"])
    assert c._pick_id() == "GPU-1234"
    fake_smi(["0"])  # an id it refuses falls through to the next
    assert c._pick_id() == "0"


def test_sampler_without_nvidia_smi_reports_nothing(fake_smi):
    fake_smi([])  # refuses every id
    c = bench.ClockSampler(0)
    c.start()
    assert c.proc is None and c.stop() is None


def test_traffic_record_is_used_only_for_the_kernels_it_was_taken_on(tmp_path, monkeypatch):
    rec = {"source_sha": bench.kernel_source_hash(),
           "kernels": {"sliding": {"dram_bytes_per_launch": 123}}}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(path))
    assert bench.traffic_for("sliding") == 123
    assert bench.traffic_for("global") is None  # no entry
    rec["source_sha"] = "0" * 16  # kernels changed since the counters were taken
    path.write_text(json.dumps(rec))
    assert bench.traffic_for("sliding") is None
    path.write_text("not json")
    assert bench.traffic_for("sliding") is None


def test_source_hash_ignores_comments_only(tmp_path):
    """A comment or layout edit keeps the traffic record valid; a code edit,
    even one inside a string literal that looks like a comment, does not."""
    src = tmp_path / "k.cuh"
    base = 'int a = 1;  // scale\nasm("mov.b32 %0, 1;  // x");\n'
    src.write_text(base)
    h0 = bench.kernel_source_hash(str(tmp_path))
    src.write_text("// header\n" + base.replace("// scale", "/* another\n comment */") + "\n\n")
    assert bench.kernel_source_hash(str(tmp_path)) == h0
    src.write_text(base.replace("int a = 1;", "int a =\n    1;"))  # re-wrapped
    assert bench.kernel_source_hash(str(tmp_path)) == h0
    src.write_text(base.replace('"mov.b32 %0, 1;', '"mov.b32 "\n    "%0, 1;'))  # literal split
    assert bench.kernel_source_hash(str(tmp_path)) == h0
    src.write_text(base.replace("1;  //", "2;  //"))
    assert bench.kernel_source_hash(str(tmp_path)) != h0
    src.write_text(base.replace("// x", "// y"))
    assert bench.kernel_source_hash(str(tmp_path)) != h0


def test_committed_traffic_record_names_every_profiled_kernel():
    with open(bench.TRAFFIC_RECORD) as f:
        rec = json.load(f)
    assert set(rec["kernels"]) >= {"sliding", "global", "combine", "fp8_sliding"}
    for ent in rec["kernels"].values():
        assert ent["dram_bytes_per_launch"] > 0


def test_peak_falls_back_without_a_measured_record(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peak_gbs() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6450.0}))
    assert bench.measured_peak_gbs() == (6450.0, "measured")


def test_multi_token_accounting_against_brute_force():
    """The verify / prefill byte and flop accounting: pairs of (token, attended
    position) and the union of the tokens' ranges, counted one by one."""
    import workloads
    from decode_attention_09_b200 import accounting
    for spec in (workloads.sliding_spec(4096, 16), workloads.global_spec(4096)):
        for L, T in ((40, 8), (10, 10), (100, 1), (3, 3), (70, 33)):
            pairs, union = 0, set()
            for t in range(T):
                p = L - T + t
                lo = max(0, p + 1 - spec.window) if spec.window > 0 else 0
                rng = range(lo, p + 1)
                pairs += len(rng)
                union.update(rng)
            assert accounting.multi_attended_pairs(spec, L, T) == pairs
            assert accounting.union_positions(spec, L, T) == len(union)
            assert accounting.layer_prefill_flops(spec, [L], T) == \
                pairs * 4 * spec.head_dim * spec.n_q_heads
            assert accounting.layer_multi_kv_bytes(spec, [L, L], T) == \
                2 * len(union) * accounting.kv_bytes_per_position(spec)
