"""The library's split planner, csrc/partition.cuh, run on the CPU.

The header is copied beside an empty ptx.cuh and compiled with g++ together
with tests/planner_host.cpp, which emulates the warp intrinsics it uses (32
lanes as fibers) and checks plan_chunk, SegmentIter, unit_chunks, segment_runs,
TileIterT and plan_unit_split on random ragged batches: every attended position
of every unit is covered exactly once, slots are unique, chunks and parts are
aligned, and tiles follow their segments without crossing the ring's end.
A planted mistake in a copy of the header must make the check fail.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
PARTITION = os.path.join(os.path.dirname(HERE), "decode_attention_09_b200", "csrc",
                         "partition.cuh")
HARNESS = os.path.join(HERE, "planner_host.cpp")


def build_harness(tmp_path, header_text):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no g++")
    (tmp_path / "partition.cuh").write_text(header_text)
    (tmp_path / "ptx.cuh").write_text("// the planner uses none of the PTX wrappers\n")
    exe = tmp_path / "planner_host"
    subprocess.run([gxx, "-std=c++17", "-O2", "-Wno-unknown-pragmas", "-I", str(tmp_path),
                    HARNESS, "-o", str(exe)], check=True)
    return exe


def test_split_planner_covers_every_position_once(tmp_path):
    with open(PARTITION) as f:
        exe = build_harness(tmp_path, f.read())
    r = subprocess.run([str(exe), "200"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok 200"


@pytest.mark.parametrize("original,planted", [
    ("const int64_t ce = imin64(cs + chunk, total);",
     "const int64_t ce = imin64(cs + chunk - 1, total);"),
    ("const int32_t first = min(len, C - s0);", "const int32_t first = min(len, C - s0 - 1);"),
    ("if (lane >= o) v += t;", "if (lane > o) v += t;"),
    ("off = seg.lo + (run == 1 ? runs.len0 : 0) + t0;", "off = seg.lo + t0;"),
])
def test_planted_planner_mistake_is_caught(tmp_path, original, planted):
    with open(PARTITION) as f:
        text = f.read()
    assert text.count(original) == 1
    exe = build_harness(tmp_path, text.replace(original, planted))
    r = subprocess.run([str(exe), "40"], capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, "the planted mistake went unnoticed"
