"""The oracle pinned to facts outside itself (CPU only)."""
import json
import os

import pytest

import oracle
import pins
import workloads

MUTATIONS = {
    1: "window one position short",
    2: "interleaved instead of contiguous GQA groups",
    3: "soft-cap applied before the scale",
    4: "LSE in log base 2",
    5: "weights not normalised",
    6: "values read from K when a separate V exists",
    7: "ring slot off by one",
    8: "scale dropped",
    9: "e4m3 exponent bias off by one",
    10: "V rows scaled by the K scales",
    11: "row scale applied twice",
    12: "row scales read token-major",
    13: "multi-query tokens not causal",
    14: "merged LSE is the largest part's",
    15: "merge weights relative to the largest part, not normalised",
    16: "soft-cap without its outer factor",
    17: "e4m3 subnormals decoded with a leading one",
    18: "multi-token window one position short",
}


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle.get())


@pytest.mark.parametrize("mutation", sorted(MUTATIONS), ids=lambda m: MUTATIONS[m])
def test_pins_catch_planted_mistake(mutation, tmp_path):
    """Each planted mistake in the oracle is caught by at least one pin."""
    mutant = oracle.load(mutation, out_dir=str(tmp_path))
    assert mutant.lib.oracle_version() == 1 + 1000 * mutation
    failed = pins.failing_pins(mutant)
    assert failed, f"no pin catches: {MUTATIONS[mutation]}"


def test_golden_kv_bytes_per_token():
    """The bench's per-token KV byte formula reproduces the figures printed for Gemma 4 12B."""
    from decode_attention_09_b200 import accounting

    with open(os.path.join(os.path.dirname(__file__), "golden", "gemma4_12b_kv_bytes.json")) as f:
        g = json.load(f)
    stack = workloads.gemma4_12b_stack(1024, 8192)
    sl = [s for s in stack if s.kind == "sliding"]
    gl = [s for s in stack if s.kind == "global"]
    assert len(sl) == g["num_layers_sliding"] and len(gl) == g["num_layers_full"]
    assert [i for i, s in enumerate(stack) if s.kind == "global"] == g["full_layer_indices"]
    per_tok = lambda specs, twice: sum(accounting.kv_bytes_per_position(s, count_shared_twice=twice)
                                       for s in specs)
    assert per_tok(sl, True) == g["sliding_bytes_per_token"]
    assert per_tok(gl, True) == g["full_bytes_per_token"]
    assert per_tok(stack, True) == g["total_bytes_per_token"]
    # K = V read once: the full layers' term halves.
    assert per_tok(stack, False) == g["sliding_bytes_per_token"] + g["full_bytes_per_token"] // 2


def test_step_bytes_of_the_headline_workload():
    """Algorithmic bytes of one 48-layer step at batch 8, context 8192, written out
    by hand: each sliding layer reads the last 1024 positions of K and V for 8 KV
    heads of 256 bf16 values; each global layer reads all 8192 positions of its
    one K = V tensor of 512 bf16 values.  With fp8 sliding caches a sliding row is
    256 one-byte codes plus a 4-byte scale."""
    from decode_attention_09_b200 import accounting

    w = workloads.gemma4_12b_b8_l8192()
    sl = w.seqlens().tolist()
    bf16 = sum(accounting.layer_kv_bytes(s, sl) for s in w.layers)
    sliding = 40 * 8 * 1024 * (8 * 256 * 2) * 2
    glob = 8 * 8 * 8192 * (1 * 512 * 2)
    assert bf16 == sliding + glob == 3_221_225_472
    fp8 = sum(accounting.layer_fp8_kv_bytes(s, sl) for s in w.layers if s.kind == "sliding")
    assert fp8 == 40 * 8 * 1024 * (8 * (256 + 4)) * 2 == 1_363_148_800
    assert accounting.layer_kv_bytes(w.layers[0], [5]) == 5 * 8 * 256 * 2 * 2  # L < w
