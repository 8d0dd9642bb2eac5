"""The headline step exactly as bench.py times it, against the oracle.

bench.py's Stack builds the 48-layer Gemma-4-12B-shaped stack (batch 8,
context 8192): 40 sliding layers and 8 global K = V layers, each with its own
workspace and GDATTN_FLAG_EVEN_UNITS (the even unit split, so the pair kernel
merges tagged parts and the 16-head kernel's parts go through its merge),
captured as 48 calls in one CUDA graph whose kernels chain by programmatic
dependent launch.  The graph is replayed twice; every layer's out and lse are
compared with the float64 oracle on two sequences per replay (different ones
in each replay), and the two replays must agree bit for bit.
"""
import numpy as np
import pytest
import torch

import bench
import workloads
from decode_attention_09_b200 import binding
from gpu_helpers import compare, oracle_per_sequence, require_gpu

pytestmark = pytest.mark.gpu


def test_headline_step_graph_matches_oracle():
    require_gpu()
    w = workloads.gemma4_12b_b8_l8192()
    dev = torch.device("cuda", torch.cuda.current_device())
    stack = bench.Stack(w, dev)
    for ly in stack.layers:
        assert ly["desc"].flags == binding.GDATTN_FLAG_EVEN_UNITS
    stream = torch.cuda.Stream(dev)
    g = stack.graph(list(range(len(w.layers))), stream)
    first = None
    for rep, picks in enumerate(([0, 7], [3, 4])):
        for ly in stack.layers:
            ly["out"].fill_(float("nan"))
            ly["lse"].fill_(float("nan"))
        with torch.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        for i, ly in enumerate(stack.layers):
            assert binding.check_device_status(ly["ws"], stream) == binding.GDATTN_OK, i
        results = [(ly["out"].clone(), ly["lse"].clone()) for ly in stack.layers]
        if first is None:
            first = results
        else:
            for i, ((o0, l0), (o1, l1)) in enumerate(zip(first, results)):
                assert torch.equal(o0, o1) and torch.equal(l0, l1), f"replays differ, layer {i}"
        for i, ly in enumerate(stack.layers):
            o_ref, l_ref = oracle_per_sequence(ly["inp"], picks)
            out, lse = results[i]
            compare(out[picks], lse[picks], o_ref, l_ref,
                    what=f"replay {rep} layer {i} ({ly['spec'].kind}) sequences {picks}")
    del g
