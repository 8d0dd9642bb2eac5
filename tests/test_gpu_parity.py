"""GPU parity: libgdattn through its C ABI versus the float64 oracle.

Inputs are seeded bf16; both sides see the same bits.  Gates: max |dout| <= 8e-3
on the bf16 output (with a one-bf16-ulp floor where heavy key rows push |out|
above 1) and max |dlse| <= 1e-3 on the fp32 LSE.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from decode_attention_09_b200 import binding
from gpu_helpers import (GpuLayer, compare, oracle_for, oracle_per_sequence, require_gpu,
                         uses_tensor_cores)

pytestmark = pytest.mark.gpu

SPLITS = [0, 1, 2, 3, 7, 33, 300]

# (B, Hq, Hkv, D, C, seqlens, window, softcap, kv_shared)
CASES = {
    # tensor-core pair path (G = 2, D = 256, separate V)
    "sliding_g2_nowrap_cap": (3, 16, 8, 256, 64, [64, 1, 37], 64, 50.0, False),
    "sliding_g2_ring_wraps": (2, 16, 8, 256, 48, [100, 47], 48, 0.0, False),
    "sliding_g2_window_lt_cap": (2, 16, 8, 256, 64, [130, 20], 40, 0.0, False),
    "sliding_g2_edges": (5, 16, 8, 256, 32, [1, 2, 31, 32, 33], 32, 0.0, False),
    "pair_multi_tile_ring": (2, 16, 8, 256, 200, [450, 130], 200, 0.0, False),
    "pair_hkv1_long": (1, 2, 1, 256, 700, [700], 0, 0.0, False),
    "pair_softcap_hkv4": (3, 8, 4, 256, 130, [130, 64, 65], 0, 30.0, False),
    # CUDA-core path (G = 1, 2, 4 otherwise)
    "core_g2_shared_d256": (2, 16, 8, 256, 90, [90, 17], 0, 0.0, True),
    "global_g1_shared_d512": (2, 8, 8, 512, 70, [70, 9], 0, 0.0, True),
    "global_g4_hkv2": (2, 8, 2, 256, 90, [90, 33], 0, 0.0, False),
    "global_g4_hkv1_d512": (1, 4, 1, 512, 200, [200], 0, 0.0, False),
    "global_g1_hkv4_shared": (2, 4, 4, 256, 50, [50, 50], 0, 5.0, True),
    # tensor-core path (G = 16, D = 512, K = V)
    "tc_multi_tile_tail": (1, 16, 1, 512, 300, [300], 0, 0.0, True),
    "tc_edges": (3, 16, 1, 512, 200, [1, 64, 200], 0, 0.0, True),
    "tc_hkv2": (2, 32, 2, 512, 150, [150, 65], 0, 0.0, True),
    "tc_window_ring": (2, 16, 1, 512, 96, [150, 96], 96, 0.0, True),
    "tc_softcap": (2, 16, 1, 512, 129, [129, 128], 0, 30.0, True),
    # tensor-core 16-head kernel with a separate V cache, and 8-head groups
    "tc16_sepv_multi_tile": (2, 16, 1, 512, 300, [300, 77], 0, 0.0, False),
    "tc16_sepv_window_ring": (2, 16, 1, 512, 96, [150, 96], 96, 0.0, False),
    "tc16_sepv_softcap_hkv2": (2, 32, 2, 512, 129, [129, 128], 0, 30.0, False),
    "tc8_shared_hkv2": (2, 16, 2, 512, 200, [200, 65], 0, 0.0, True),
    "tc8_sepv_ring_edges": (3, 8, 1, 512, 96, [150, 96, 1], 96, 20.0, False),
}

_ref_cache = {}


def case_inputs(name):
    B, Hq, Hkv, D, C, sl, w, cap, shared = CASES[name]
    seed = 100 + sorted(CASES).index(name)
    return workloads.random_case(seed, B, Hq, Hkv, D, C, sl, window=w, softcap=cap,
                                 kv_shared=shared)


def case_ref(name):
    if name not in _ref_cache:
        inp = case_inputs(name)
        _ref_cache[name] = (inp, oracle_for(inp))
    return _ref_cache[name]


@pytest.mark.parametrize("split", SPLITS)
@pytest.mark.parametrize("name", sorted(CASES))
def test_sweep(name, split):
    require_gpu()
    inp, (o_ref, l_ref) = case_ref(name)
    out, lse = GpuLayer(inp, split_ctas=split).run()
    compare(out, lse, o_ref, l_ref, what=f"{name} split={split}")


# ---------------------------------------------------------------- workloads


def test_single_sliding_layer():
    """q [1,16,256], K/V [2048,8,256], w 512, cap 50, scale 1/16."""
    require_gpu()
    w = workloads.single_sliding()
    inp = workloads.workload_layer_inputs(w, 0)
    o_ref, l_ref = oracle_for(inp)
    out, lse = GpuLayer(inp).run()
    compare(out, lse, o_ref, l_ref, what=w.name)


def test_single_global_layer():
    """q [1,16,512], one K=V tensor [32768,1,512], split-KV + LSE combine."""
    require_gpu()
    w = workloads.single_global()
    inp = workloads.workload_layer_inputs(w, 0)
    o_ref, l_ref = oracle_for(inp)
    out, lse = GpuLayer(inp).run()
    compare(out, lse, o_ref, l_ref, what=w.name)


@pytest.mark.parametrize("flags", [0, binding.GDATTN_FLAG_EVEN_UNITS])
@pytest.mark.parametrize("layer", [0, 5])
def test_gemma4_12b_stack_layers(layer, flags):
    """Batch 8, context 8192: one sliding layer (ring of 1024) and one global K=V
    layer, with the default planner and with the even unit split the bench uses."""
    require_gpu()
    w = workloads.gemma4_12b_b8_l8192()
    inp = workloads.workload_layer_inputs(w, layer)
    o_ref, l_ref = oracle_for(inp)
    layer_gpu = GpuLayer(inp)
    if flags:
        layer_gpu.set_desc(binding.desc_from_spec(inp.spec, flags=flags))
    out, lse = layer_gpu.run()
    compare(out, lse, o_ref, l_ref, what=f"{w.name} layer {layer} flags {flags}")


@pytest.mark.parametrize("layer", [0, 1])
def test_ragged_batch(layer):
    """Batch 64, L ~ U[512, 32768]: every sequence against the oracle."""
    require_gpu()
    w = workloads.ragged_b64()
    inp = workloads.workload_layer_inputs(w, layer, device="cuda")
    o_ref, l_ref = oracle_per_sequence(inp)
    out, lse = GpuLayer(inp).run()
    compare(out, lse, o_ref, l_ref, what=f"{w.name} layer {layer}")


@pytest.mark.parametrize("layer", [0, 5])
def test_long_context(layer):
    """Batch 4, context 131072, 1 % of key rows x8: every sequence, ulp floor."""
    require_gpu()
    w = workloads.long_context_b4()
    inp = workloads.workload_layer_inputs(w, layer, device="cuda")
    o_ref, l_ref = oracle_per_sequence(inp)
    out, lse = GpuLayer(inp).run()
    compare(out, lse, o_ref, l_ref, ulp_floor=True, what=f"{w.name} layer {layer}")


# --------------------------------------------------------------- invariants


@pytest.mark.parametrize("name", ["sliding_g2_window_lt_cap", "sliding_g2_ring_wraps",
                                  "pair_multi_tile_ring", "tc_multi_tile_tail", "tc_window_ring",
                                  "tc_edges", "tc16_sepv_window_ring", "tc8_sepv_ring_edges"])
def test_unattended_slots_never_matter(name):
    """NaN in every cache slot outside the attended range leaves the result unchanged."""
    require_gpu()
    inp, _ = case_ref(name)
    clean_out, clean_lse = GpuLayer(inp, split_ctas=3).run()
    k = inp.k.clone()
    v = inp.v.clone() if inp.v is not None else None
    C = k.shape[1]
    w = inp.spec.window
    for b, L in enumerate(inp.seqlens.tolist()):
        n = min(L, w) if w > 0 else L
        keep = torch.zeros(C, dtype=torch.bool)
        for p in range(L - n, L):
            keep[p % C] = True
        k[b, ~keep] = float("nan")
        if v is not None:
            v[b, ~keep] = float("nan")
    poisoned = workloads.LayerInputs(inp.q, k, v, inp.seqlens, inp.spec)
    out, lse = GpuLayer(poisoned, split_ctas=3).run()
    assert torch.equal(out, clean_out)
    assert torch.equal(lse, clean_lse)


@pytest.mark.parametrize("which", ["single_sliding", "single_global"])
def test_split_count_invariance(which):
    """One CTA or many: the same result up to rounding.

    The CUDA-core path keeps the softmax weights in fp32, so only the last bf16
    rounding of out may differ (one ulp).  The tensor-core path rounds each
    weight p = exp(s - m) to bf16 against the running max m, which depends on
    where the range is cut; a weight's relative error is up to 2^-9, so two
    splits may differ by ~2^-8 * max|v| in the worst case: gate at 4e-3, half
    the oracle gate.
    """
    require_gpu()
    w = getattr(workloads, which)()
    inp = workloads.workload_layer_inputs(w, 0)
    o1, l1 = GpuLayer(inp, split_ctas=1).run()
    tensor_path = uses_tensor_cores(inp.spec)
    for split in (2, 5, 148, 296):
        o2, l2 = GpuLayer(inp, split_ctas=split).run()
        d = (o1.float() - o2.float()).abs()
        if tensor_path:
            tol = torch.full_like(d, 4e-3)
        else:
            tol = torch.from_numpy(np.exp2(np.floor(np.log2(np.maximum(
                o1.float().abs().cpu().numpy(), 1e-30))) - 7)).to(d.device) + 1e-12
        assert bool((d <= tol).all()), f"split {split}: max {d.max().item()}"
        assert (l1 - l2).abs().max().item() <= (1e-4 if tensor_path else 2e-5)


def test_bitwise_reproducible():
    require_gpu()
    for name in ("sliding_g2_ring_wraps", "tc_multi_tile_tail"):
        inp, _ = case_ref(name)
        layer = GpuLayer(inp, split_ctas=7)
        a = layer.run()
        b = layer.run()
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_combine_matches_oracle_merge():
    """gdattn_combine on oracle-made partials equals the oracle's own LSE merge."""
    require_gpu()
    orc = oracle.get()
    inp = workloads.random_case(55, 2, 8, 2, 256, 120, [120, 77], window=0, softcap=0.0)
    s = inp.spec
    cuts = [[0, 10, 10, 64, 120], [0, 5, 40, 77, 77]]  # includes empty parts
    parts_o, parts_l = [], []
    for p in range(4):
        lo = [c[p] for c in cuts]
        hi = [c[p + 1] for c in cuts]
        o, l = orc.attend(inp.q, inp.k, inp.v, lo, hi, s.softcap, s.scale)
        parts_o.append(o)
        parts_l.append(l)
    po = np.stack(parts_o, axis=2)
    pl = np.stack(parts_l, axis=2)
    o_ref, l_ref = orc.combine(po, pl)
    out, lse = binding.combine(torch.from_numpy(po).float().cuda().contiguous(),
                               torch.from_numpy(pl).float().cuda().contiguous())
    torch.cuda.synchronize()
    compare(out, lse, o_ref, l_ref, what="combine")
    # all-empty parts: out = 0, lse = -inf
    out, lse = binding.combine(torch.zeros((1, 2, 3, 256), device="cuda"),
                               torch.full((1, 2, 3), float("-inf"), device="cuda"))
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def test_device_detects_impossible_seqlens():
    """L = 0, or a global layer's L beyond the cache: status word says so, no fault."""
    require_gpu()
    inp = workloads.random_case(56, 3, 16, 8, 256, 32, [5, 0, 9], window=16)
    layer = GpuLayer(inp, max_seqlen=16)
    out, lse = binding.decode(layer.q, layer.k, layer.v, layer.seqlens, layer.desc, 16,
                              workspace=layer.ws)
    assert binding.check_device_status(layer.ws) == binding.GDATTN_ERR_DEVICE_SEQLEN
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
    assert binding.check_device_status(layer.ws) == binding.GDATTN_OK  # cleared by the read
    inp = workloads.random_case(57, 1, 16, 1, 512, 64, [100], window=0, kv_shared=True)
    layer = GpuLayer(inp, max_seqlen=100)
    binding.decode(layer.q, layer.k, layer.v, layer.seqlens, layer.desc, 100, workspace=layer.ws)
    assert binding.check_device_status(layer.ws) == binding.GDATTN_ERR_DEVICE_SEQLEN


def test_cuda_graph_replay_matches_eager():
    """Decode calls captured in a CUDA graph give the eager results."""
    require_gpu()
    layers = [GpuLayer(case_ref(n)[0]) for n in ("sliding_g2_ring_wraps", "tc_multi_tile_tail")]
    eager = [ly.run() for ly in layers]
    outs = [(torch.empty_like(e[0]), torch.empty_like(e[1])) for e in eager]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for ly, (o, l) in zip(layers, outs):
                binding.decode(ly.q, ly.k, ly.v, ly.seqlens, ly.desc, ly.max_seqlen, out=o, lse=l,
                               workspace=ly.ws, stream=s)
    g.replay()
    torch.cuda.synchronize()
    for (o, l), (eo, el) in zip(outs, eager):
        assert torch.equal(o, eo) and torch.equal(l, el)


def test_latched_timeout_is_reported_then_cleared():
    """Failure detection's host side, with no wait made to run out: a workspace
    whose status word carries the timeout bit (what a kernel whose bounded wait
    expired leaves behind) reads as GDATTN_ERR_DEVICE_TIMEOUT.  Kernels only set
    bits, so the latch survives a later call; the read clears it.  With both bits
    set, the timeout is the one reported."""
    require_gpu()
    inp = workloads.random_case(59, 2, 16, 8, 256, 64, [64, 30], window=64)
    o_ref, l_ref = oracle_for(inp)
    layer = GpuLayer(inp)
    word = layer.ws[:4].view(torch.int32)
    word.fill_(1)  # the timeout bit
    out, lse = layer.run(check_status=False)
    assert binding.check_device_status(layer.ws) == binding.GDATTN_ERR_DEVICE_TIMEOUT
    assert binding.check_device_status(layer.ws) == binding.GDATTN_OK
    compare(out, lse, o_ref, l_ref, ulp_floor=True, what="call after a latched timeout")
    word.fill_(3)  # the timeout and sequence-length bits
    assert binding.check_device_status(layer.ws) == binding.GDATTN_ERR_DEVICE_TIMEOUT
    assert binding.check_device_status(layer.ws) == binding.GDATTN_OK


@pytest.mark.parametrize("split", [2, 7, 33])
def test_part_counters_return_to_zero(split):
    """Units merged inside the decode kernel leave their arrival counters at
    zero (the workspace holds the status word, then one counter per unit)."""
    require_gpu()
    inp, (o_ref, l_ref) = case_ref("pair_multi_tile_ring")
    layer = GpuLayer(inp, split_ctas=split)
    for _ in range(3):
        out, lse = layer.run()
        units = inp.q.shape[0] * inp.spec.n_kv_heads
        cnt = layer.ws[256:256 + 4 * units].view(torch.int32)
        assert int(cnt.abs().sum()) == 0
    compare(out, lse, o_ref, l_ref, ulp_floor=True, what=f"split {split}")


# (B, Hq, Hkv, D, C, seqlens, window, softcap, kv_shared) run with
# GDATTN_FLAG_EVEN_UNITS: every (sequence, KV head) unit cut into k whole-tile parts
EVEN_CASES = {
    "pair_k2_empty_rank": (2, 16, 8, 256, 200, [450, 130], 200, 0.0, False),
    "pair_one_unit": (1, 2, 1, 256, 700, [700], 0, 0.0, False),
    "pair_long": (1, 4, 2, 256, 2048, [2048], 0, 0.0, False),
    "pair_ragged_mostly_empty": (3, 8, 4, 256, 1000, [1000, 64, 1], 0, 0.0, False),
    "pair_softcap_ring": (2, 16, 8, 256, 512, [1300, 700], 512, 30.0, False),
    "tc16_one_unit": (1, 16, 1, 512, 3000, [3000], 0, 0.0, True),
    "tc16_ragged": (3, 16, 1, 512, 2000, [2000, 100, 1], 0, 0.0, True),
    "tc16_hkv2_softcap": (2, 32, 2, 512, 700, [700, 650], 0, 20.0, True),
    "tc16_k3_uneven_slices": (40, 16, 1, 512, 192, [192] * 40, 0, 0.0, True),
    "tc16_many_parts_combine": (1, 16, 1, 512, 4096, [4096], 0, 0.0, True),
    "tc16_sepv_ragged": (3, 16, 1, 512, 2000, [2000, 100, 1], 0, 0.0, False),
    "tc8_sepv_softcap": (2, 16, 2, 512, 700, [700, 650], 0, 20.0, False),
    "tc16_one_unit_64_parts": (1, 16, 1, 512, 32768, [32768], 0, 0.0, True),
}


@pytest.mark.parametrize("name", sorted(EVEN_CASES))
def test_even_unit_split_matches_oracle(name):
    """Units cut into k whole-tile parts (ragged lengths and empty parts
    included: the flag only promises balance) give the oracle's result."""
    require_gpu()
    B, Hq, Hkv, D, C, sl, w, cap, shared = EVEN_CASES[name]
    inp = workloads.random_case(300 + sorted(EVEN_CASES).index(name), B, Hq, Hkv, D, C, sl,
                                window=w, softcap=cap, kv_shared=shared)
    o_ref, l_ref = oracle_for(inp)
    layer = GpuLayer(inp)
    layer.set_desc(binding.desc_from_spec(inp.spec, capacity=C,
                                          flags=binding.GDATTN_FLAG_EVEN_UNITS))
    units = B * Hkv
    splits = binding.plan_splits(B, layer.max_seqlen, layer.desc)
    assert splits % units == 0 and splits // units >= 2, splits  # the unit split was taken
    expect_launches = 2 if D == 512 else 1  # the 16-head kernel merges in the combine kernel
    assert binding.launches_per_call(B, layer.max_seqlen, layer.desc) == expect_launches
    for _ in range(2):
        out, lse = layer.run()
        compare(out, lse, o_ref, l_ref, ulp_floor=True, what=f"{name} k={splits // units}")


def test_even_split_workspace_shared_by_two_geometries():
    """Two even-split layers with different unit counts and part counts take
    turns on one workspace: per-unit tags and cleared words keep every call's
    merge on its own parts."""
    require_gpu()
    a = workloads.random_case(401, 2, 16, 8, 256, 300, [300, 300], window=300)   # 16 units
    b = workloads.random_case(402, 1, 4, 2, 256, 1500, [1500], window=0)         # 2 units, more parts
    refs = [oracle_for(x) for x in (a, b)]
    layers = [GpuLayer(x) for x in (a, b)]
    for ly, x in zip(layers, (a, b)):
        ly.desc = binding.desc_from_spec(x.spec, capacity=x.k.shape[1],
                                         flags=binding.GDATTN_FLAG_EVEN_UNITS)
    need = max(binding.workspace_size(ly.B, ly.max_seqlen, ly.desc) for ly in layers)
    shared = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for ly in layers:
        ly.ws = shared
    ks = [binding.plan_splits(ly.B, ly.max_seqlen, ly.desc) // (ly.B * x.spec.n_kv_heads)
          for ly, x in zip(layers, (a, b))]
    assert ks[0] != ks[1] and min(ks) >= 2, ks
    for rep in range(3):
        for ly, (o_ref, l_ref), name in zip(layers, refs, "ab"):
            out, lse = ly.run()
            compare(out, lse, o_ref, l_ref, ulp_floor=True, what=f"{name} call {rep}")


def test_workspace_shared_by_plans_with_many_units():
    """One workspace, sized for the largest plan, serves a ragged sliding layer
    (512 units, counted merge), a global layer (combine kernel) and even-split
    sliding layers (tagged merge) in turn: each call equals the same call on a
    workspace of its own, bit for bit, with no device-side error."""
    require_gpu()
    g = torch.Generator(device="cpu").manual_seed(417)
    rag = torch.randint(1, 2100, (64,), generator=g).tolist()
    even = binding.GDATTN_FLAG_EVEN_UNITS
    specs = [(421, 64, 16, 8, 256, 1024, rag, 1024, 50.0, False, 0),
             (422, 64, 16, 1, 512, 2100, rag, 0, 0.0, True, 0),
             (423, 9, 16, 8, 256, 256, [700] * 9, 256, 0.0, False, even),
             (424, 64, 16, 8, 256, 1024, [1024] * 64, 1024, 0.0, False, even)]
    layers = []
    for seed, B, Hq, Hkv, D, C, sl, w, cap, shared, flags in specs:
        inp = workloads.random_case(seed, B, Hq, Hkv, D, C, sl, window=w, softcap=cap,
                                    kv_shared=shared, device="cuda")
        ly = GpuLayer(inp)
        ly.set_desc(binding.desc_from_spec(inp.spec, capacity=C, flags=flags))
        layers.append(ly)
    ref = [ly.run() for ly in layers]
    need = max(binding.workspace_size(ly.B, ly.max_seqlen, ly.desc) for ly in layers)
    shared_ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for ly in layers:
        ly.ws = shared_ws
    for rep, seq in enumerate([[0, 1, 2, 3], [3, 2, 1, 0], [0, 2, 0, 3, 1, 3]]):
        for i in seq:
            o, l = layers[i].run()
            assert torch.equal(o, ref[i][0]) and torch.equal(l, ref[i][1]), (rep, i)
