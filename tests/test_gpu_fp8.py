"""GPU parity of gdattn_decode_fp8 (fp8 e4m3 KV cache with per-row scales)
against the float64 oracle, on the same codes, scales and bf16 queries.

Gates as for the bf16 cache: max |dout| <= 8e-3 with a one-bf16-ulp floor (V
rows carry a per-row spread, so some outputs exceed 1) and max |dlse| <= 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from decode_attention_09_b200 import binding
from gpu_helpers import Guarded, compare, guarded_workspace, require_gpu

pytestmark = pytest.mark.gpu


class Fp8Layer:
    """Device copies of an fp8 layer's inputs plus a workspace."""

    def __init__(self, inp, split_ctas=0, flags=0, device="cuda"):
        self.inp = inp
        self.q = inp.q.to(device)
        self.kc = inp.k_codes.to(device)
        self.vc = inp.v_codes.to(device)
        self.ks = inp.k_scale.to(device)
        self.vs = inp.v_scale.to(device)
        self.seqlens = inp.seqlens.to(device=device, dtype=torch.int32)
        self.B = inp.q.shape[0]
        self.max_seqlen = int(inp.seqlens.max())
        self.desc = binding.desc_from_spec(inp.spec, split_ctas, capacity=inp.k_codes.shape[1],
                                           flags=flags)
        # outputs, LSE and workspace between guard bytes checked after every run
        self._ws = guarded_workspace(self.B, self.max_seqlen, self.desc, device)
        self.ws = self._ws.t
        self._out = Guarded(tuple(self.q.shape), torch.bfloat16, device)
        self._lse = Guarded((self.B, self.q.shape[1]), torch.float32, device)

    def run(self, check_status=True):
        out, lse = binding.decode_fp8(self.q, self.kc, self.vc, self.ks, self.vs, self.seqlens,
                                      self.desc, self.max_seqlen, out=self._out.t,
                                      lse=self._lse.t, workspace=self.ws)
        if check_status:
            st = binding.check_device_status(self.ws)
            assert st == binding.GDATTN_OK, binding.status_string(st)
        torch.cuda.synchronize()
        for g, what in ((self._out, "out"), (self._lse, "lse"), (self._ws, "workspace")):
            g.check(what)
        return out.clone(), lse.clone()


def fp8_ref(inp):
    s = inp.spec
    return oracle.get().decode_fp8(inp.q, inp.k_codes, inp.v_codes, inp.k_scale, inp.v_scale,
                                   inp.seqlens, s.window, s.softcap, s.scale)


SPLITS = [0, 1, 2, 3, 7, 33, 300]

# (B, Hq, Hkv, C, seqlens, window, softcap, spread); D = 256, two query heads per KV head
CASES = {
    "one_tile_partial": (2, 16, 8, 64, [64, 37], 64, 0.0, 1.5),
    "ring_wraps": (2, 16, 8, 48, [100, 47], 48, 0.0, 1.5),
    "window_lt_cap": (2, 16, 8, 64, [130, 20], 40, 0.0, 1.5),
    "edges": (5, 16, 8, 32, [1, 2, 31, 32, 33], 32, 0.0, 1.5),
    "multi_tile_ring": (2, 16, 8, 200, [450, 130], 200, 0.0, 1.5),
    "hkv1_long": (1, 2, 1, 700, [700], 0, 0.0, 1.5),
    "softcap_hkv4": (3, 8, 4, 130, [130, 64, 65], 0, 30.0, 1.5),
    "wide_row_scales": (2, 16, 8, 300, [300, 299], 0, 0.0, 6.0),
}

_ref_cache = {}


def case_ref(name):
    if name not in _ref_cache:
        B, Hq, Hkv, C, sl, w, cap, spread = CASES[name]
        inp = workloads.random_fp8_case(500 + sorted(CASES).index(name), B, Hq, Hkv, 256, C, sl,
                                        window=w, softcap=cap, spread=spread)
        _ref_cache[name] = (inp, fp8_ref(inp))
    return _ref_cache[name]


@pytest.mark.parametrize("split", SPLITS)
@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8_sweep(name, split):
    require_gpu()
    inp, (o_ref, l_ref) = case_ref(name)
    out, lse = Fp8Layer(inp, split_ctas=split).run()
    compare(out, lse, o_ref, l_ref, ulp_floor=True, what=f"fp8 {name} split={split}")


@pytest.mark.parametrize("name", ["multi_tile_ring", "hkv1_long", "wide_row_scales"])
def test_fp8_even_unit_split(name):
    """The even unit split: whole-tile parts merged as tagged words in the kernel."""
    require_gpu()
    inp, (o_ref, l_ref) = case_ref(name)
    layer = Fp8Layer(inp, flags=binding.GDATTN_FLAG_EVEN_UNITS)
    for rep in range(3):  # the tag epochs advance from call to call
        out, lse = layer.run()
        compare(out, lse, o_ref, l_ref, ulp_floor=True, what=f"fp8 even {name} call {rep}")


def _sliding_bench_layer(seed=77, batch=8, ctx=8192):
    spec = workloads.sliding_spec(capacity=1024, window=1024)
    sl = torch.full((batch,), ctx, dtype=torch.int32)
    return workloads.fp8_layer_inputs(spec, batch, sl, seed)


@pytest.mark.parametrize("flags", [0, binding.GDATTN_FLAG_EVEN_UNITS])
def test_fp8_sliding_layer_full_size(flags):
    """The 12B sliding layer at batch 8, context 8192 (window 1024, ring of 1024
    slots), every output compared."""
    require_gpu()
    inp = _sliding_bench_layer()
    o_ref, l_ref = fp8_ref(inp)
    out, lse = Fp8Layer(inp, flags=flags).run()
    compare(out, lse, o_ref, l_ref, ulp_floor=True, what=f"fp8 sliding b8 flags={flags}")


def test_fp8_signed_and_zero_scales():
    """Scales of either sign, and zero scales (rows of value 0), per the definition."""
    require_gpu()
    inp = workloads.random_fp8_case(611, 3, 16, 8, 256, 256, [256, 200, 77], window=256)
    g = torch.Generator().manual_seed(612)
    for t in (inp.k_scale, inp.v_scale):
        sign = torch.where(torch.rand(t.shape, generator=g) < 0.5, -1.0, 1.0)
        t.mul_(sign)
        t[torch.rand(t.shape, generator=g) < 0.05] = 0.0
    o_ref, l_ref = fp8_ref(inp)
    out, lse = Fp8Layer(inp).run()
    compare(out, lse, o_ref, l_ref, ulp_floor=True, what="fp8 signed/zero scales")


def test_fp8_rows_outside_window_are_not_read():
    """NaN codes in every slot outside the attended range leave the result unchanged."""
    require_gpu()
    inp = workloads.random_fp8_case(613, 2, 16, 8, 256, 320, [300, 100], window=200)
    o_ref, l_ref = fp8_ref(inp)
    for b, L in enumerate([300, 100]):
        attended = set(p % 320 for p in range(max(0, L - 200), L))
        for slot in range(320):
            if slot not in attended:
                inp.k_codes[b, slot] = 0x7F
                inp.v_codes[b, slot] = 0x7F
                inp.k_scale[b, :, slot] = float("nan")
                inp.v_scale[b, :, slot] = float("nan")
    out, lse = Fp8Layer(inp).run()
    compare(out, lse, o_ref, l_ref, ulp_floor=True, what="fp8 poisoned outside window")


def test_fp8_bad_seqlen_is_reported():
    require_gpu()
    inp = workloads.random_fp8_case(614, 3, 16, 8, 256, 64, [5, 0, 9], window=64)
    layer = Fp8Layer(inp)
    layer.max_seqlen = 9
    out, lse = layer.run(check_status=False)
    assert binding.check_device_status(layer.ws) == binding.GDATTN_ERR_DEVICE_SEQLEN
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
    o_ref, l_ref = oracle.get().decode_fp8(inp.q[[0, 2]], inp.k_codes[[0, 2]],
                                           inp.v_codes[[0, 2]], inp.k_scale[[0, 2]],
                                           inp.v_scale[[0, 2]], inp.seqlens[[0, 2]], 64, 0.0,
                                           inp.spec.scale)
    compare(out[[0, 2]], lse[[0, 2]], o_ref, l_ref, ulp_floor=True, what="fp8 valid rows")


def test_fp8_repeatable_and_graph_capturable():
    """Two calls give the same bits; a captured call replays to the same bits."""
    require_gpu()
    inp = _sliding_bench_layer(seed=78, batch=4, ctx=3000)
    layer = Fp8Layer(inp, flags=binding.GDATTN_FLAG_EVEN_UNITS)
    o1, l1 = layer.run()
    o2, l2 = layer.run()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1.view(torch.int32), l2.view(torch.int32))
    out = torch.empty_like(o1)
    lse = torch.empty_like(l1)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            binding.decode_fp8(layer.q, layer.kc, layer.vc, layer.ks, layer.vs, layer.seqlens,
                               layer.desc, layer.max_seqlen, out=out, lse=lse,
                               workspace=layer.ws, stream=s)
    for _ in range(2):
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), o1.view(torch.int16))
        assert torch.equal(lse.view(torch.int32), l1.view(torch.int32))
    assert binding.check_device_status(layer.ws) == binding.GDATTN_OK
    del g
