"""gdattn_decode_append: the current token's K/V rows are written into ring
slot (L - 1) mod C by the kernel itself, then attention runs over the updated
cache.  Checked against the oracle over a host copy of the cache with the same
rows written, and the device cache bit for bit (only those slots may change)."""
import pytest
import torch

import workloads
from decode_attention_09_b200 import binding
from gpu_helpers import Guarded, compare, guarded_workspace, oracle_for, require_gpu

pytestmark = pytest.mark.gpu

# (B, Hq, Hkv, D, C, seqlens, window, softcap, kv_shared, split, flags)
CASES = {
    "pair_ring_wraps": (3, 16, 8, 256, 128, [300, 128, 5], 128, 0.0, False, 0, 0),
    "pair_even_split": (2, 16, 8, 256, 256, [700, 256], 256, 50.0, False, 0, 1),
    "pair_forced_split": (2, 16, 8, 256, 200, [450, 130], 200, 0.0, False, 7, 0),
    "tc16_kv_shared": (2, 16, 1, 512, 400, [400, 77], 0, 0.0, True, 0, 0),
    "tc16_even_split": (2, 32, 2, 512, 300, [300, 290], 0, 0.0, True, 0, 1),
    "tc16_sepv": (2, 16, 1, 512, 400, [400, 77], 0, 0.0, False, 0, 0),
    "tc8_sepv_ring_even": (2, 16, 2, 512, 128, [300, 128], 128, 30.0, False, 0, 1),
    "core_g4": (2, 8, 2, 256, 90, [90, 33], 0, 0.0, False, 3, 0),
    "core_g2_shared": (2, 16, 8, 256, 70, [150, 70], 70, 5.0, True, 0, 0),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_append_then_decode_matches_oracle(name):
    require_gpu()
    B, Hq, Hkv, D, C, sl, w, cap, shared, split, flags = CASES[name]
    inp = workloads.random_case(500 + sorted(CASES).index(name), B, Hq, Hkv, D, C, sl, window=w,
                                softcap=cap, kv_shared=shared)
    g = torch.Generator().manual_seed(600 + sorted(CASES).index(name))
    k_new = torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16)
    v_new = None if shared else torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16)
    # Host reference: write the rows, then the plain oracle over the result.
    k_after = inp.k.clone()
    v_after = inp.v.clone() if inp.v is not None else None
    for b, L in enumerate(sl):
        k_after[b, (L - 1) % C] = k_new[b]
        if v_after is not None:
            v_after[b, (L - 1) % C] = v_new[b]
    ref_inp = workloads.LayerInputs(inp.q, k_after, v_after, inp.seqlens, inp.spec)
    o_ref, l_ref = oracle_for(ref_inp)

    dev = "cuda"
    # The caches, outputs, LSE and workspace sit between guard bytes: the append
    # writes into the caches, so a row written past either end is caught.
    kg = Guarded(tuple(inp.k.shape), torch.bfloat16, dev)
    kg.t.copy_(inp.k)
    k_dev = kg.t
    vg = None
    if inp.v is not None:
        vg = Guarded(tuple(inp.v.shape), torch.bfloat16, dev)
        vg.t.copy_(inp.v)
    v_dev = vg.t if vg is not None else None
    desc = binding.desc_from_spec(inp.spec, split, capacity=C, flags=flags)
    wsg = guarded_workspace(B, max(sl), desc)
    ws = wsg.t
    og = Guarded(tuple(inp.q.shape), torch.bfloat16, dev)
    lg = Guarded((B, Hq), torch.float32, dev)
    for rep in range(2):  # the same rows twice: the second call rewrites them
        out, lse = binding.decode_append(inp.q.to(dev), k_new.to(dev),
                                         v_new.to(dev) if v_new is not None else None, k_dev,
                                         v_dev, inp.seqlens.to(dev), desc, max(sl), out=og.t,
                                         lse=lg.t, workspace=ws)
        st = binding.check_device_status(ws)
        assert st == binding.GDATTN_OK, binding.status_string(st)
        torch.cuda.synchronize()
        for g, what in ((kg, "k cache"), (vg, "v cache"), (wsg, "workspace"), (og, "out"),
                        (lg, "lse")):
            if g is not None:
                g.check(f"{name} call {rep}: {what}")
        compare(out, lse, o_ref, l_ref, ulp_floor=True, what=f"{name} call {rep}")
        assert torch.equal(k_dev.cpu().view(torch.int16), k_after.view(torch.int16))
        if v_dev is not None:
            assert torch.equal(v_dev.cpu().view(torch.int16), v_after.view(torch.int16))
