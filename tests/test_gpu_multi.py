"""GPU parity of gdattn_decode_multi (T query tokens per sequence, each at its
own position, attending causally) against the float64 oracle's multi-query
decode, on the same bf16 inputs.  Gates as for single-token decode."""
import pytest
import torch

import oracle
import workloads
from decode_attention_09_b200 import binding
from gpu_helpers import Guarded, compare, require_gpu

pytestmark = pytest.mark.gpu

# (T, B, Hq, Hkv, D, C, seqlens, window, softcap, kv_shared, flags[, split_ctas])
CASES = {
    # single-pass pair kernel (sliding, T <= 8): ring of w + T - 1 slots that wraps
    "pair_ring_t4": (4, 3, 16, 8, 256, 259, [700, 256, 4], 256, 0.0, False, 0),
    "pair_even_t2_cap": (2, 2, 16, 8, 256, 1025, [4000, 4000], 1024, 50.0, False, 1),
    "pair_no_wrap_t7": (7, 2, 16, 8, 256, 300, [300, 9], 128, 0.0, False, 0),
    # all 16 query rows; ragged lengths, one shorter than a tile, one of exactly T
    "pair_t8_ragged": (8, 4, 16, 8, 256, 519, [2000, 519, 61, 8], 512, 0.0, False, 0),
    "pair_t8_even_cap": (8, 3, 32, 16, 256, 1031, [1500, 1500, 1500], 1024, 50.0, False, 1),
    # one token: the single-pass kernel as a plain decode
    "pair_t1": (1, 2, 16, 8, 256, 600, [600, 200], 512, 0.0, False, 1),
    # global pair layer (window 0)
    "pair_global_t5": (5, 2, 4, 2, 256, 700, [700, 333], 0, 0.0, False, 0),
    # forced flattened chunks: tokens' windows cut across many parts
    "pair_split40_t6": (6, 2, 16, 8, 256, 1100, [1100, 800], 1024, 0.0, False, 0, 40),
    # past 8 tokens the pair geometry runs as flash prefill: 64-token query blocks
    "prefill_t9": (9, 3, 16, 8, 256, 600, [600, 9, 300], 512, 0.0, False, 0),
    "prefill_t64_prompt": (64, 2, 16, 8, 256, 1100, [1100, 64], 1024, 0.0, False, 0),
    "prefill_t200_ring_cap": (200, 2, 16, 8, 256, 1223, [3000, 1223], 1024, 50.0, False, 0),
    "prefill_t130_small_w": (130, 2, 16, 8, 256, 300, [300, 131], 100, 0.0, False, 0),
    "prefill_t513_global": (513, 1, 4, 2, 256, 700, [600], 0, 0.0, False, 0),
    # flash prefill on the global geometry (K = V, head_dim 512): 64-row blocks of
    # 64 / G tokens, each on two CTAs (one per half of the head dimension)
    "gprefill_t64_g16": (64, 2, 16, 1, 512, 300, [300, 64], 0, 0.0, True, 0),
    "gprefill_t100_g8_cap": (100, 1, 16, 2, 512, 400, [350], 0, 30.0, True, 0),
    "gprefill_t40_ring": (40, 2, 16, 1, 512, 200, [900, 150], 128, 0.0, True, 0),
    # tcgen05 16-head kernel (global, K = V)
    "tc16_t3": (3, 2, 16, 1, 512, 400, [400, 77], 0, 0.0, True, 0),
    "tc16_even_t2": (2, 2, 32, 2, 512, 300, [300, 300], 0, 30.0, True, 1),
    # tcgen05 16-head kernel with a separate V, and an 8-head group
    "tc16_sepv_t4": (4, 2, 16, 1, 512, 400, [400, 77], 0, 0.0, False, 0),
    "tc8_sepv_ring_t3": (3, 2, 16, 2, 512, 130, [500, 130], 128, 0.0, False, 1),
    # CUDA-core kernel
    "core_g4_t3": (3, 2, 8, 2, 256, 90, [90, 33], 0, 0.0, False, 0),
}


def case_inputs(name):
    T, B, Hq, Hkv, D, C, sl, w, cap, shared, flags = CASES[name][:11]
    idx = sorted(CASES).index(name)
    inp = workloads.random_case(700 + idx, B, Hq, Hkv, D, C, sl, window=w, softcap=cap,
                                kv_shared=shared)
    g = torch.Generator().manual_seed(800 + idx)
    q = torch.randn((T, B, Hq, D), generator=g).to(torch.bfloat16)
    return q, inp


@pytest.mark.parametrize("name", sorted(CASES))
def test_multi_matches_oracle(name):
    require_gpu()
    T, B, Hq, Hkv, D, C, sl, w, cap, shared, flags = CASES[name][:11]
    split = CASES[name][11] if len(CASES[name]) > 11 else 0
    q, inp = case_inputs(name)
    s = inp.spec
    o_ref, l_ref = oracle.get().decode_multi(q, inp.k, inp.v, inp.seqlens, s.window, s.softcap,
                                             s.scale)
    dev = "cuda"
    desc = binding.desc_from_spec(s, capacity=C, flags=flags, split_ctas=split)
    wsg = Guarded((binding.multi_workspace_size(B, T, max(sl), desc),), torch.uint8, dev)
    ws = wsg.t
    binding.workspace_init(ws)
    og = Guarded((T, B, Hq, D), torch.bfloat16, dev)
    lg = Guarded((T, B, Hq), torch.float32, dev)
    k = inp.k.to(dev)
    v = inp.v.to(dev) if inp.v is not None else None
    for rep in range(2):  # consecutive calls on one workspace
        out, lse = binding.decode_multi(q.to(dev), k, v, inp.seqlens.to(dev), desc, max(sl),
                                        out=og.t, lse=lg.t, workspace=ws)
        st = binding.check_device_status(ws)
        assert st == binding.GDATTN_OK, binding.status_string(st)
        torch.cuda.synchronize()
        for g, what in ((wsg, "workspace"), (og, "out"), (lg, "lse")):
            g.check(f"{name} call {rep}: {what}")
        for t in range(T):
            compare(out[t], lse[t], o_ref[t], l_ref[t], ulp_floor=True,
                    what=f"{name} token {t} call {rep}")


@pytest.mark.parametrize("name,short_len", [("core_g4_t3", 2), ("pair_no_wrap_t7", 5),
                                            ("prefill_t130_small_w", 70),
                                            ("gprefill_t64_g16", 20)])
def test_multi_tokens_before_the_context_are_reported(name, short_len):
    """A sequence shorter than T: its tokens at positions below 0 attend nothing;
    the device reports it, gives them zero output and LSE -inf, and its other
    tokens and the other sequence are still right."""
    require_gpu()
    q, inp = case_inputs(name)
    inp.seqlens[1] = short_len  # sequence 1's first T - short_len tokens sit below 0
    s = inp.spec
    dev = "cuda"
    desc = binding.desc_from_spec(s, capacity=inp.k.shape[1])
    T = q.shape[0]
    max_len = int(inp.seqlens.max())
    ws = torch.empty(binding.multi_workspace_size(2, T, max_len, desc), dtype=torch.uint8,
                     device=dev)
    binding.workspace_init(ws)
    v = inp.v.to(dev) if inp.v is not None else None
    out, lse = binding.decode_multi(q.to(dev), inp.k.to(dev), v, inp.seqlens.to(dev), desc,
                                    max_len, workspace=ws)
    assert binding.check_device_status(ws) == binding.GDATTN_ERR_DEVICE_SEQLEN
    missing = T - short_len
    for t in range(missing):
        assert torch.all(out[t, 1] == 0) and torch.all(torch.isneginf(lse[t, 1]))
    vs = (lambda i: inp.v[i:i + 1]) if inp.v is not None else (lambda i: None)
    o_ref, l_ref = oracle.get().decode_multi(q[missing:, 1:2], inp.k[1:2], vs(1),
                                             inp.seqlens[1:2], s.window, s.softcap, s.scale)
    for t in range(missing, T):
        compare(out[t, 1:2], lse[t, 1:2], o_ref[t - missing], l_ref[t - missing], ulp_floor=True,
                what=f"token {t} of the short sequence")
    o_ref, l_ref = oracle.get().decode_multi(q[:, 0:1], inp.k[0:1], vs(0),
                                             inp.seqlens[0:1], s.window, s.softcap, s.scale)
    for t in range(T):
        compare(out[t, 0:1], lse[t, 0:1], o_ref[t], l_ref[t], ulp_floor=True,
                what=f"token {t} of the full-length sequence")
