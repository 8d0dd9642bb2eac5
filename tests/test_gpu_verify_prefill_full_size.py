"""The multi-token steps at the sizes and in the launch configuration bench.py
times them, against the float64 oracle.

- Verify steps: the 12B stack's sliding layer shape (16 query / 8 KV heads,
  head_dim 256, window 1024) on rings of w + 7 slots, batch 8, L = 8192, the even
  unit split, T = 4 and 8. Every token, sequence and head is compared.
- Flash prefill: one 8192-token prompt (L = T, a cache of 8192 slots) on the
  stack's sliding and global layer shapes. Sampled tokens are compared: the first
  and last of the prompt, the edges of query blocks and of the window, and
  random ones. Each is checked with the oracle's single-token decode at the
  token's own position, which is what the multi-token step defines for it. The
  oracle pins fix that equivalence ("multi-query brute force", "multi-query
  reductions"). Every token must also have a finite LSE, and every output must
  lie within the cache's value range, since each output is a convex combination
  of V rows.
"""
import dataclasses

import pytest
import torch

import oracle
import workloads
from decode_attention_09_b200 import binding
from gpu_helpers import compare, require_gpu

pytestmark = pytest.mark.gpu

DEV = "cuda"
STACK = workloads.gemma4_12b_b8_l8192()
SLIDING = STACK.layers[0]
GLOBAL = STACK.layers[workloads.GEMMA4_12B_GLOBAL_LAYERS[0]]


@pytest.mark.parametrize("T", [4, 8])
def test_verify_step_at_bench_size(T):
    require_gpu()
    assert SLIDING.kind == "sliding"
    dev = DEV
    spec = dataclasses.replace(SLIDING, capacity=SLIDING.window + 7)
    seqlens = STACK.seqlens()
    desc = binding.desc_from_spec(spec, flags=binding.GDATTN_FLAG_EVEN_UNITS)
    inp = workloads.layer_inputs(spec, STACK.batch, seqlens, 5100 + T, device=dev)
    g = torch.Generator().manual_seed(5200 + T)
    q = torch.randn((T, STACK.batch, spec.n_q_heads, spec.head_dim), generator=g).to(
        torch.bfloat16)
    max_len = int(seqlens.max())
    ws = torch.empty(binding.multi_workspace_size(STACK.batch, T, max_len, desc),
                     dtype=torch.uint8, device=dev)
    binding.workspace_init(ws)
    o_ref, l_ref = oracle.get().decode_multi(q, inp.k.cpu(), inp.v.cpu(), seqlens, spec.window,
                                             spec.softcap, spec.scale)
    qd = q.to(dev)
    for rep in range(2):  # consecutive calls on one workspace
        out, lse = binding.decode_multi(qd, inp.k, inp.v, inp.seqlens, desc, max_len,
                                        workspace=ws)
        st = binding.check_device_status(ws)
        assert st == binding.GDATTN_OK, binding.status_string(st)
        for t in range(T):
            compare(out[t], lse[t], o_ref[t], l_ref[t], ulp_floor=True,
                    what=f"T={T} token {t} call {rep}")


def prompt_samples(T, window, seed):
    """Token indices to check: the prompt's ends, 64-token block edges, the
    window's edge, and random tokens."""
    picks = {0, 1, 63, 64, 65, 127, 128, 4095, 4096, T - 65, T - 64, T - 2, T - 1}
    if window > 0:
        picks |= {window - 1, window, window + 1}
    g = torch.Generator().manual_seed(seed)
    picks |= set(torch.randint(0, T, (8,), generator=g).tolist())
    return sorted(p for p in picks if 0 <= p < T)


@pytest.mark.parametrize("kind", ["sliding", "global"])
def test_prefill_at_bench_size(kind):
    require_gpu()
    base = SLIDING if kind == "sliding" else GLOBAL
    assert base.kind == kind
    T = 8192
    dev = DEV
    spec = dataclasses.replace(base, capacity=T)
    seqlens = torch.full((1,), T, dtype=torch.int32)
    desc = binding.desc_from_spec(spec)
    inp = workloads.layer_inputs(spec, 1, seqlens, 5300 + len(kind), device=dev)
    g = torch.Generator().manual_seed(5400 + len(kind))
    q = torch.randn((T, 1, spec.n_q_heads, spec.head_dim), generator=g).to(torch.bfloat16)
    ws = torch.empty(binding.multi_workspace_size(1, T, T, desc), dtype=torch.uint8, device=dev)
    binding.workspace_init(ws)
    out, lse = binding.decode_multi(q.to(dev), inp.k, inp.v, inp.seqlens, desc, T, workspace=ws)
    st = binding.check_device_status(ws)
    assert st == binding.GDATTN_OK, binding.status_string(st)
    # properties of every token
    assert torch.isfinite(lse).all(), "a token that attends its own position has a finite LSE"
    vals = inp.k if inp.v is None else inp.v
    vmax = float(vals.float().abs().max())
    assert float(out.float().abs().max()) <= vmax * (1 + 2 ** -7), "output outside the V range"
    # sampled tokens against the oracle, each at its own position
    k = inp.k.cpu()
    v = inp.v.cpu() if inp.v is not None else None
    orc = oracle.get()
    for t in prompt_samples(T, spec.window, 5500 + len(kind)):
        o_ref, l_ref = orc.decode(q[t], k, v, torch.tensor([t + 1], dtype=torch.int32),
                                  spec.window, spec.softcap, spec.scale)
        compare(out[t], lse[t], o_ref, l_ref, ulp_floor=True, what=f"{kind} prompt token {t}")
