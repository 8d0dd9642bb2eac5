"""The oracle against the independent numpy brute force on random small geometries.

The pins fix the oracle on chosen cases; here hypothesis draws the geometry
(query and KV heads, head size, ring capacity, window, soft-cap, K = V, lengths
that wrap the ring or not, T for multi-query) and the seeds, so the agreement
holds away from the hand-picked cases too.  Derandomised: the same examples on
every run.
"""
import numpy as np
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
import workloads
from pins import _close, brute_force, dequantize

SETTINGS = settings(max_examples=40, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow])


@st.composite
def geometry(draw, with_tokens=False):
    hkv = draw(st.sampled_from([1, 2, 4]))
    g = draw(st.sampled_from([1, 2, 4, 16]))
    d = draw(st.sampled_from([4, 8, 16, 32]))
    cap = draw(st.integers(1, 48))
    sliding = draw(st.booleans())
    window = draw(st.integers(1, cap)) if sliding else 0
    tokens = draw(st.integers(1, 4)) if with_tokens else 1
    if with_tokens and sliding:
        # a ring of C slots holds [L - C, L): the first token needs w + T - 1 <= C
        window = min(window, cap - tokens + 1)
        if window < 1:
            cap, window = tokens, 1
    batch = draw(st.integers(1, 3))
    hi = 3 * cap if sliding else cap
    seqlens = [draw(st.integers(tokens, max(tokens, hi))) for _ in range(batch)]
    softcap = draw(st.sampled_from([0.0, 0.0, 2.0, 30.0]))
    shared = draw(st.booleans())
    seed = draw(st.integers(0, 2**31 - 1))
    return dict(B=batch, Hq=hkv * g, Hkv=hkv, D=d, C=cap, seqlens=seqlens, window=window,
                softcap=softcap, shared=shared, seed=seed, T=tokens)


@SETTINGS
@given(geometry())
def test_decode_matches_brute_force(gm):
    inp = workloads.random_case(gm["seed"], gm["B"], gm["Hq"], gm["Hkv"], gm["D"], gm["C"],
                                gm["seqlens"], window=gm["window"], softcap=gm["softcap"],
                                kv_shared=gm["shared"])
    s = inp.spec
    o1, l1 = oracle.get().decode(inp.q, inp.k, inp.v, inp.seqlens, s.window, s.softcap, s.scale)
    o2, l2 = brute_force(inp.q, inp.k, inp.v, inp.seqlens.numpy(), s.window, s.softcap, s.scale)
    _close(o1, o2, 1e-12, f"out {gm}")
    _close(l1, l2, 1e-12, f"lse {gm}")


@SETTINGS
@given(geometry())
def test_fp8_decode_matches_brute_force(gm):
    inp = workloads.random_fp8_case(gm["seed"], gm["B"], gm["Hq"], gm["Hkv"], gm["D"], gm["C"],
                                    gm["seqlens"], window=gm["window"], softcap=gm["softcap"],
                                    kv_shared=gm["shared"], spread=3.0)
    s = inp.spec
    o1, l1 = oracle.get().decode_fp8(inp.q, inp.k_codes, inp.v_codes, inp.k_scale,
                                     inp.v_scale, inp.seqlens, s.window, s.softcap, s.scale)
    kf = dequantize(inp.k_codes, inp.k_scale)
    vf = None if gm["shared"] else dequantize(inp.v_codes, inp.v_scale)
    o2, l2 = brute_force(inp.q, kf, vf, inp.seqlens.numpy(), s.window, s.softcap, s.scale)
    _close(o1, o2, 1e-12, f"fp8 out {gm}")
    _close(l1, l2, 1e-12, f"fp8 lse {gm}")


@SETTINGS
@given(geometry(with_tokens=True))
def test_multi_query_matches_brute_force(gm):
    inp = workloads.random_case(gm["seed"], gm["B"], gm["Hq"], gm["Hkv"], gm["D"], gm["C"],
                                gm["seqlens"], window=gm["window"], softcap=gm["softcap"],
                                kv_shared=gm["shared"])
    T = gm["T"]
    g = torch.Generator().manual_seed(gm["seed"] % 1000003)
    q = torch.randn((T, gm["B"], gm["Hq"], gm["D"]), generator=g).to(torch.bfloat16)
    s = inp.spec
    o, l = oracle.get().decode_multi(q, inp.k, inp.v, inp.seqlens, s.window, s.softcap, s.scale)
    for t in range(T):
        sl = inp.seqlens.numpy() - (T - 1 - t)
        o2, l2 = brute_force(q[t], inp.k, inp.v, sl, s.window, s.softcap, s.scale)
        _close(o[t], o2, 1e-12, f"multi out token {t} {gm}")
        _close(l[t], l2, 1e-12, f"multi lse token {t} {gm}")
    assert np.isfinite(l).all()
