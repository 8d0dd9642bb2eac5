"""Pins for the float64 oracle: facts fixed by the mathematics, not by the oracle.

Each pin takes an ``oracle.Oracle`` and raises AssertionError when the oracle
disagrees with what the definition of decode attention forces.  The same pins run
against the real oracle (must all pass) and against variants with one planted
mistake (each must fail at least one), so a pin set that cannot tell a wrong
window, GQA map, scale, soft-cap order, log base, normalisation, value tensor or
ring index from the right one fails the test suite.

Independent references used here:
  * ``brute_force`` -- a second restatement in vectorised numpy: gathers the
    attended cache rows by slot, forms the score vector with a matrix product and
    normalises with scipy's logsumexp.  No code is shared with oracle.c.
  * torch's scaled_dot_product_attention in float64 with an explicit boolean
    mask over cache slots (library routine; soft-cap off).
  * closed forms and invariants of softmax attention.
"""
from __future__ import annotations

import math

import numpy as np
import torch
from scipy.special import logsumexp

import workloads

RTOL_EXACT = 1e-12


# --------------------------------------------------------------------------
# Independent brute force
# --------------------------------------------------------------------------


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def brute_force(q, k, v, seqlens, window, softcap, scale):
    """Decode attention by gathering rows and taking a softmax (numpy, float64)."""
    qf, kf = _f64(q), _f64(k)
    vf = kf if v is None else _f64(v)
    B, Hq, D = qf.shape
    _, C, Hkv, _ = kf.shape
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        L = int(seqlens[b])
        first = L - min(L, window) if window > 0 else 0
        slots = np.arange(first, L) % C
        for kv in range(Hkv):
            Ksel = kf[b, slots, kv, :]  # [n, D]
            Vsel = vf[b, slots, kv, :]
            heads = np.arange(kv * G, (kv + 1) * G)
            x = scale * (qf[b, heads, :] @ Ksel.T)  # [G, n]
            s = softcap * np.tanh(x / softcap) if softcap > 0 else x
            ls = logsumexp(s, axis=1)  # [G]
            w = np.exp(s - ls[:, None])
            out[b, heads, :] = w @ Vsel
            lse[b, heads] = ls
    return out, lse


def sdpa_reference(q, k, v, seqlens, window, scale):
    """torch SDPA in float64 with a boolean slot mask (soft-cap off)."""
    B, Hq, D = q.shape
    _, C, Hkv, _ = k.shape
    G = Hq // Hkv
    kk = k.to(torch.float64).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)  # [B,Hq,C,D]
    vv = (k if v is None else v).to(torch.float64).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    mask = torch.zeros((B, 1, 1, C), dtype=torch.bool)
    for b in range(B):
        L = int(seqlens[b])
        first = L - min(L, window) if window > 0 else 0
        for p in range(first, L):
            mask[b, 0, 0, p % C] = True
    o = torch.nn.functional.scaled_dot_product_attention(
        q.to(torch.float64).unsqueeze(2), kk, vv, attn_mask=mask, scale=scale)
    return o.squeeze(2).numpy()


def _close(a, b, tol, what):
    a = np.asarray(a)
    b = np.asarray(b)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert np.all(np.isfinite(a) == np.isfinite(b)), f"{what}: finiteness differs"
    fin = np.isfinite(a)
    err = np.max(np.abs(a[fin] - b[fin])) if fin.any() else 0.0
    assert err <= tol, f"{what}: max |diff| = {err:.3e} > {tol:.1e}"


# --------------------------------------------------------------------------
# Case grid
# --------------------------------------------------------------------------

# (B, Hq, Hkv, D, C, seqlens, window, softcap, kv_shared)
SMALL_CASES = [
    (1, 2, 1, 8, 40, [40], 0, 0.0, False),
    (2, 4, 2, 8, 40, [17, 40], 0, 0.0, False),
    (2, 4, 2, 16, 12, [37, 12], 12, 0.0, False),  # ring wraps, window = capacity
    (2, 4, 2, 16, 16, [39, 5], 9, 0.0, False),  # ring wraps, window < capacity
    (1, 16, 1, 16, 30, [30], 0, 0.0, True),  # K serves as V
    (2, 16, 1, 512, 24, [24, 11], 0, 0.0, True),
    (2, 16, 8, 256, 10, [33, 7], 10, 50.0, False),
    (1, 4, 1, 8, 40, [40], 6, 2.0, True),  # strong soft-cap
    (2, 8, 2, 8, 20, [20, 3], 0, 5.0, False),
]


def case_inputs(i, case):
    B, Hq, Hkv, D, C, sl, w, cap, shared = case
    inp = workloads.random_case(1000 + i, B, Hq, Hkv, D, C, sl, window=w, softcap=cap,
                                kv_shared=shared)
    return inp


# --------------------------------------------------------------------------
# Pins
# --------------------------------------------------------------------------


def pin_brute_force(orc):
    """Oracle == independent numpy restatement on tiny inputs (1e-12)."""
    for i, case in enumerate(SMALL_CASES):
        inp = case_inputs(i, case)
        s = inp.spec
        o1, l1 = orc.decode(inp.q, inp.k, inp.v, inp.seqlens, s.window, s.softcap, s.scale)
        o2, l2 = brute_force(inp.q, inp.k, inp.v, inp.seqlens.numpy(), s.window, s.softcap,
                             s.scale)
        _close(o1, o2, 1e-12, f"brute force out, case {i}")
        _close(l1, l2, 1e-12, f"brute force lse, case {i}")


def pin_sdpa(orc):
    """Oracle == torch float64 scaled_dot_product_attention with a slot mask (soft-cap off)."""
    for i, case in enumerate(SMALL_CASES):
        if case[7] > 0:
            continue
        inp = case_inputs(i, case)
        s = inp.spec
        o1, _ = orc.decode(inp.q, inp.k, inp.v, inp.seqlens, s.window, 0.0, s.scale)
        o2 = sdpa_reference(inp.q, inp.k, inp.v, inp.seqlens.numpy(), s.window, s.scale)
        _close(o1, o2, 1e-10, f"sdpa out, case {i}")


def pin_window_covers_context(orc):
    """A window at least as long as the context equals global attention."""
    inp = workloads.random_case(7, 2, 4, 2, 16, 40, [40, 23], window=0)
    s = inp.spec
    og, lg = orc.decode(inp.q, inp.k, inp.v, inp.seqlens, 0, 0.0, s.scale)
    for w in (40, 41, 1000):
        ow, lw = orc.decode(inp.q, inp.k, inp.v, inp.seqlens, w, 0.0, s.scale)
        _close(ow, og, RTOL_EXACT, f"window {w} vs global out")
        _close(lw, lg, RTOL_EXACT, f"window {w} vs global lse")


def pin_cap_to_infinity(orc):
    """cap -> infinity equals no cap."""
    inp = workloads.random_case(8, 2, 4, 2, 16, 24, [24, 9], window=0)
    s = inp.spec
    o0, l0 = orc.decode(inp.q, inp.k, inp.v, inp.seqlens, 0, 0.0, s.scale)
    o1, l1 = orc.decode(inp.q, inp.k, inp.v, inp.seqlens, 0, 1e30, s.scale)
    _close(o1, o0, RTOL_EXACT, "cap 1e30 out")
    _close(l1, l0, RTOL_EXACT, "cap 1e30 lse")


def pin_identical_keys(orc):
    """All attended keys equal: out = mean of V over the range, LSE = s + ln n."""
    B, Hq, Hkv, D, C = 1, 4, 2, 16, 32
    inp = workloads.random_case(9, B, Hq, Hkv, D, C, [30], window=11)
    k = inp.k.clone()
    k[:, :, :, :] = k[:, 0:1, :, :]  # every slot holds the same key row
    s = inp.spec
    for cap in (0.0, 3.0):
        o, l = orc.decode(inp.q, k, inp.v, inp.seqlens, 11, cap, s.scale)
        slots = np.arange(30 - 11, 30) % C
        vf = inp.v.to(torch.float64).numpy()[0]
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            mean_v = vf[slots, kv, :].mean(axis=0)
            _close(o[0, h], mean_v, 1e-12, f"identical keys out h{h}")
            x = s.scale * float(np.dot(inp.q[0, h].to(torch.float64).numpy(),
                                       k[0, 0, kv].to(torch.float64).numpy()))
            sc = cap * math.tanh(x / cap) if cap > 0 else x
            _close(l[0, h], sc + math.log(11), 1e-12, f"identical keys lse h{h}")


def pin_zero_query(orc):
    """q = 0: uniform weights, out = mean of V, LSE = ln n (any cap, any scale)."""
    inp = workloads.random_case(10, 2, 8, 4, 8, 16, [16, 5], window=7, softcap=5.0)
    q = torch.zeros_like(inp.q)
    o, l = orc.decode(q, inp.k, inp.v, inp.seqlens, 7, 5.0, 0.37)
    vf = inp.v.to(torch.float64).numpy()
    for b, L in enumerate([16, 5]):
        n = min(L, 7)
        slots = np.arange(L - n, L) % 16
        for h in range(8):
            _close(o[b, h], vf[b, slots, h // 2, :].mean(axis=0), 1e-12, "zero q out")
            _close(l[b, h], math.log(n), 1e-12, "zero q lse")


def pin_single_position(orc):
    """L = 1: out = v_0 exactly and LSE = s_0."""
    inp = workloads.random_case(11, 2, 4, 1, 16, 8, [1, 1], window=3, kv_shared=False)
    o, l = orc.decode(inp.q, inp.k, inp.v, inp.seqlens, 3, 0.0, 0.25)
    vf = inp.v.to(torch.float64).numpy()
    for b in range(2):
        for h in range(4):
            _close(o[b, h], vf[b, 0, 0, :], 0.0, "L=1 out")


def pin_two_positions(orc):
    """Two positions: out = sigmoid(s0 - s1) v0 + sigmoid(s1 - s0) v1."""
    inp = workloads.random_case(12, 1, 2, 1, 16, 4, [2], window=0, softcap=0.0)
    scale = 0.5
    o, l = orc.decode(inp.q, inp.k, inp.v, inp.seqlens, 0, 0.0, scale)
    qf = inp.q.to(torch.float64).numpy()[0]
    kf = inp.k.to(torch.float64).numpy()[0, :, 0, :]
    vf = inp.v.to(torch.float64).numpy()[0, :, 0, :]
    for h in range(2):
        s0, s1 = scale * qf[h] @ kf[0], scale * qf[h] @ kf[1]
        sig = 1.0 / (1.0 + math.exp(-(s0 - s1)))
        _close(o[0, h], sig * vf[0] + (1 - sig) * vf[1], 1e-12, "two positions out")
        _close(l[0, h], max(s0, s1) + math.log1p(math.exp(-abs(s0 - s1))), 1e-12,
               "two positions lse")


def pin_softcap_bound(orc):
    """Soft-capped logits lie in (-cap, cap), so ln n - cap < LSE < ln n + cap."""
    inp = workloads.random_case(13, 2, 4, 2, 16, 32, [32, 20], window=0)
    q = (inp.q.float() * 40).to(torch.bfloat16)  # large logits
    for cap in (0.5, 2.0):
        _, l = orc.decode(q, inp.k, inp.v, inp.seqlens, 0, cap, 1.0)
        for b, L in enumerate([32, 20]):
            assert np.all(l[b] < math.log(L) + cap) and np.all(l[b] > math.log(L) - cap), \
                "soft-cap bound violated"


def pin_sliding_ignores_old_positions(orc):
    """A sliding layer's output depends only on the last w positions: poison the rest."""
    B, Hq, Hkv, D, C, w = 2, 4, 2, 16, 40, 9
    inp = workloads.random_case(14, B, Hq, Hkv, D, C, [40, 25], window=w)
    o0, l0 = orc.decode(inp.q, inp.k, inp.v, inp.seqlens, w, 0.0, inp.spec.scale)
    k = inp.k.clone()
    v = inp.v.clone()
    for b, L in enumerate([40, 25]):
        k[b, : L - w] = float("nan")
        v[b, : L - w] = float("nan")
        k[b, L:] = float("nan")
        v[b, L:] = float("nan")
    o1, l1 = orc.decode(inp.q, k, v, inp.seqlens, w, 0.0, inp.spec.scale)
    _close(o1, o0, 0.0, "poisoned old positions out")
    _close(l1, l0, 0.0, "poisoned old positions lse")


def pin_ring_equals_linear(orc):
    """A ring cache (slot = pos mod C) gives the same result as a linear cache."""
    B, Hq, Hkv, D, w = 1, 4, 2, 16, 8
    for L in (8, 13, 21, 24):
        lin = workloads.random_case(15 + L, B, Hq, Hkv, D, L, [L], window=w)
        ring_k = torch.zeros((B, w, Hkv, D), dtype=torch.bfloat16)
        ring_v = torch.zeros((B, w, Hkv, D), dtype=torch.bfloat16)
        for p in range(L - w, L):
            ring_k[:, p % w] = lin.k[:, p]
            ring_v[:, p % w] = lin.v[:, p]
        o_lin, l_lin = orc.decode(lin.q, lin.k, lin.v, lin.seqlens, w, 0.0, lin.spec.scale)
        o_ring, l_ring = orc.decode(lin.q, ring_k, ring_v, lin.seqlens, w, 0.0, lin.spec.scale)
        _close(o_ring, o_lin, 1e-14, f"ring vs linear out L={L}")
        _close(l_ring, l_lin, 1e-14, f"ring vs linear lse L={L}")


def pin_split_recombine(orc):
    """Any partition of the position range, recombined by LSE, equals one pass."""
    B, Hq, Hkv, D, C = 2, 4, 2, 16, 64
    inp = workloads.random_case(16, B, Hq, Hkv, D, C, [64, 50], window=0, softcap=7.0)
    s = inp.spec
    full_o, full_l = orc.decode(inp.q, inp.k, inp.v, inp.seqlens, 0, s.softcap, s.scale)
    rng = np.random.default_rng(0)
    for trial in range(4):
        parts_o, parts_l = [], []
        cuts = [sorted(set([0, L] + list(rng.integers(0, L, size=trial + 1)))) for L in (64, 50)]
        n_parts = max(len(c) - 1 for c in cuts) + 1  # +1: an empty part
        for p in range(n_parts):
            lo = [c[p] if p < len(c) - 1 else c[-1] for c in cuts]
            hi = [c[p + 1] if p < len(c) - 1 else c[-1] for c in cuts]
            o, l = orc.attend(inp.q, inp.k, inp.v, lo, hi, s.softcap, s.scale)
            parts_o.append(o)
            parts_l.append(l)
        po = np.stack(parts_o, axis=2)  # [B,Hq,S,D]
        pl = np.stack(parts_l, axis=2)  # [B,Hq,S]
        co, cl = orc.combine(po, pl)
        _close(co, full_o, 1e-12, "split+combine out")
        _close(cl, full_l, 1e-12, "split+combine lse")


def pin_combine_closed_form(orc):
    """Combine of two parts: weights sigmoid(l0 - l1); LSE = logaddexp; -inf parts drop out."""
    o = np.array([[[1.0, 2.0], [3.0, -1.0], [7.0, 7.0]]])
    l = np.array([[0.3, -1.2, -np.inf]])
    co, cl = orc.combine(o, l)
    w0 = 1.0 / (1.0 + math.exp(-(0.3 + 1.2)))
    _close(co[0], w0 * o[0, 0] + (1 - w0) * o[0, 1], 1e-15, "combine closed form out")
    _close(cl[0], np.logaddexp(0.3, -1.2), 1e-15, "combine closed form lse")
    co, cl = orc.combine(np.zeros((1, 2, 2)), np.full((1, 2), -np.inf))
    assert cl[0] == -np.inf and np.all(co == 0)


def pin_separate_v(orc):
    """A separate V tensor is what gets averaged (K = V only when told so)."""
    inp = workloads.random_case(17, 1, 2, 1, 8, 6, [6], window=0)
    q = torch.zeros_like(inp.q)
    o, _ = orc.decode(q, inp.k, inp.v, inp.seqlens, 0, 0.0, 1.0)
    _close(o[0, 0], inp.v.to(torch.float64).numpy()[0, :, 0, :].mean(axis=0), 1e-12,
           "separate V mean")
    o, _ = orc.decode(q, inp.k, None, inp.seqlens, 0, 0.0, 1.0)
    _close(o[0, 0], inp.k.to(torch.float64).numpy()[0, :, 0, :].mean(axis=0), 1e-12,
           "shared K=V mean")


# --------------------------------------------------------------------------
# fp8 e4m3 caches with per-row scales
# --------------------------------------------------------------------------


def e4m3_reference(codes) -> np.ndarray:
    """Values of e4m3 codes by torch's float8_e4m3fn decoding (a library routine)."""
    t = torch.as_tensor(np.asarray(codes, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def dequantize(codes: torch.Tensor, scales: torch.Tensor) -> torch.Tensor:
    """codes [B, C, Hkv, D] e4m3, scales [B, Hkv, C] -> float64 values [B, C, Hkv, D]."""
    vals = codes.view(torch.float8_e4m3fn).to(torch.float64)
    return vals * scales.to(torch.float64).permute(0, 2, 1).unsqueeze(-1)


def pin_e4m3_codes(orc):
    """Every one of the 256 e4m3 codes decodes as torch's float8_e4m3fn does, and the
    format's landmarks hold: 1.0, the largest finite 448, the smallest normal 2^-6 and
    subnormal 2^-9, sign symmetry, NaN only at S.1111.111."""
    ref = e4m3_reference(np.arange(256))
    got = np.array([orc.e4m3_value(c) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref)), "e4m3 NaN codes differ"
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin]), "e4m3 decoding differs from float8_e4m3fn"
    landmarks = {0x38: 1.0, 0x7E: 448.0, 0x08: 2.0 ** -6, 0x01: 2.0 ** -9, 0x00: 0.0,
                 0xB8: -1.0, 0x40: 2.0, 0x3C: 1.5}
    for code, val in landmarks.items():
        assert orc.e4m3_value(code) == val, f"e4m3 code {code:#04x}"
    assert np.isnan(orc.e4m3_value(0x7F)) and np.isnan(orc.e4m3_value(0xFF))


# (B, Hq, Hkv, D, C, seqlens, window, softcap, kv_shared)
FP8_CASES = [
    (2, 4, 2, 16, 12, [37, 12], 12, 0.0, False),  # ring wraps
    (2, 16, 8, 32, 10, [33, 7], 10, 30.0, False),
    (1, 16, 1, 32, 30, [30], 0, 0.0, True),  # K serves as V
    (2, 4, 2, 8, 20, [20, 3], 0, 5.0, False),
]


def pin_fp8_equals_bf16_when_exact(orc):
    """With power-of-two row scales every value code * scale is a bf16 number, so
    the fp8 decode must equal the (separately pinned) bf16 decode of those values,
    exactly.  K and V scales differ and vary per (sequence, head, slot)."""
    for i, (B, Hq, Hkv, D, C, sl, w, cap, shared) in enumerate(FP8_CASES):
        inp = workloads.random_fp8_case(2000 + i, B, Hq, Hkv, D, C, sl, window=w, softcap=cap,
                                        kv_shared=shared)
        g = torch.Generator().manual_seed(3000 + i)
        pow2 = lambda: torch.exp2(torch.randint(-4, 5, (B, Hkv, C), generator=g).float())
        ks, vs = pow2(), pow2()
        k_bf = dequantize(inp.k_codes, ks).to(torch.bfloat16)
        assert torch.equal(k_bf.to(torch.float64), dequantize(inp.k_codes, ks)), "not exact"
        v_bf = None
        if not shared:
            v_bf = dequantize(inp.v_codes, vs).to(torch.bfloat16)
        s = inp.spec
        o1, l1 = orc.decode_fp8(inp.q, inp.k_codes, inp.v_codes if not shared else None, ks,
                                vs if not shared else None, inp.seqlens, s.window, s.softcap,
                                s.scale)
        o2, l2 = orc.decode(inp.q, k_bf, v_bf, inp.seqlens, s.window, s.softcap, s.scale)
        _close(o1, o2, 0.0, f"fp8 vs bf16 out, case {i}")
        _close(l1, l2, 0.0, f"fp8 vs bf16 lse, case {i}")


def pin_fp8_brute_force(orc):
    """fp8 decode == the numpy brute force over values dequantized with torch's e4m3
    decoding and the row scales (arbitrary float scales, soft-cap on and off)."""
    for i, (B, Hq, Hkv, D, C, sl, w, cap, shared) in enumerate(FP8_CASES):
        inp = workloads.random_fp8_case(2100 + i, B, Hq, Hkv, D, C, sl, window=w, softcap=cap,
                                        kv_shared=shared, spread=3.0)
        s = inp.spec
        o1, l1 = orc.decode_fp8(inp.q, inp.k_codes, inp.v_codes, inp.k_scale, inp.v_scale,
                                inp.seqlens, s.window, s.softcap, s.scale)
        kf = dequantize(inp.k_codes, inp.k_scale)
        vf = None if shared else dequantize(inp.v_codes, inp.v_scale)
        o2, l2 = brute_force(inp.q, kf, vf, inp.seqlens.numpy(), s.window, s.softcap, s.scale)
        _close(o1, o2, 1e-12, f"fp8 brute force out, case {i}")
        _close(l1, l2, 1e-12, f"fp8 brute force lse, case {i}")


def pin_fp8_zero_scale_row(orc):
    """A row whose scale is 0 has value 0 whatever its codes: with q = 0 the output
    is the mean of V over the attended rows, counting the zero rows as zeros."""
    inp = workloads.random_fp8_case(2200, 1, 2, 1, 8, 6, [6], window=0)
    vs = inp.v_scale.clone()
    vs[0, 0, 2] = 0.0
    vs[0, 0, 4] = 0.0
    o, l = orc.decode_fp8(torch.zeros_like(inp.q), inp.k_codes, inp.v_codes, inp.k_scale, vs,
                          inp.seqlens, 0, 0.0, 1.0)
    vf = dequantize(inp.v_codes, vs).numpy()[0, :, 0, :]
    assert np.all(vf[2] == 0) and np.all(vf[4] == 0)
    _close(o[0, 0], vf.mean(axis=0), 1e-12, "zero-scale rows out")
    _close(l[0], np.full(2, math.log(6)), 1e-12, "zero-scale rows lse")


# --------------------------------------------------------------------------
# Multi-query decode (T query tokens per sequence, causal)
# --------------------------------------------------------------------------

# (T, B, Hq, Hkv, D, C, seqlens, window, softcap, kv_shared)
MULTI_CASES = [
    (3, 2, 4, 2, 16, 12, [37, 12], 10, 0.0, False),  # ring wraps, C = w + T - 1
    (4, 2, 16, 1, 32, 40, [40, 9], 0, 0.0, True),    # whole context, K = V
    (2, 2, 4, 2, 8, 20, [20, 3], 0, 5.0, False),
]


def multi_inputs(i, case):
    T, B, Hq, Hkv, D, C, sl, w, cap, shared = case
    inp = workloads.random_case(4000 + i, B, Hq, Hkv, D, C, sl, window=w, softcap=cap,
                                kv_shared=shared)
    g = torch.Generator().manual_seed(4100 + i)
    q = torch.randn((T, B, Hq, D), generator=g).to(torch.bfloat16)
    return q, inp


def pin_multi_brute_force(orc):
    """Query t of a T-token step equals the numpy brute force at context length
    L - (T - 1 - t): it attends causally up to its own position."""
    for i, case in enumerate(MULTI_CASES):
        T = case[0]
        q, inp = multi_inputs(i, case)
        s = inp.spec
        o, l = orc.decode_multi(q, inp.k, inp.v, inp.seqlens, s.window, s.softcap, s.scale)
        for t in range(T):
            sl = inp.seqlens.numpy() - (T - 1 - t)
            o2, l2 = brute_force(q[t], inp.k, inp.v, sl, s.window, s.softcap, s.scale)
            _close(o[t], o2, 1e-12, f"multi brute force out, case {i} token {t}")
            _close(l[t], l2, 1e-12, f"multi brute force lse, case {i} token {t}")


def pin_multi_reduces_to_decode(orc):
    """T = 1 is single-token decode, and the last of T tokens sees what a single
    token at L sees (exactly)."""
    q, inp = multi_inputs(0, MULTI_CASES[0])
    s = inp.spec
    o1, l1 = orc.decode_multi(q[-1:], inp.k, inp.v, inp.seqlens, s.window, s.softcap, s.scale)
    o2, l2 = orc.decode(q[-1], inp.k, inp.v, inp.seqlens, s.window, s.softcap, s.scale)
    _close(o1[0], o2, 0.0, "T=1 out")
    _close(l1[0], l2, 0.0, "T=1 lse")
    o3, l3 = orc.decode_multi(q, inp.k, inp.v, inp.seqlens, s.window, s.softcap, s.scale)
    _close(o3[-1], o2, 0.0, "last token out")
    _close(l3[-1], l2, 0.0, "last token lse")


def pin_multi_ring_capacity(orc):
    """A ring of C slots holds positions [L - C, L): with a window w, T tokens
    need C >= w + T - 1, else the first token's oldest position is gone."""
    q, inp = multi_inputs(0, MULTI_CASES[0])  # C = 12 = w + T - 1
    s = inp.spec
    orc.decode_multi(q, inp.k, inp.v, inp.seqlens, s.window, s.softcap, s.scale)
    q4 = torch.cat([q, q[:1]], dim=0)  # T = 4 > C - w + 1
    try:
        orc.decode_multi(q4, inp.k, inp.v, inp.seqlens, s.window, s.softcap, s.scale)
    except ValueError:
        return
    raise AssertionError("a query reaching an overwritten slot was accepted")


def pin_multi_causal_sdpa(orc):
    """A whole prompt (L_b = T on a linear cache) is textbook causal attention:
    torch SDPA in float64 with a causal mask, banded for a sliding window, and
    the LSE from torch.logsumexp over the same masked scores."""
    for i, (B, Hq, Hkv, D, T, w) in enumerate(((2, 4, 2, 16, 9, 0), (1, 4, 1, 8, 12, 5))):
        inp = workloads.random_case(4200 + i, B, Hq, Hkv, D, T, [T] * B, window=w)
        s = inp.spec
        g = torch.Generator().manual_seed(4300 + i)
        q = torch.randn((T, B, Hq, D), generator=g).to(torch.bfloat16)
        o, l = orc.decode_multi(q, inp.k, inp.v, inp.seqlens, s.window, s.softcap, s.scale)
        tq = torch.arange(T)[:, None]
        j = torch.arange(T)[None, :]
        allowed = (j <= tq) & ((j > tq - w) if w > 0 else torch.ones((T, T), dtype=torch.bool))
        G = Hq // Hkv
        for b in range(B):
            Q = q[:, b].to(torch.float64).permute(1, 0, 2)                        # [Hq, T, D]
            K = inp.k[b, :T].to(torch.float64).permute(1, 0, 2).repeat_interleave(G, dim=0)
            V = inp.v[b, :T].to(torch.float64).permute(1, 0, 2).repeat_interleave(G, dim=0)
            ref = torch.nn.functional.scaled_dot_product_attention(
                Q, K, V, attn_mask=allowed, scale=s.scale)                       # [Hq, T, D]
            scores = torch.matmul(Q, K.transpose(1, 2)) * s.scale
            ref_lse = torch.logsumexp(scores.masked_fill(~allowed, -float("inf")), dim=-1)
            _close(o[:, b], ref.permute(1, 0, 2).numpy(), 1e-12, f"prompt {i} seq {b} out")
            _close(l[:, b], ref_lse.T.numpy(), 1e-12, f"prompt {i} seq {b} lse")


ALL_PINS = [pin_brute_force, pin_sdpa, pin_window_covers_context, pin_cap_to_infinity,
            pin_identical_keys, pin_zero_query, pin_single_position, pin_two_positions,
            pin_softcap_bound, pin_sliding_ignores_old_positions, pin_ring_equals_linear,
            pin_split_recombine, pin_combine_closed_form, pin_separate_v, pin_e4m3_codes,
            pin_fp8_equals_bf16_when_exact, pin_fp8_brute_force, pin_fp8_zero_scale_row,
            pin_multi_brute_force, pin_multi_reduces_to_decode, pin_multi_ring_capacity,
            pin_multi_causal_sdpa]


def failing_pins(orc):
    failed = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError) as e:
            failed.append((pin.__name__, str(e)))
    return failed
