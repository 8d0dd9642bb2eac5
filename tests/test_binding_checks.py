"""The Python binding's argument checks, on the CPU.

The C ABI receives bare addresses, so the tensor wrappers check what it cannot
see: dtype, contiguity, that each tensor reaches as far as the call reads or
writes, and the device.  Here the inputs the tests and the bench build pass those
checks (with the device check patched out, as there is no GPU), CPU tensors are
refused, and each kind of wrong argument is refused with its name before
anything is enqueued.
"""
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import workloads
from decode_attention_09_b200 import binding


@pytest.fixture
def any_device(monkeypatch):
    monkeypatch.setattr(binding, "_on", lambda t, name, device: None)


# (B, Hq, Hkv, D, C, seqlens, window, kv_shared): the three kernel families' geometries
GEOMETRIES = {
    "sliding_pair": (3, 16, 8, 256, 259, [700, 256, 4], 256, False),
    "global_kv_shared": (2, 16, 1, 512, 400, [400, 77], 0, True),
    "core_g4": (2, 8, 2, 256, 90, [90, 33], 0, False),
}


def layer(name):
    B, Hq, Hkv, D, C, sl, w, shared = GEOMETRIES[name]
    inp = workloads.random_case(3, B, Hq, Hkv, D, C, sl, window=w, kv_shared=shared)
    desc = binding.desc_from_spec(inp.spec, capacity=C)
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16)
    lse = torch.empty((B, Hq), dtype=torch.float32)
    return inp, desc, out, lse


def check_decode(inp, desc, o, l, **swap):
    a = dict(q=inp.q, k=inp.k, v=inp.v, seqlens=inp.seqlens, out=o, lse=l)
    a.update(swap)
    B = inp.q.shape[0]
    binding._check_layer(a["q"], a["k"], a["v"], a["seqlens"], a["out"], a["lse"], desc, B, B)


@pytest.mark.parametrize("name", sorted(GEOMETRIES))
def test_workload_layers_pass(any_device, name):
    inp, desc, out, lse = layer(name)
    check_decode(inp, desc, out, lse)
    check_decode(inp, desc, out, None)  # lse is optional


def test_strided_cache_within_its_storage_passes(any_device):
    """A cache whose sequences sit cache_batch_stride apart inside a larger buffer."""
    inp, _, out, lse = layer("sliding_pair")
    B, C, Hkv, D = inp.k.shape
    big = torch.zeros((B, C + 5, Hkv, D), dtype=torch.bfloat16)
    big[:, :C] = inp.k
    desc = binding.desc_from_spec(inp.spec, capacity=C)
    desc.cache_batch_stride = (C + 5) * Hkv * D
    check_decode(inp, desc, out, lse, k=big[:, :C], v=big[:, :C])


def test_multi_query_arguments_pass(any_device):
    inp, desc, _, _ = layer("global_kv_shared")
    T, (B, Hq, D) = 3, inp.q.shape
    q = torch.zeros((T, B, Hq, D), dtype=torch.bfloat16)
    out = torch.empty_like(q)
    lse = torch.empty((T, B, Hq), dtype=torch.float32)
    binding._check_layer(q, inp.k, inp.v, inp.seqlens, out, lse, desc, T * B, B)
    with pytest.raises(ValueError, match="out: .* the call reaches"):  # one token's worth only
        binding._check_layer(q, inp.k, inp.v, inp.seqlens, out[0], lse, desc, T * B, B)


def test_append_rows(any_device):
    inp, desc, _, _ = layer("sliding_pair")
    B, _, Hkv, D = inp.k.shape
    rows = torch.zeros((B, Hkv, D), dtype=torch.bfloat16)
    binding._check_new_rows(rows, rows, desc, B, None)
    binding._check_new_rows(rows, None, desc, B, None)
    with pytest.raises(ValueError, match="v_new: .* the call reaches"):
        binding._check_new_rows(rows, rows[:-1], desc, B, None)
    with pytest.raises(ValueError, match="k_new: dtype"):
        binding._check_new_rows(rows.float(), rows, desc, B, None)


def fp8_case():
    inp = workloads.random_fp8_case(5, 3, 16, 8, 256, 64, [64, 37, 5], window=64)
    desc = binding.desc_from_spec(inp.spec, capacity=64)
    B, Hq, D = inp.q.shape
    return inp, desc, torch.empty((B, Hq, D), dtype=torch.bfloat16), torch.empty((B, Hq))


def check_fp8(inp, desc, o, l, **swap):
    a = dict(q=inp.q, kc=inp.k_codes, vc=inp.v_codes, ks=inp.k_scale, vs=inp.v_scale,
             seqlens=inp.seqlens, out=o, lse=l)
    a.update(swap)
    binding._check_fp8(a["q"], a["kc"], a["vc"], a["ks"], a["vs"], a["seqlens"], a["out"],
                       a["lse"], desc, inp.q.shape[0])


def test_fp8_arguments(any_device):
    inp, desc, out, lse = fp8_case()
    check_fp8(inp, desc, out, lse)
    check_fp8(inp, desc, out, lse, kc=inp.k_codes.view(torch.float8_e4m3fn),
              vc=inp.v_codes.view(torch.float8_e4m3fn))
    with pytest.raises(ValueError, match="k_scale: .* the call reaches"):
        check_fp8(inp, desc, out, lse, ks=inp.k_scale[:, :, :-1].contiguous())
    with pytest.raises(ValueError, match="v_codes: dtype"):
        check_fp8(inp, desc, out, lse, vc=inp.v_codes.to(torch.bfloat16))
    with pytest.raises(ValueError, match="v_scale: must be contiguous"):
        check_fp8(inp, desc, out, lse, vs=inp.v_scale.transpose(1, 2))


def test_combine_arguments(any_device):
    po = torch.zeros((2, 4, 3, 256))
    pl = torch.zeros((2, 4, 3))
    out = torch.empty((2, 4, 256), dtype=torch.bfloat16)
    binding._check_combine(po, pl, out, torch.empty((2, 4)))
    with pytest.raises(ValueError, match="lse_partial: dtype"):
        binding._check_combine(po, pl.double(), out, None)
    with pytest.raises(ValueError, match="out: .* the call reaches"):
        binding._check_combine(po, pl, out[:1], None)


def wrong(name):
    """Each entry: (keyword to swap, how to spoil it, expected message)."""
    inp, desc, out, lse = layer(name)
    B, C, Hkv, D = inp.k.shape
    return [
        ("q", inp.q.float(), "q: dtype"),
        ("q", inp.q[:-1], "q: .* the call reaches"),
        ("out", out.transpose(1, 2), "out: must be contiguous"),
        ("lse", lse.flatten()[:-1], "lse: .* the call reaches"),
        ("seqlens", inp.seqlens.long(), "seqlens: dtype"),
        ("seqlens", inp.seqlens[:-1], "seqlens: .* the call reaches"),
        ("k", inp.k[1:], "k: storage holds"),
        ("k", inp.k[:, :C - 1].contiguous(), "k: storage holds"),
    ] + ([] if inp.v is None else [("v", inp.v.view(torch.int16), "v: dtype"),
                                   ("v", inp.v[:-1].clone(), "v: storage holds")])


@pytest.mark.parametrize("name", sorted(GEOMETRIES))
def test_wrong_arguments_are_refused(any_device, name):
    inp, desc, out, lse = layer(name)
    for key, bad, msg in wrong(name):
        with pytest.raises(ValueError, match=msg):
            check_decode(inp, desc, out, lse, **{key: bad})


def test_capacity_beyond_the_cache_is_refused(any_device):
    inp, desc, out, lse = layer("sliding_pair")
    desc.cache_capacity += 1
    with pytest.raises(ValueError, match="k: storage holds"):
        check_decode(inp, desc, out, lse)


def test_cpu_tensors_are_refused_before_any_call():
    """No patch: the wrappers refuse host tensors before enqueueing anything."""
    inp, desc, out, lse = layer("sliding_pair")
    with pytest.raises(ValueError, match="q: must be a CUDA tensor"):
        binding.decode(inp.q, inp.k, inp.v, inp.seqlens, desc, 700, out=out, lse=lse,
                       workspace=torch.empty(16, dtype=torch.uint8))


def test_headline_stack_layers_pass(any_device):
    """A sliding and a global layer of the 48-layer stack at batch 8, context 8192,
    with the descriptors the bench builds, and the fp8 cache of the sliding one."""
    w = workloads.gemma4_12b_b8_l8192()
    sl = w.seqlens()
    for i in (0, 5):
        spec = w.layers[i]
        assert spec.kind == ("sliding" if i == 0 else "global")
        inp = workloads.layer_inputs(spec, w.batch, sl, 1)
        desc = binding.desc_from_spec(spec, flags=binding.GDATTN_FLAG_EVEN_UNITS)
        check_decode(inp, desc, torch.empty_like(inp.q),
                     torch.empty(inp.q.shape[:2], dtype=torch.float32))
    spec = w.layers[0]
    f8 = workloads.fp8_layer_inputs(spec, w.batch, sl, 2)
    check_fp8(f8, binding.desc_from_spec(spec), torch.empty_like(f8.q),
              torch.empty(f8.q.shape[:2]))


# the fixture only patches out the device check: the same for every example
@settings(max_examples=30, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(hkv=st.sampled_from([1, 2, 4, 8]), g=st.sampled_from([1, 2, 4, 16]),
       d=st.sampled_from([256, 512]), cap=st.integers(1, 70), batch=st.integers(1, 4),
       tokens=st.integers(1, 4), shared=st.booleans(), pad=st.integers(0, 3))
def test_any_well_formed_call_passes(any_device, hkv, g, d, cap, batch, tokens, shared, pad):
    """Whatever the geometry, the tensors a caller lays out as the header says pass
    the checks, with dense caches or with sequences `pad` rows apart."""
    inp = workloads.random_case(7, batch, hkv * g, hkv, d, cap, [cap] * batch,
                                kv_shared=shared)
    desc = binding.desc_from_spec(inp.spec, capacity=cap)
    if pad:
        big = torch.zeros((batch, cap + pad, hkv, d), dtype=torch.bfloat16)
        big[:, :cap] = inp.k
        desc.cache_batch_stride = (cap + pad) * hkv * d
        k = big[:, :cap]
        v = None if shared else big[:, :cap]
    else:
        k, v = inp.k, inp.v
    out = torch.empty((batch, hkv * g, d), dtype=torch.bfloat16)
    binding._check_layer(inp.q, k, v, inp.seqlens, out, None, desc, batch, batch)
    q = torch.zeros((tokens, batch, hkv * g, d), dtype=torch.bfloat16)
    binding._check_layer(q, k, v, inp.seqlens, torch.empty_like(q),
                         torch.empty((tokens, batch, hkv * g)), desc, tokens * batch, batch)
