"""gdattn_decode_noalloc: gdattn_decode with its split-KV scratch in a fixed
device array inside the library (a library addition with no counterpart in the
pages).  Its results must be bit-identical to gdattn_decode's, whatever the
previous call left in the shared scratch.

This file sorts last so that its GPU tests also run after everything else in
one process; they pass on their own too.
"""
from __future__ import annotations

import pytest
import torch

import workloads
from decode_attention_09_b200 import binding
from gpu_helpers import require_gpu

A = 1 << 20  # a 16-byte aligned non-null address; host checks never dereference it


def sliding_desc(**kw):
    d = dict(n_q_heads=16, n_kv_heads=8, head_dim=256, window=1024, softcap=0.0,
             scale=1 / 16, kv_shared=False, cache_capacity=1024)
    d.update(kw)
    return binding.make_desc(**d)


def call(desc, q=A, k=A, v=A, seqlens=A, batch=1, max_seqlen=8, out=A, lse=A):
    return binding.decode_noalloc_raw(q, k, v, seqlens, batch, max_seqlen, desc, out, lse, None)


# ---------------------------------------------------------------- host checks
@pytest.mark.parametrize("case,expect", [
    (dict(q=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(k=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(seqlens=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(out=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(v=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(batch=0), binding.GDATTN_ERR_INVALID_ARG),
    (dict(max_seqlen=-3), binding.GDATTN_ERR_INVALID_ARG),
    (dict(q=A + 8), binding.GDATTN_ERR_MISALIGNED),
    (dict(v=A + 4), binding.GDATTN_ERR_MISALIGNED),
    (dict(lse=A + 2), binding.GDATTN_ERR_MISALIGNED),
])
def test_noalloc_host_checks(case, expect):
    """The same argument checks as gdattn_decode, made before any CUDA call."""
    binding.lib()
    assert call(sliding_desc(), **case) == expect


@pytest.mark.parametrize("desc_kw,expect", [
    (dict(n_q_heads=12), binding.GDATTN_ERR_INVALID_ARG),
    (dict(softcap=float("nan")), binding.GDATTN_ERR_INVALID_ARG),
    (dict(head_dim=128), binding.GDATTN_ERR_UNSUPPORTED),
])
def test_noalloc_rejects_bad_desc(desc_kw, expect):
    binding.lib()
    assert call(sliding_desc(**desc_kw)) == expect


def test_scratch_size_constant_matches_header():
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "include", "gdattn.h")).read()
    m = re.search(r"#define GDATTN_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", hdr)
    assert m and int(m.group(1)) << int(m.group(2)) == binding.NOALLOC_SCRATCH_BYTES


# ------------------------------------------------------------------ GPU tests
def _layers():
    """Two sliding (tcgen05 pair kernel) and two global (tcgen05 16-head kernel)
    inputs; each pair differs in seed and lengths, so stale scratch would change
    results."""
    core = [
        (workloads.random_case(901, 4, 16, 8, 256, 1024, [1500, 700, 1, 4096], window=1024), 0),
        (workloads.random_case(902, 4, 16, 8, 256, 1024, [333, 4000, 1024, 90], window=1024), 37),
    ]
    tc = [
        (workloads.random_case(903, 3, 16, 1, 512, 4096, [4096, 1234, 65], window=0,
                               kv_shared=True), 0),
        (workloads.random_case(904, 3, 16, 1, 512, 4096, [17, 3000, 4000], window=0,
                               kv_shared=True, softcap=30.0), 11),
    ]
    return [core[0], tc[0], core[1], tc[1]]


class Dev:
    def __init__(self, inp, split):
        self.q = inp.q.cuda()
        self.k = inp.k.cuda()
        self.v = inp.v.cuda() if inp.v is not None else None
        self.seqlens = inp.seqlens.to(device="cuda", dtype=torch.int32)
        self.B = inp.q.shape[0]
        self.max_seqlen = int(inp.seqlens.max())
        self.desc = binding.desc_from_spec(inp.spec, split, capacity=inp.k.shape[1])
        assert binding.workspace_size(self.B, self.max_seqlen, self.desc) <= \
            binding.NOALLOC_SCRATCH_BYTES

    def outputs(self):
        return (torch.full_like(self.q, float("nan")),
                torch.full((self.B, self.q.shape[1]), float("nan"), device="cuda"))

    def with_workspace(self):
        out, lse = self.outputs()
        ws = binding.alloc_workspace(self.B, self.max_seqlen, self.desc)
        binding.decode(self.q, self.k, self.v, self.seqlens, self.desc, self.max_seqlen, out=out,
                       lse=lse, workspace=ws)
        assert binding.check_device_status(ws) == binding.GDATTN_OK
        return out, lse

    def noalloc(self, out, lse, stream=None):
        binding.decode_noalloc(self.q, self.k, self.v, self.seqlens, self.desc, self.max_seqlen,
                               out, lse, stream=stream)


def assert_same(a, b, what):
    ao, al = a
    bo, bl = b
    assert torch.equal(ao.view(torch.int16), bo.view(torch.int16)), f"{what}: out differs"
    assert torch.equal(al.view(torch.int32), bl.view(torch.int32)), f"{what}: lse differs"


@pytest.mark.gpu
def test_noalloc_matches_workspace_decode_on_consecutive_calls():
    """Back-to-back calls on one stream, alternating the two kernels' scratch
    layouts, equal gdattn_decode bit for bit; then the same sequence again."""
    require_gpu()
    layers = [Dev(inp, split) for inp, split in _layers()]
    ref = [ly.with_workspace() for ly in layers]
    for rep in range(2):
        got = [ly.outputs() for ly in layers]
        for ly, (o, l) in zip(layers, got):
            ly.noalloc(o, l)  # no synchronisation between the calls
        torch.cuda.synchronize()
        assert binding.check_device_status(None) == binding.GDATTN_OK
        for i, (g, r) in enumerate(zip(got, ref)):
            assert_same(g, r, f"pass {rep} layer {i}")


@pytest.mark.gpu
def test_noalloc_rejects_oversize_and_enqueues_nothing():
    require_gpu()
    inp, _ = _layers()[1]
    ly = Dev(inp, 0)
    big = binding.desc_from_spec(inp.spec, 4000, capacity=inp.k.shape[1])
    assert binding.workspace_size(ly.B, ly.max_seqlen, big) > binding.NOALLOC_SCRATCH_BYTES
    out, lse = ly.outputs()
    st = binding.decode_noalloc_raw(binding._ptr(ly.q), binding._ptr(ly.k), None,
                                    binding._ptr(ly.seqlens), ly.B, ly.max_seqlen, big,
                                    binding._ptr(out), binding._ptr(lse), None)
    assert st == binding.GDATTN_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.isnan(out.float()).all() and torch.isnan(lse).all()


@pytest.mark.gpu
def test_noalloc_calls_take_no_device_memory():
    """After a first call, further calls leave the device's free memory as it was."""
    require_gpu()
    layers = [Dev(inp, split) for inp, split in _layers()]
    bufs = [ly.outputs() for ly in layers]
    for ly, (o, l) in zip(layers, bufs):
        ly.noalloc(o, l)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        for ly, (o, l) in zip(layers, bufs):
            ly.noalloc(o, l)
    torch.cuda.synchronize()
    assert binding.check_device_status(None) == binding.GDATTN_OK
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


@pytest.mark.gpu
def test_noalloc_status_word_latches_and_clears():
    """A device-side error lands in the fixed scratch's status word."""
    require_gpu()
    inp = workloads.random_case(905, 3, 16, 8, 256, 32, [5, 0, 9], window=16)
    ly = Dev(inp, 0)
    ly.max_seqlen = 16
    out, lse = ly.outputs()
    assert binding.check_device_status(None) == binding.GDATTN_OK
    ly.noalloc(out, lse)
    assert binding.check_device_status(None) == binding.GDATTN_ERR_DEVICE_SEQLEN
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
    assert binding.check_device_status(None) == binding.GDATTN_OK


@pytest.mark.gpu
def test_noalloc_graph_replay_matches_workspace_decode():
    require_gpu()
    layers = [Dev(inp, split) for inp, split in _layers()]
    ref = [ly.with_workspace() for ly in layers]
    bufs = [ly.outputs() for ly in layers]
    layers[0].noalloc(*bufs[0])  # first call on the device outside capture
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for ly, (o, l) in zip(layers, bufs):
                ly.noalloc(o, l, stream=s)
    for _ in range(2):
        for o, l in bufs:
            o.fill_(float("nan"))
            l.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for i, (b, r) in enumerate(zip(bufs, ref)):
            assert_same(b, r, f"graph layer {i}")
    assert binding.check_device_status(None) == binding.GDATTN_OK
    del g


@pytest.mark.gpu
def test_noalloc_even_split_matches_workspace_decode():
    """With the even unit split the pair kernel merges tagged parts, whose
    per-unit epochs live in the fixed scratch between calls: consecutive
    no-alloc calls equal gdattn_decode bit for bit."""
    require_gpu()
    inp = workloads.random_case(906, 4, 16, 8, 256, 512, [512, 700, 900, 512], window=512)
    ly = Dev(inp, 0)
    ly.desc = binding.desc_from_spec(inp.spec, capacity=512, flags=binding.GDATTN_FLAG_EVEN_UNITS)
    splits = binding.plan_splits(ly.B, ly.max_seqlen, ly.desc)
    assert splits // (ly.B * 8) >= 2, splits  # the unit split (tagged merge) is in use
    ref = ly.with_workspace()
    for rep in range(3):
        got = ly.outputs()
        ly.noalloc(*got)
        torch.cuda.synchronize()
        assert binding.check_device_status(None) == binding.GDATTN_OK
        assert_same(got, ref, f"even split call {rep}")


def _many_unit_layers():
    """Plans whose header use and partial areas differ widely, drawn on the GPU
    (the test compares two library paths, not the oracle): a ragged sliding
    layer of 512 units (counted merge), a global layer of 64 units (combine
    kernel, partials right after the header), and even-split sliding layers of
    136 and 512 units (tagged merge), some with soft-cap."""
    g = torch.Generator(device="cpu").manual_seed(907)
    rag = torch.randint(1, 2200, (64,), generator=g).tolist()
    specs = [
        # (seed, B, Hq, Hkv, D, C, seqlens, window, cap, shared, flags)
        (911, 64, 16, 8, 256, 1024, rag, 1024, 50.0, False, 0),
        (912, 64, 16, 1, 512, 2200, rag, 0, 0.0, True, 0),
        (913, 17, 16, 8, 256, 512, [1500] * 17, 512, 0.0, False, binding.GDATTN_FLAG_EVEN_UNITS),
        (914, 64, 16, 8, 256, 1024, [3000] * 64, 1024, 30.0, False,
         binding.GDATTN_FLAG_EVEN_UNITS),
        (915, 64, 16, 1, 512, 1024, [1024] * 64, 0, 0.0, True, binding.GDATTN_FLAG_EVEN_UNITS),
    ]
    layers = []
    for seed, B, Hq, Hkv, D, C, sl, w, cap, shared, flags in specs:
        inp = workloads.random_case(seed, B, Hq, Hkv, D, C, sl, window=w, softcap=cap,
                                    kv_shared=shared, device="cuda")
        ly = Dev(inp, 0)
        ly.desc = binding.desc_from_spec(inp.spec, capacity=C, flags=flags)
        layers.append(ly)
    return layers


@pytest.mark.gpu
def test_noalloc_alternating_plans_with_many_units():
    """Layouts whose unit counts exceed 64 take turns on the fixed scratch, in
    both orders, twice: every call equals gdattn_decode bit for bit and no
    device-side error is latched.  (Counters and epochs sit at fixed offsets,
    so no plan's partials land on another plan's counters.)"""
    require_gpu()
    layers = _many_unit_layers()
    for ly in layers:
        assert binding.workspace_size(ly.B, ly.max_seqlen, ly.desc) <= \
            binding.NOALLOC_SCRATCH_BYTES
    ref = [ly.with_workspace() for ly in layers]
    order = list(range(len(layers)))
    for rep, seq in enumerate([order, order[::-1], order, [0, 2, 0, 3, 1, 3, 2]]):
        for i in seq:
            got = layers[i].outputs()
            layers[i].noalloc(*got)  # no synchronisation between the calls
            torch.cuda.synchronize()
            assert binding.check_device_status(None) == binding.GDATTN_OK, (rep, i)
            assert_same(got, ref[i], f"sequence {rep} layer {i}")


_FIRST_CALL_CAPTURED = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
import workloads
from decode_attention_09_b200 import binding
inp = workloads.random_case(921, 2, 16, 8, 256, 128, [128, 77], window=128, device="cuda")
desc = binding.desc_from_spec(inp.spec, capacity=128)
out = torch.empty_like(inp.q)
lse = torch.empty(inp.q.shape[:2], device="cuda")
args = lambda s: (binding._ptr(inp.q), binding._ptr(inp.k), binding._ptr(inp.v),
                  binding._ptr(inp.seqlens), 2, 128, desc, binding._ptr(out), binding._ptr(lse), s)
torch.cuda.synchronize()
s = torch.cuda.Stream()
g = torch.cuda.CUDAGraph()
with torch.cuda.stream(s):
    with torch.cuda.graph(g, stream=s):
        st_captured = binding.decode_noalloc_raw(*args(s.cuda_stream))
st_eager = binding.decode_noalloc_raw(*args(None))
torch.cuda.synchronize()
ref_out, ref_lse = binding.decode(inp.q, inp.k, inp.v, inp.seqlens, desc, 128)
torch.cuda.synchronize()
same = torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
print(st_captured, st_eager, binding.check_device_status(None), int(same))
"""


@pytest.mark.gpu
def test_noalloc_first_call_refused_under_capture():
    """In a fresh process (so the call really is the context's first), a first
    call made while its stream is capturing returns GDATTN_ERR_INVALID_ARG and
    enqueues nothing; the next, eager call sets the scratch up and computes
    gdattn_decode's result."""
    require_gpu()
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _FIRST_CALL_CAPTURED, root], capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    st_cap, st_eager, st_dev, same = (int(x) for x in r.stdout.split()[-4:])
    assert st_cap == binding.GDATTN_ERR_INVALID_ARG
    assert st_eager == binding.GDATTN_OK and st_dev == binding.GDATTN_OK and same == 1
