"""Shared helpers for the GPU tests: run one layer through the C ABI and compare
with the float64 oracle on the very same bf16 inputs."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from decode_attention_09_b200 import binding

OUT_TOL = 8e-3  # max |out_gpu - out_oracle|, bf16 output
LSE_TOL = 1e-3  # max |lse_gpu - lse_oracle|, fp32


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def uses_tensor_cores(spec) -> bool:
    """Whether the library runs this geometry on its tcgen05 kernels: 8 or 16
    query heads per KV head with head_dim 512 (K = V or a separate V), or pairs
    of query heads with head_dim 256 and separate V.  Other geometries take the
    CUDA-core kernel."""
    g = spec.n_q_heads // spec.n_kv_heads
    return ((g in (8, 16) and spec.head_dim == 512)
            or (g == 2 and spec.head_dim == 256 and not spec.kv_shared))


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(ax)) - 7)


GUARD_BYTES = 4096
GUARD_BYTE = 0xA5


class Guarded:
    """A device tensor with GUARD_BYTES of a known byte pattern on each side, so
    a kernel that writes past either end of it is caught (``check``).  Write-side
    bounds checks in place of a memory checker."""

    _all = []

    def __init__(self, shape, dtype, device="cuda", fill=None):
        n = 1
        for d in shape:
            n *= int(d)
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((GUARD_BYTES + nbytes + GUARD_BYTES,), GUARD_BYTE, dtype=torch.uint8,
                              device=device)
        self.nbytes = nbytes
        self.t = self.raw[GUARD_BYTES:GUARD_BYTES + nbytes].view(dtype).view(*shape)
        if fill is not None:
            self.t.fill_(fill)
        Guarded._all.append(self)

    def check(self, what=""):
        lo = self.raw[:GUARD_BYTES]
        hi = self.raw[GUARD_BYTES + self.nbytes:]
        bad_lo = int((lo != GUARD_BYTE).sum())
        bad_hi = int((hi != GUARD_BYTE).sum())
        assert bad_lo == 0 and bad_hi == 0, (
            f"{what}: {bad_lo} bytes written before and {bad_hi} bytes after the buffer")


def guarded_workspace(B, max_seqlen, desc, device="cuda"):
    n = binding.workspace_size(B, max_seqlen, desc)
    assert n > 0
    ws = Guarded((n,), torch.uint8, device)
    binding.workspace_init(ws.t)
    return ws


class GpuLayer:
    """Device copies of a layer's inputs plus a workspace.  The outputs, the LSE
    and the workspace sit between guard bytes that every run checks."""

    def __init__(self, inp, split_ctas=0, max_seqlen=None, device="cuda"):
        self.inp = inp
        self.device = device
        self.q = inp.q.to(device)
        self.k = inp.k.to(device)
        self.v = inp.v.to(device) if inp.v is not None else None
        self.seqlens = inp.seqlens.to(device=device, dtype=torch.int32)
        self.B = inp.q.shape[0]
        self.max_seqlen = int(max_seqlen or int(inp.seqlens.max()))
        self.desc = binding.desc_from_spec(inp.spec, split_ctas, capacity=inp.k.shape[1])
        self._ws = None
        self.ws = None  # set below; replaced by tests that share workspaces
        self._guard_ws = guarded_workspace(self.B, self.max_seqlen, self.desc, device)
        self.ws = self._guard_ws.t
        self._out = Guarded(tuple(self.q.shape), torch.bfloat16, device)
        self._lse = Guarded((self.B, self.q.shape[1]), torch.float32, device)

    def set_desc(self, desc):
        """Use another descriptor (and a fresh guarded workspace sized for it)."""
        self.desc = desc
        self._guard_ws = guarded_workspace(self.B, self.max_seqlen, desc, self.device)
        self.ws = self._guard_ws.t

    def run(self, check_status=True):
        out, lse = self._out.t, self._lse.t
        binding.decode(self.q, self.k, self.v, self.seqlens, self.desc, self.max_seqlen, out=out,
                       lse=lse, workspace=self.ws)
        if check_status:
            st = binding.check_device_status(self.ws)
            assert st == binding.GDATTN_OK, binding.status_string(st)
        torch.cuda.synchronize()
        self._out.check("out")
        self._lse.check("lse")
        if self.ws is self._guard_ws.t:
            self._guard_ws.check("workspace")
        return out.clone(), lse.clone()


def compare(out_gpu, lse_gpu, out_ref, lse_ref, ulp_floor=False, what=""):
    """Element-wise parity: |dout| <= 8e-3 (or 1 bf16 ulp of the reference when
    ``ulp_floor``) and |dlse| <= 1e-3."""
    og = out_gpu.float().cpu().numpy().astype(np.float64)
    lg = lse_gpu.float().cpu().numpy().astype(np.float64)
    assert og.shape == out_ref.shape and lg.shape == lse_ref.shape
    assert np.all(np.isfinite(og)), f"{what}: non-finite output"
    tol = OUT_TOL
    if ulp_floor:
        tol = np.maximum(OUT_TOL, bf16_ulp(out_ref))
    err = np.abs(og - out_ref)
    bad = err > tol
    assert not bad.any(), (f"{what}: {bad.sum()} outputs off, max |d| = {err.max():.3e} at "
                           f"{np.unravel_index(err.argmax(), err.shape)}")
    lerr = np.abs(lg - lse_ref)
    assert lerr.max() <= LSE_TOL, f"{what}: max |dlse| = {lerr.max():.3e}"
    return float(err.max()), float(lerr.max())


def oracle_for(inp, batch_index=None):
    """Oracle result for all sequences, or for the listed ones."""
    orc = oracle.get()
    s = inp.spec
    if batch_index is None:
        return orc.decode(inp.q, inp.k, inp.v, inp.seqlens, s.window, s.softcap, s.scale)
    idx = torch.as_tensor(batch_index, dtype=torch.long)
    q = inp.q.index_select(0, idx.to(inp.q.device)).cpu()
    k = inp.k.index_select(0, idx.to(inp.k.device)).cpu()
    v = inp.v.index_select(0, idx.to(inp.v.device)).cpu() if inp.v is not None else None
    sl = inp.seqlens.cpu().index_select(0, idx)
    return orc.decode(q, k, v, sl, s.window, s.softcap, s.scale)


def oracle_per_sequence(inp, batch_index=None, workers=None):
    """Oracle result for the listed sequences (all by default), one oracle call
    per sequence spread over the host cores: the C oracle releases the GIL, so
    threads run it in parallel.  Each sequence's inputs are copied to the host
    first (in this thread).  Returns (out [n,Hq,D], lse [n,Hq]) float64 in the
    order of ``batch_index``."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    orc = oracle.get()
    s = inp.spec
    picks = list(range(inp.q.shape[0])) if batch_index is None else list(batch_index)
    jobs = []
    for b in picks:
        q = inp.q[b:b + 1].cpu()
        k = inp.k[b:b + 1].cpu()
        v = inp.v[b:b + 1].cpu() if inp.v is not None else None
        sl = inp.seqlens[b:b + 1].cpu()
        jobs.append((q, k, v, sl))
    n = workers or max(1, min(len(jobs), len(os.sched_getaffinity(0))))
    with ThreadPoolExecutor(max_workers=n) as ex:
        res = list(ex.map(lambda a: orc.decode(a[0], a[1], a[2], a[3], s.window, s.softcap,
                                               s.scale), jobs))
    return (np.concatenate([r[0] for r in res], axis=0),
            np.concatenate([r[1] for r in res], axis=0))
