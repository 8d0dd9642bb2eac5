"""Float64 CPU oracle for decode attention (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library under test never does, and it
shares no code with it.  The arithmetic lives in ``oracle.c`` (plain definition,
float64); this module only marshals arguments through ctypes.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np
import torch

from . import build as _build

_LIBS: dict = {}


class Oracle:
    """A loaded oracle library (the real one, or a planted-mistake variant)."""

    def __init__(self, path: str):
        self.path = path
        lib = ctypes.CDLL(path)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        i32p = ctypes.POINTER(ctypes.c_int32)
        f64p = ctypes.POINTER(ctypes.c_double)
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.oracle_attend.argtypes = [u16p, u16p, u16p, i32, i32, i32, i32, i32, i64, i32p, i32p,
                                      f64, f64, i32, f64p, f64p]
        lib.oracle_attend.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [u16p, u16p, u16p, i32p, i32, i32, i32, i32, i32, i64, i32,
                                      f64, f64, i32, f64p, f64p]
        lib.oracle_decode.restype = ctypes.c_int
        u8p = ctypes.POINTER(ctypes.c_uint8)
        f32p = ctypes.POINTER(ctypes.c_float)
        lib.oracle_decode_fp8.argtypes = [u16p, u8p, u8p, f32p, f32p, i32p, i32, i32, i32, i32,
                                          i32, i64, i32, f64, f64, i32, f64p, f64p]
        lib.oracle_decode_fp8.restype = ctypes.c_int
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8, f64p]
        lib.oracle_e4m3_to_double.restype = ctypes.c_int
        lib.oracle_decode_multi.argtypes = [u16p, u16p, u16p, i32p, i32, i32, i32, i32, i32, i32,
                                            i64, i32, f64, f64, i32, f64p, f64p]
        lib.oracle_decode_multi.restype = ctypes.c_int
        lib.oracle_combine.argtypes = [f64p, f64p, i32, i32, f64p, f64p]
        lib.oracle_combine.restype = None
        lib.oracle_version.restype = ctypes.c_int
        self.lib = lib

    # ---------------------------------------------------------------- helpers
    @staticmethod
    def _bits(t) -> np.ndarray:
        """bf16 torch tensor (or uint16 array of bf16 bits) -> contiguous uint16 array."""
        if isinstance(t, torch.Tensor):
            assert t.dtype == torch.bfloat16, t.dtype
            return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy()
                                        .view(np.uint16))
        a = np.ascontiguousarray(t)
        assert a.dtype == np.uint16
        return a

    @staticmethod
    def _ptr(a: np.ndarray, ctype):
        return a.ctypes.data_as(ctypes.POINTER(ctype))

    # ------------------------------------------------------------------ calls
    def decode(self, q, k, v, seqlens, window: int, softcap: float, scale: float,
               capacity: Optional[int] = None):
        """One decode-attention layer.  Returns (out [B,Hq,D] float64, lse [B,Hq] float64).

        q: bf16 [B,Hq,D]; k (v): bf16 [B,C,Hkv,D]; v=None means K serves as V.
        """
        qb, kb = self._bits(q), self._bits(k)
        B, Hq, D = qb.shape
        _, C, Hkv, Dk = kb.shape
        assert Dk == D and kb.shape[0] == B
        if capacity is not None:
            assert capacity == C
        vb = self._bits(v) if v is not None else None
        sl = np.ascontiguousarray(np.asarray(seqlens.cpu() if isinstance(seqlens, torch.Tensor)
                                             else seqlens, dtype=np.int32))
        out = np.zeros((B, Hq, D), dtype=np.float64)
        lse = np.zeros((B, Hq), dtype=np.float64)
        rc = self.lib.oracle_decode(
            self._ptr(qb, ctypes.c_uint16), self._ptr(kb, ctypes.c_uint16),
            self._ptr(vb, ctypes.c_uint16) if vb is not None else None,
            self._ptr(sl, ctypes.c_int32), B, Hq, Hkv, D, C, C * Hkv * D, int(window),
            float(softcap), float(scale), 1 if vb is None else 0,
            self._ptr(out, ctypes.c_double), self._ptr(lse, ctypes.c_double))
        if rc != 0:
            raise ValueError("oracle_decode rejected its arguments")
        return out, lse

    @staticmethod
    def _codes(t) -> np.ndarray:
        """fp8 codes (torch uint8 / float8_e4m3fn tensor or uint8 array) -> contiguous uint8."""
        if isinstance(t, torch.Tensor):
            return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.uint8).numpy())
        a = np.ascontiguousarray(t)
        assert a.dtype == np.uint8
        return a

    @staticmethod
    def _f32(t) -> np.ndarray:
        if isinstance(t, torch.Tensor):
            assert t.dtype == torch.float32, t.dtype
            return np.ascontiguousarray(t.detach().cpu().contiguous().numpy())
        return np.ascontiguousarray(np.asarray(t, dtype=np.float32))

    def e4m3_value(self, code: int) -> float:
        """The value of one e4m3 code, as the oracle decodes it."""
        v = ctypes.c_double()
        self.lib.oracle_e4m3_to_double(int(code) & 0xFF, ctypes.byref(v))
        return v.value

    def decode_fp8(self, q, k_codes, v_codes, k_scale, v_scale, seqlens, window: int,
                   softcap: float, scale: float):
        """One decode-attention layer over an fp8 cache.  Returns (out, lse) float64.

        q: bf16 [B,Hq,D]; k_codes (v_codes): e4m3 codes [B,C,Hkv,D]; k_scale (v_scale):
        float32 [B,Hkv,C] per-row scales.  v_codes=None means K (with its scales) serves as V.
        """
        qb, kc = self._bits(q), self._codes(k_codes)
        B, Hq, D = qb.shape
        _, C, Hkv, Dk = kc.shape
        assert Dk == D and kc.shape[0] == B
        ks = self._f32(k_scale)
        assert ks.shape == (B, Hkv, C), ks.shape
        vc = self._codes(v_codes) if v_codes is not None else None
        vs = self._f32(v_scale) if v_codes is not None else None
        if vc is not None:
            assert vc.shape == kc.shape and vs.shape == ks.shape
        sl = np.ascontiguousarray(np.asarray(seqlens.cpu() if isinstance(seqlens, torch.Tensor)
                                             else seqlens, dtype=np.int32))
        out = np.zeros((B, Hq, D), dtype=np.float64)
        lse = np.zeros((B, Hq), dtype=np.float64)
        rc = self.lib.oracle_decode_fp8(
            self._ptr(qb, ctypes.c_uint16), self._ptr(kc, ctypes.c_uint8),
            self._ptr(vc, ctypes.c_uint8) if vc is not None else None,
            self._ptr(ks, ctypes.c_float),
            self._ptr(vs, ctypes.c_float) if vs is not None else None,
            self._ptr(sl, ctypes.c_int32), B, Hq, Hkv, D, C, C * Hkv * D, int(window),
            float(softcap), float(scale), 1 if vc is None else 0,
            self._ptr(out, ctypes.c_double), self._ptr(lse, ctypes.c_double))
        if rc != 0:
            raise ValueError("oracle_decode_fp8 rejected its arguments")
        return out, lse

    def attend(self, q, k, v, lo: Sequence[int], hi: Sequence[int], softcap: float,
               scale: float):
        """Attention over explicit logical position ranges [lo_b, hi_b) (slot = pos mod C)."""
        qb, kb = self._bits(q), self._bits(k)
        B, Hq, D = qb.shape
        _, C, Hkv, _ = kb.shape
        vb = self._bits(v) if v is not None else None
        lo_a = np.ascontiguousarray(np.asarray(lo, dtype=np.int32))
        hi_a = np.ascontiguousarray(np.asarray(hi, dtype=np.int32))
        out = np.zeros((B, Hq, D), dtype=np.float64)
        lse = np.zeros((B, Hq), dtype=np.float64)
        rc = self.lib.oracle_attend(
            self._ptr(qb, ctypes.c_uint16), self._ptr(kb, ctypes.c_uint16),
            self._ptr(vb, ctypes.c_uint16) if vb is not None else None, B, Hq, Hkv, D, C,
            C * Hkv * D, self._ptr(lo_a, ctypes.c_int32), self._ptr(hi_a, ctypes.c_int32),
            float(softcap), float(scale), 1 if vb is None else 0,
            self._ptr(out, ctypes.c_double), self._ptr(lse, ctypes.c_double))
        if rc != 0:
            raise ValueError("oracle_attend rejected its arguments")
        return out, lse

    def combine(self, o_parts, lse_parts):
        """LSE merge of partial results.  o_parts [..., S, D], lse_parts [..., S]."""
        o = np.asarray(o_parts, dtype=np.float64)
        l = np.asarray(lse_parts, dtype=np.float64)
        lead = o.shape[:-2]
        S, D = o.shape[-2:]
        o2 = np.ascontiguousarray(o.reshape(-1, S, D))
        l2 = np.ascontiguousarray(l.reshape(-1, S))
        out = np.zeros((o2.shape[0], D), dtype=np.float64)
        lse = np.zeros((o2.shape[0],), dtype=np.float64)
        for i in range(o2.shape[0]):
            oi = np.ascontiguousarray(o2[i])
            li = np.ascontiguousarray(l2[i])
            oo = np.zeros(D, dtype=np.float64)
            ll = np.zeros(1, dtype=np.float64)
            self.lib.oracle_combine(self._ptr(oi, ctypes.c_double), self._ptr(li, ctypes.c_double),
                                    S, D, self._ptr(oo, ctypes.c_double),
                                    self._ptr(ll, ctypes.c_double))
            out[i] = oo
            lse[i] = ll[0]
        return out.reshape(*lead, D), lse.reshape(lead)

    def decode_multi(self, q, k, v, seqlens, window: int, softcap: float, scale: float):
        """Multi-query decode: q bf16 [T,B,Hq,D], query t of sequence b at position
        L_b - T + t, attending causally.  Returns (out [T,B,Hq,D], lse [T,B,Hq]) float64."""
        qb, kb = self._bits(q), self._bits(k)
        T, B, Hq, D = qb.shape
        _, C, Hkv, Dk = kb.shape
        assert Dk == D and kb.shape[0] == B
        vb = self._bits(v) if v is not None else None
        sl = np.ascontiguousarray(np.asarray(seqlens.cpu() if isinstance(seqlens, torch.Tensor)
                                             else seqlens, dtype=np.int32))
        out = np.zeros((T, B, Hq, D), dtype=np.float64)
        lse = np.zeros((T, B, Hq), dtype=np.float64)
        rc = self.lib.oracle_decode_multi(
            self._ptr(qb, ctypes.c_uint16), self._ptr(kb, ctypes.c_uint16),
            self._ptr(vb, ctypes.c_uint16) if vb is not None else None,
            self._ptr(sl, ctypes.c_int32), T, B, Hq, Hkv, D, C, C * Hkv * D, int(window),
            float(softcap), float(scale), 1 if vb is None else 0,
            self._ptr(out, ctypes.c_double), self._ptr(lse, ctypes.c_double))
        if rc != 0:
            raise ValueError("oracle_decode_multi rejected its arguments")
        return out, lse

    def decode_layer(self, inputs):
        """Convenience: run ``decode`` on a ``workloads.LayerInputs``."""
        s = inputs.spec
        return self.decode(inputs.q, inputs.k, inputs.v, inputs.seqlens, s.window, s.softcap,
                           s.scale)


def load(mutation: int = 0, out_dir: Optional[str] = None) -> Oracle:
    key = (mutation, out_dir)
    if key not in _LIBS:
        _LIBS[key] = Oracle(_build.build(mutation, out_dir))
    return _LIBS[key]


def get() -> Oracle:
    """The oracle (built on first use)."""
    return load(0)


def position_range(seqlen: int, window: int):
    """Logical positions a decode step attends (window 0 = whole context)."""
    lo = max(0, seqlen - window) if window > 0 else 0
    return lo, seqlen


__all__ = ["Oracle", "load", "get", "position_range"]
