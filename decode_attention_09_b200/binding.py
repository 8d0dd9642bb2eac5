"""ctypes binding of libgdattn's C ABI (include/gdattn.h).

Argument marshalling only: every step of decode attention runs in the CUDA
kernels of libgdattn.so.  The tensor wrappers check what the C ABI cannot see
(dtype, contiguity, that each tensor reaches as far as the call reads or
writes, and its device) and raise ValueError before anything is enqueued; the
``*_raw`` functions pass addresses through unchecked.  Torch supplies device memory and streams.  There is no
fallback: if the library has not been built, loading it raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdattn.so")

GDATTN_OK = 0
GDATTN_ERR_INVALID_ARG = 1
GDATTN_ERR_UNSUPPORTED = 2
GDATTN_ERR_MISALIGNED = 3
GDATTN_ERR_WORKSPACE = 4
GDATTN_ERR_CUDA = 5
GDATTN_ERR_DEVICE_TIMEOUT = 6
GDATTN_ERR_DEVICE_SEQLEN = 7


class LayerDesc(ctypes.Structure):
    """Mirror of gdattn_layer_desc."""

    _fields_ = [
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("softcap", ctypes.c_float),
        ("scale", ctypes.c_float),
        ("kv_shared", ctypes.c_int32),
        ("cache_capacity", ctypes.c_int32),
        ("cache_batch_stride", ctypes.c_int64),
        ("split_ctas", ctypes.c_int32),
        ("flags", ctypes.c_int32),
    ]


class GdattnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libgdattn.so.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libgdattn.so not found at {LIB_PATH}; build it with "
                "`python decode_attention_09_b200/build.py` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
        descp = ctypes.POINTER(LayerDesc)
        L.gdattn_version.restype = i32
        L.gdattn_status_string.argtypes = [ctypes.c_int]
        L.gdattn_status_string.restype = ctypes.c_char_p
        L.gdattn_workspace_size.argtypes = [i32, i32, descp]
        L.gdattn_workspace_size.restype = sz
        L.gdattn_plan_splits.argtypes = [i32, i32, descp]
        L.gdattn_plan_splits.restype = i32
        L.gdattn_plan_launches.argtypes = [i32, i32, descp]
        L.gdattn_plan_launches.restype = i32
        L.gdattn_workspace_init.argtypes = [vp, sz, vp]
        L.gdattn_workspace_init.restype = ctypes.c_int
        L.gdattn_decode.argtypes = [vp, vp, vp, vp, i32, i32, descp, vp, vp, vp, sz, vp]
        L.gdattn_decode.restype = ctypes.c_int
        if hasattr(L, "gdattn_decode_append"):  # libraries built before it was added lack it
            L.gdattn_decode_append.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, descp, vp, vp,
                                               vp, sz, vp]
            L.gdattn_decode_append.restype = ctypes.c_int
        if hasattr(L, "gdattn_decode_multi"):
            L.gdattn_multi_workspace_size.argtypes = [i32, i32, i32, descp]
            L.gdattn_multi_workspace_size.restype = sz
            L.gdattn_decode_multi.argtypes = [vp, vp, vp, vp, i32, i32, i32, descp, vp, vp, vp,
                                              sz, vp]
            L.gdattn_decode_multi.restype = ctypes.c_int
        if hasattr(L, "gdattn_decode_fp8"):
            L.gdattn_decode_fp8.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, descp, vp, vp, vp,
                                            sz, vp]
            L.gdattn_decode_fp8.restype = ctypes.c_int
        L.gdattn_decode_noalloc.argtypes = [vp, vp, vp, vp, i32, i32, descp, vp, vp, vp]
        L.gdattn_decode_noalloc.restype = ctypes.c_int
        L.gdattn_combine.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp]
        L.gdattn_combine.restype = ctypes.c_int
        L.gdattn_check_device_status.argtypes = [vp, vp]
        L.gdattn_check_device_status.restype = ctypes.c_int
        L.gdattn_read_probe.argtypes = [vp, sz, i32, vp, vp]
        L.gdattn_read_probe.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gdattn_status_string(int(status)).decode()


def version() -> int:
    return int(lib().gdattn_version())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dense(t: torch.Tensor, name: str, dtypes, numel: int, device) -> None:
    """A dense tensor argument: one of ``dtypes``, contiguous, holding at least
    ``numel`` elements (what the call reads or writes through its pointer), on
    the CUDA device of the call.  The C ABI sees only the address, so a tensor
    that is too small would be read or written past its end on the device."""
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {' or '.join(map(str, dtypes))}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, the call reaches {numel}")
    _on(t, name, device)


def _extent(t: torch.Tensor, name: str, dtypes, numel: int, device) -> None:
    """A strided cache argument: one of ``dtypes``, with at least ``numel``
    elements of storage from its first element on (the rows the call may reach
    through ``cache_batch_stride``), on the CUDA device of the call."""
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {' or '.join(map(str, dtypes))}")
    have = t.untyped_storage().nbytes() // t.element_size() - t.storage_offset()
    if have < numel:
        raise ValueError(f"{name}: storage holds {have} elements, the call reaches {numel}")
    _on(t, name, device)


def _on(t: torch.Tensor, name: str, device) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: on {t.device}, the call runs on {device}")


def _cache_elems(batch: int, desc: "LayerDesc") -> int:
    """Elements of a cache that sequences 0..batch-1 span: sequence b starts at
    b * cache_batch_stride (0 = C * Hkv * D) and holds C * Hkv * D."""
    rows = int(desc.cache_capacity) * int(desc.n_kv_heads) * int(desc.head_dim)
    stride = int(desc.cache_batch_stride) or rows
    return (batch - 1) * stride + rows if batch > 0 else 0


_BF16 = (torch.bfloat16,)
_F32 = (torch.float32,)
_I32 = (torch.int32,)
_CODES = (torch.uint8, torch.float8_e4m3fn)


def _check_layer(q, k, v, seqlens, out, lse, desc, n_seq: int, n_cache: int) -> None:
    """The arguments every decode entry point shares: q and out are bf16
    [n_seq, Hq, D] (possibly with a leading token axis folded into n_seq), lse fp32
    [n_seq, Hq] or None, seqlens int32 [n_cache], and bf16 K / V caches spanning
    n_cache sequences."""
    dev = q.device
    hq, d = int(desc.n_q_heads), int(desc.head_dim)
    _dense(q, "q", _BF16, n_seq * hq * d, dev)
    _extent(k, "k", _BF16, _cache_elems(n_cache, desc), dev)
    if v is not None:
        _extent(v, "v", _BF16, _cache_elems(n_cache, desc), dev)
    _dense(seqlens, "seqlens", _I32, n_cache, dev)
    _dense(out, "out", _BF16, n_seq * hq * d, dev)
    if lse is not None:
        _dense(lse, "lse", _F32, n_seq * hq, dev)


def _check_new_rows(k_new, v_new, desc, batch: int, device) -> None:
    """gdattn_decode_append's rows: bf16 [batch, Hkv, D] (v_new None when K = V)."""
    rows = batch * int(desc.n_kv_heads) * int(desc.head_dim)
    _dense(k_new, "k_new", _BF16, rows, device)
    if v_new is not None:
        _dense(v_new, "v_new", _BF16, rows, device)


def _check_fp8(q, k_codes, v_codes, k_scale, v_scale, seqlens, out, lse, desc,
               batch: int) -> None:
    """gdattn_decode_fp8's arguments: e4m3 code caches (uint8 or float8_e4m3fn)
    spanning ``batch`` sequences, fp32 scales [batch, Hkv, C], the rest as for
    gdattn_decode."""
    dev = q.device
    hq, d = int(desc.n_q_heads), int(desc.head_dim)
    _dense(q, "q", _BF16, batch * hq * d, dev)
    n_scales = batch * int(desc.n_kv_heads) * int(desc.cache_capacity)
    _extent(k_codes, "k_codes", _CODES, _cache_elems(batch, desc), dev)
    _dense(k_scale, "k_scale", _F32, n_scales, dev)
    if v_codes is not None:  # None is the C ABI's to refuse (no fp8 path for K = V)
        _extent(v_codes, "v_codes", _CODES, _cache_elems(batch, desc), dev)
    if v_scale is not None:
        _dense(v_scale, "v_scale", _F32, n_scales, dev)
    _dense(seqlens, "seqlens", _I32, batch, dev)
    _dense(out, "out", _BF16, batch * hq * d, dev)
    if lse is not None:
        _dense(lse, "lse", _F32, batch * hq, dev)


def _check_combine(o_partial, lse_partial, out, lse) -> None:
    """gdattn_combine's arguments: fp32 partials [B, Hq, S, D] and [B, Hq, S],
    bf16 out [B, Hq, D], fp32 lse [B, Hq]."""
    B, Hq, S, D = o_partial.shape
    dev = o_partial.device
    _dense(o_partial, "o_partial", _F32, B * Hq * S * D, dev)
    _dense(lse_partial, "lse_partial", _F32, B * Hq * S, dev)
    _dense(out, "out", _BF16, B * Hq * D, dev)
    if lse is not None:
        _dense(lse, "lse", _F32, B * Hq, dev)


GDATTN_FLAG_EVEN_UNITS = 1
GDATTN_FLAG_TEST_WITHHOLD_KV = 2


def make_desc(n_q_heads: int, n_kv_heads: int, head_dim: int, window: int, softcap: float,
              scale: float, kv_shared: bool, cache_capacity: int, cache_batch_stride: int = 0,
              split_ctas: int = 0, flags: int = 0) -> LayerDesc:
    return LayerDesc(int(n_q_heads), int(n_kv_heads), int(head_dim), int(window),
                     float(softcap), float(scale), 1 if kv_shared else 0, int(cache_capacity),
                     int(cache_batch_stride), int(split_ctas), int(flags))


def desc_from_spec(spec, split_ctas: int = 0, capacity: Optional[int] = None,
                   flags: int = 0) -> LayerDesc:
    """Descriptor for a ``workloads.LayerSpec``."""
    return make_desc(spec.n_q_heads, spec.n_kv_heads, spec.head_dim, spec.window, spec.softcap,
                     spec.scale, spec.kv_shared,
                     capacity if capacity is not None else spec.capacity, 0, split_ctas, flags)


def workspace_size(batch: int, max_seqlen: int, desc: LayerDesc) -> int:
    return int(lib().gdattn_workspace_size(int(batch), int(max_seqlen), ctypes.byref(desc)))


def plan_splits(batch: int, max_seqlen: int, desc: LayerDesc) -> int:
    """CTAs the planner splits the KV range across (0 on invalid arguments)."""
    return int(lib().gdattn_plan_splits(int(batch), int(max_seqlen), ctypes.byref(desc)))


def launches_per_call(batch: int, max_seqlen: int, desc: LayerDesc) -> int:
    """Kernel launches one gdattn_decode call makes (1, or 2 with a separate combine)."""
    return int(lib().gdattn_plan_launches(int(batch), int(max_seqlen), ctypes.byref(desc)))


def workspace_init(workspace: torch.Tensor, stream=None) -> None:
    st = lib().gdattn_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream_handle(stream))
    if st != GDATTN_OK:
        raise GdattnError(st, "gdattn_workspace_init")


def alloc_workspace(batch: int, max_seqlen: int, desc: LayerDesc, device="cuda",
                    stream=None) -> torch.Tensor:
    n = workspace_size(batch, max_seqlen, desc)
    if n == 0:
        raise GdattnError(GDATTN_ERR_INVALID_ARG, "gdattn_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    workspace_init(ws, stream)
    return ws


def decode_raw(q, k, v, seqlens, batch, max_seqlen, desc, out, lse, workspace, workspace_bytes,
               stream) -> int:
    """gdattn_decode on raw addresses (ints); returns the status code."""
    return int(lib().gdattn_decode(q, k, v, seqlens, int(batch), int(max_seqlen),
                                   ctypes.byref(desc), out, lse, workspace,
                                   int(workspace_bytes), stream))


def decode(q: torch.Tensor, k: torch.Tensor, v: Optional[torch.Tensor], seqlens: torch.Tensor,
           desc: LayerDesc, max_seqlen: int, out: Optional[torch.Tensor] = None,
           lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
           stream=None, want_lse: bool = True):
    """One decode-attention layer through gdattn_decode.  Returns (out, lse)."""
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _check_layer(q, k, v, seqlens, out, lse, desc, B, B)
    if workspace is None:
        workspace = alloc_workspace(B, max_seqlen, desc, q.device, stream)
    _on(workspace, "workspace", q.device)
    st = decode_raw(_ptr(q), _ptr(k), _ptr(v), _ptr(seqlens), B, max_seqlen, desc, _ptr(out),
                    _ptr(lse), _ptr(workspace), workspace.numel(), _stream_handle(stream))
    if st != GDATTN_OK:
        raise GdattnError(st, "gdattn_decode")
    return out, lse


def decode_append(q: torch.Tensor, k_new: torch.Tensor, v_new: Optional[torch.Tensor],
                  k: torch.Tensor, v: Optional[torch.Tensor], seqlens: torch.Tensor,
                  desc: LayerDesc, max_seqlen: int, out: Optional[torch.Tensor] = None,
                  lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None):
    """gdattn_decode_append: write k_new / v_new ([B, Hkv, D]) into slot
    (L - 1) mod C of the caches, then decode.  Returns (out, lse)."""
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _check_layer(q, k, v, seqlens, out, lse, desc, B, B)
    _check_new_rows(k_new, v_new, desc, B, q.device)
    if workspace is None:
        workspace = alloc_workspace(B, max_seqlen, desc, q.device, stream)
    _on(workspace, "workspace", q.device)
    st = int(lib().gdattn_decode_append(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k), _ptr(v),
                                        _ptr(seqlens), B, int(max_seqlen), ctypes.byref(desc),
                                        _ptr(out), _ptr(lse), _ptr(workspace),
                                        workspace.numel(), _stream_handle(stream)))
    if st != GDATTN_OK:
        raise GdattnError(st, "gdattn_decode_append")
    return out, lse


def decode_fp8_raw(q, k_codes, v_codes, k_scale, v_scale, seqlens, batch, max_seqlen, desc, out,
                   lse, workspace, workspace_bytes, stream) -> int:
    """gdattn_decode_fp8 on raw addresses (ints); returns the status code."""
    return int(lib().gdattn_decode_fp8(q, k_codes, v_codes, k_scale, v_scale, seqlens,
                                       int(batch), int(max_seqlen), ctypes.byref(desc), out, lse,
                                       workspace, int(workspace_bytes), stream))


def decode_fp8(q: torch.Tensor, k_codes: torch.Tensor, v_codes: torch.Tensor,
               k_scale: torch.Tensor, v_scale: torch.Tensor, seqlens: torch.Tensor,
               desc: LayerDesc, max_seqlen: int, out: Optional[torch.Tensor] = None,
               lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               stream=None):
    """One layer over an fp8 e4m3 cache through gdattn_decode_fp8.  Returns (out, lse).

    k_codes / v_codes: uint8 (or float8_e4m3fn) [B, C, Hkv, D]; k_scale / v_scale:
    float32 [B, Hkv, C], the scale of each cache row.
    """
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _check_fp8(q, k_codes, v_codes, k_scale, v_scale, seqlens, out, lse, desc, B)
    if workspace is None:
        workspace = alloc_workspace(B, max_seqlen, desc, q.device, stream)
    _on(workspace, "workspace", q.device)
    st = decode_fp8_raw(_ptr(q), _ptr(k_codes), _ptr(v_codes), _ptr(k_scale), _ptr(v_scale),
                        _ptr(seqlens), B, max_seqlen, desc, _ptr(out), _ptr(lse),
                        _ptr(workspace), workspace.numel(), _stream_handle(stream))
    if st != GDATTN_OK:
        raise GdattnError(st, "gdattn_decode_fp8")
    return out, lse


def multi_workspace_size(batch: int, n_tokens: int, max_seqlen: int, desc: LayerDesc) -> int:
    return int(lib().gdattn_multi_workspace_size(int(batch), int(n_tokens), int(max_seqlen),
                                                 ctypes.byref(desc)))


def decode_multi_raw(q, k, v, seqlens, batch, n_tokens, max_seqlen, desc, out, lse, workspace,
                     workspace_bytes, stream) -> int:
    """gdattn_decode_multi on raw addresses (ints); returns the status code."""
    return int(lib().gdattn_decode_multi(q, k, v, seqlens, int(batch), int(n_tokens),
                                         int(max_seqlen), ctypes.byref(desc), out, lse, workspace,
                                         int(workspace_bytes), stream))


def decode_multi(q: torch.Tensor, k: torch.Tensor, v: Optional[torch.Tensor],
                 seqlens: torch.Tensor, desc: LayerDesc, max_seqlen: int,
                 out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None):
    """Multi-token step through gdattn_decode_multi: a verify step, or a prompt chunk
    (flash prefill).  q bf16 [T, B, Hq, D]: token t of sequence b at position
    L_b - T + t, attending causally.  Returns (out, lse), token-major."""
    T, B, Hq, D = q.shape
    if out is None:
        out = torch.empty((T, B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((T, B, Hq), dtype=torch.float32, device=q.device)
    _check_layer(q, k, v, seqlens, out, lse, desc, T * B, B)
    if workspace is None:
        n = multi_workspace_size(B, T, max_seqlen, desc)
        if n == 0:
            raise GdattnError(GDATTN_ERR_INVALID_ARG, "gdattn_multi_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
        workspace_init(workspace, stream)
    _on(workspace, "workspace", q.device)
    st = decode_multi_raw(_ptr(q), _ptr(k), _ptr(v), _ptr(seqlens), B, T, max_seqlen, desc,
                          _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                          _stream_handle(stream))
    if st != GDATTN_OK:
        raise GdattnError(st, "gdattn_decode_multi")
    return out, lse


NOALLOC_SCRATCH_BYTES = 8 << 20  # GDATTN_NOALLOC_SCRATCH_BYTES


def decode_noalloc_raw(q, k, v, seqlens, batch, max_seqlen, desc, out, lse, stream) -> int:
    """gdattn_decode_noalloc on raw addresses (ints); returns the status code."""
    return int(lib().gdattn_decode_noalloc(q, k, v, seqlens, int(batch), int(max_seqlen),
                                           ctypes.byref(desc), out, lse, stream))


def decode_noalloc(q: torch.Tensor, k: torch.Tensor, v: Optional[torch.Tensor],
                   seqlens: torch.Tensor, desc: LayerDesc, max_seqlen: int,
                   out: torch.Tensor, lse: Optional[torch.Tensor] = None, stream=None):
    """One layer through gdattn_decode_noalloc (scratch inside the library).

    `out` (and `lse`, if wanted) are caller-owned; nothing is allocated here.
    Calls that can overlap in time on one device race on the shared scratch.
    """
    B = q.shape[0]
    _check_layer(q, k, v, seqlens, out, lse, desc, B, B)
    st = decode_noalloc_raw(_ptr(q), _ptr(k), _ptr(v), _ptr(seqlens), B, max_seqlen, desc,
                            _ptr(out), _ptr(lse), _stream_handle(stream))
    if st != GDATTN_OK:
        raise GdattnError(st, "gdattn_decode_noalloc")
    return out, lse


def combine(o_partial: torch.Tensor, lse_partial: torch.Tensor, out: Optional[torch.Tensor] = None,
            lse: Optional[torch.Tensor] = None, stream=None):
    """gdattn_combine: o_partial fp32 [B,Hq,S,D], lse_partial fp32 [B,Hq,S]."""
    B, Hq, S, D = o_partial.shape
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=o_partial.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=o_partial.device)
    _check_combine(o_partial, lse_partial, out, lse)
    st = lib().gdattn_combine(_ptr(o_partial), _ptr(lse_partial), B, Hq, S, D, _ptr(out), _ptr(lse),
                              _stream_handle(stream))
    if st != GDATTN_OK:
        raise GdattnError(st, "gdattn_combine")
    return out, lse


def check_device_status(workspace: Optional[torch.Tensor], stream=None) -> int:
    """Read and clear a workspace's status word (None: the no-alloc scratch)."""
    return int(lib().gdattn_check_device_status(_ptr(workspace), _stream_handle(stream)))


def read_probe(src: torch.Tensor, mode: int, sink: torch.Tensor, stream=None) -> None:
    """gdattn_read_probe over the whole of ``src`` (a contiguous device tensor);
    ``sink``: int32 tensor of 2 elements on the same device."""
    _on(sink, "sink", src.device)
    if not src.is_contiguous() or sink.numel() < 2 or sink.dtype != torch.int32:
        raise ValueError("read_probe: contiguous src and an int32 sink of 2 elements")
    st = lib().gdattn_read_probe(_ptr(src), src.numel() * src.element_size(), int(mode),
                                 _ptr(sink), _stream_handle(stream))
    if st != GDATTN_OK:
        raise GdattnError(st, "gdattn_read_probe")
