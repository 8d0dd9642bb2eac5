"""Seeded synthetic workloads for Gemma-4-style decode attention.

This module only draws inputs: shapes, seeds, value distributions and the
per-layer geometry of the stacks.  It holds none of the attention arithmetic,
so the float64 oracle and the CUDA library can both take their inputs from
here without sharing any of the method.

Geometry follows the "Gemma 4 12B" record (KV GEOMETRY paragraph): sliding
layers use head_dim 256 with 8 KV heads, full ("global") layers use
global_head_dim 512 with a single KV head and attention_k_eq_v, and the 48-layer
schedule puts the full layers at 0-based indices 5, 11, ..., 47.  The query-side
scale defaults to 1/sqrt(head_dim) per geometry ("Gemma4-26B-A4B ... NO-GO",
section 5, per-attention-scale assumption).

Every tensor is bf16 drawn from N(0, 1) with a torch.Generator seeded as stated,
except the per-sequence context lengths of the ragged workload (uniform integers)
and the heavy-row stress of the long-context workload (a Bernoulli row mask whose
rows are multiplied by a constant before rounding to bf16).

fp8 caches (``fp8_layer_inputs``): each cache row (one token of one KV head) is
N(0, 1) times a per-row spread 2^u, u uniform in [-spread, spread], then stored
the way a quantizing cache writer would store it: scale = the row's largest
|value| / 448 and codes = value / scale rounded to e4m3 (torch's float8_e4m3fn
conversion).  The decode under test only reads the codes and scales.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import List, Optional

import torch

# --------------------------------------------------------------------------
# Layer geometry
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class LayerSpec:
    """One attention layer's geometry as the decode call sees it."""

    kind: str  # "sliding" or "global"
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    window: int  # 0 = attend the whole context
    softcap: float  # 0 = off
    scale: float
    kv_shared: bool  # K serves as V (attention_k_eq_v)
    capacity: int  # cache slots per sequence (ring size for sliding layers)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


def sliding_spec(capacity: int, window: int, softcap: float = 0.0, n_q_heads: int = 16,
                 n_kv_heads: int = 8, head_dim: int = 256) -> LayerSpec:
    return LayerSpec("sliding", n_q_heads, n_kv_heads, head_dim, window, softcap,
                     1.0 / math.sqrt(head_dim), False, capacity)


def global_spec(capacity: int, softcap: float = 0.0, n_q_heads: int = 16,
                n_kv_heads: int = 1, head_dim: int = 512, kv_shared: bool = True) -> LayerSpec:
    return LayerSpec("global", n_q_heads, n_kv_heads, head_dim, 0, softcap,
                     1.0 / math.sqrt(head_dim), kv_shared, capacity)


GEMMA4_12B_GLOBAL_LAYERS = tuple(range(5, 48, 6))  # 5, 11, ..., 47


def gemma4_12b_stack(sliding_capacity: int, global_capacity: int, softcap: float = 0.0,
                     window: int = 1024) -> List[LayerSpec]:
    """The 48-layer schedule: 40 sliding + 8 global (K = V) layers."""
    layers = []
    for i in range(48):
        if i in GEMMA4_12B_GLOBAL_LAYERS:
            layers.append(global_spec(global_capacity, softcap))
        else:
            layers.append(sliding_spec(sliding_capacity, window, softcap))
    return layers


# --------------------------------------------------------------------------
# Named workloads
# --------------------------------------------------------------------------


@dataclass
class Workload:
    name: str
    batch: int
    layers: List[LayerSpec]
    seed: int
    seqlen: Optional[int] = None  # uniform context length, or None when ragged
    ragged: Optional[tuple] = None  # (lo, hi) inclusive bounds for per-sequence lengths
    heavy_row_frac: float = 0.0  # fraction of K rows scaled by heavy_row_scale
    heavy_row_scale: float = 8.0
    note: str = ""

    def seqlens(self) -> torch.Tensor:
        """Per-sequence context length L_b (tokens attended, current token included)."""
        if self.ragged is None:
            return torch.full((self.batch,), int(self.seqlen), dtype=torch.int32)
        g = torch.Generator().manual_seed(self.seed)
        lo, hi = self.ragged
        return torch.randint(lo, hi + 1, (self.batch,), generator=g).to(torch.int32)


def single_sliding() -> Workload:
    """Single sliding layer, batch 1: q [1,16,256], K/V [2048,8,256], w 512, cap 50."""
    spec = replace(sliding_spec(2048, 512, softcap=50.0), scale=1.0 / 16.0)
    return Workload("single_sliding_b1_c2048_w512", 1, [spec], seed=1, seqlen=2048,
                    note="cache full (L = C = 2048); the last 512 positions are attended")


def single_global() -> Workload:
    """Single global K=V layer, batch 1, context 32768, hd 512, one KV head."""
    return Workload("single_global_b1_l32768", 1, [global_spec(32768)], seed=2, seqlen=32768)


def gemma4_12b_b8_l8192() -> Workload:
    """Gemma-4-12B-shaped 48-layer decode-attention stack, batch 8, context 8192."""
    return Workload("gemma4_12b_stack_b8_l8192", 8, gemma4_12b_stack(1024, 8192), seed=3,
                    seqlen=8192)


def ragged_b64() -> Workload:
    """Batch 64, L_b ~ U[512, 32768]; one sliding (w 1024) + one global K=V layer, cap 50."""
    layers = [sliding_spec(1024, 1024, softcap=50.0), global_spec(32768, softcap=50.0)]
    return Workload("ragged_b64_l512_32768", 64, layers, seed=4, ragged=(512, 32768))


def long_context_b4() -> Workload:
    """Batch 4, context 131072, the 48-layer stack; 1 % of K rows scaled x8."""
    return Workload("gemma4_12b_stack_b4_l131072", 4, gemma4_12b_stack(1024, 131072), seed=5,
                    seqlen=131072, heavy_row_frac=0.01, heavy_row_scale=8.0)


def gemma4_12b_two_layers_b8_l8192() -> Workload:
    """Layers 0 (sliding) and 5 (global) of the 12B stack at batch 8, context 8192:
    the headline's per-layer shapes and launch configurations on a few hundred MB
    of device memory, for profiler captures."""
    stack = gemma4_12b_stack(1024, 8192)
    return Workload("gemma4_12b_two_layers_b8_l8192", 8, [stack[0], stack[5]], seed=3,
                    seqlen=8192)


ALL_WORKLOADS = {w().name: w for w in (single_sliding, single_global, gemma4_12b_b8_l8192,
                                       ragged_b64, long_context_b4,
                                       gemma4_12b_two_layers_b8_l8192)}


# --------------------------------------------------------------------------
# Tensor generation
# --------------------------------------------------------------------------


@dataclass
class LayerInputs:
    q: torch.Tensor  # bf16 [B, Hq, D]
    k: torch.Tensor  # bf16 [B, C, Hkv, D]
    v: Optional[torch.Tensor]  # bf16 [B, C, Hkv, D] or None when K serves as V
    seqlens: torch.Tensor  # int32 [B]
    spec: LayerSpec = field(repr=False, default=None)


def _gen(seed: int, device) -> torch.Generator:
    return torch.Generator(device=device).manual_seed(int(seed))


def layer_inputs(spec: LayerSpec, batch: int, seqlens: torch.Tensor, seed: int,
                 device="cpu", heavy_row_frac: float = 0.0, heavy_row_scale: float = 8.0,
                 capacity: Optional[int] = None) -> LayerInputs:
    """Draw q, K (and V unless K serves as V) for one layer.

    Values are N(0, 1) rounded to bf16.  With ``heavy_row_frac`` > 0 a Bernoulli
    mask over cache rows (b, slot) picks rows of K whose every head is multiplied
    by ``heavy_row_scale`` before rounding; for a K = V layer that is the one
    shared tensor.  Streams depend on ``device`` (torch's CPU and CUDA generators
    differ); tests compare both sides on the very same tensors.
    """
    C = int(capacity if capacity is not None else spec.capacity)
    g = _gen(seed, device)
    B, Hq, Hkv, D = batch, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
    q = torch.randn((B, Hq, D), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn((B, C, Hkv, D), generator=g, device=device, dtype=torch.float32)
    if heavy_row_frac > 0:
        rows = torch.rand((B, C), generator=g, device=device) < heavy_row_frac
        k[rows] *= heavy_row_scale
    k = k.to(torch.bfloat16)
    v = None
    if not spec.kv_shared:
        v = torch.randn((B, C, Hkv, D), generator=g, device=device,
                        dtype=torch.float32).to(torch.bfloat16)
    return LayerInputs(q, k, v, seqlens.to(torch.int32).to(device), spec)


def workload_layer_inputs(w: Workload, layer: int, device="cpu") -> LayerInputs:
    spec = w.layers[layer]
    return layer_inputs(spec, w.batch, w.seqlens(), w.seed * 1000 + layer, device=device,
                        heavy_row_frac=w.heavy_row_frac, heavy_row_scale=w.heavy_row_scale)


def random_case(seed: int, batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                capacity: int, seqlens, window: int = 0, softcap: float = 0.0,
                scale: Optional[float] = None, kv_shared: bool = False,
                device="cpu") -> LayerInputs:
    """A small seeded case of arbitrary geometry (for sweeps and edge cases)."""
    spec = LayerSpec("sliding" if window > 0 else "global", n_q_heads, n_kv_heads, head_dim,
                     window, softcap, (1.0 / math.sqrt(head_dim)) if scale is None else scale,
                     kv_shared, capacity)
    sl = torch.as_tensor(seqlens, dtype=torch.int32).reshape(batch)
    return layer_inputs(spec, batch, sl, seed, device=device)


# --------------------------------------------------------------------------
# fp8 e4m3 caches with per-row scales
# --------------------------------------------------------------------------

E4M3_MAX = 448.0


@dataclass
class Fp8LayerInputs:
    q: torch.Tensor  # bf16 [B, Hq, D]
    k_codes: torch.Tensor  # uint8 e4m3 codes [B, C, Hkv, D]
    v_codes: Optional[torch.Tensor]  # uint8 [B, C, Hkv, D] or None when K serves as V
    k_scale: torch.Tensor  # float32 [B, Hkv, C]: scale of row (b, kv, slot)
    v_scale: Optional[torch.Tensor]  # float32 [B, Hkv, C] or None
    seqlens: torch.Tensor  # int32 [B]
    spec: LayerSpec = field(repr=False, default=None)


def quantize_rows_e4m3(x: torch.Tensor):
    """Rows of x [B, C, Hkv, D] (float32) -> (codes uint8 [B, C, Hkv, D], scales float32
    [B, Hkv, C]) with scale = row max |x| / 448 (1 for an all-zero row)."""
    amax = x.abs().amax(dim=-1)  # [B, C, Hkv]
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    codes = (x / scale.unsqueeze(-1)).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.permute(0, 2, 1).contiguous()


def fp8_layer_inputs(spec: LayerSpec, batch: int, seqlens: torch.Tensor, seed: int,
                     device="cpu", capacity: Optional[int] = None,
                     spread: float = 1.5) -> Fp8LayerInputs:
    """q as in ``layer_inputs``; K (and V unless K serves as V) rows N(0, 1) * 2^u,
    u ~ U(-spread, spread) per row, quantized per row to e4m3 codes and a scale."""
    C = int(capacity if capacity is not None else spec.capacity)
    g = _gen(seed, device)
    B, Hq, Hkv, D = batch, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
    q = torch.randn((B, Hq, D), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)

    def rows():
        x = torch.randn((B, C, Hkv, D), generator=g, device=device, dtype=torch.float32)
        u = (torch.rand((B, C, Hkv, 1), generator=g, device=device) * 2 - 1) * spread
        return quantize_rows_e4m3(x * torch.exp2(u))

    k_codes, k_scale = rows()
    v_codes = v_scale = None
    if not spec.kv_shared:
        v_codes, v_scale = rows()
    return Fp8LayerInputs(q, k_codes, v_codes, k_scale, v_scale,
                          seqlens.to(torch.int32).to(device), spec)


def random_fp8_case(seed: int, batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                    capacity: int, seqlens, window: int = 0, softcap: float = 0.0,
                    scale: Optional[float] = None, kv_shared: bool = False, spread: float = 1.5,
                    device="cpu") -> Fp8LayerInputs:
    """A small seeded fp8-cache case of arbitrary geometry."""
    spec = LayerSpec("sliding" if window > 0 else "global", n_q_heads, n_kv_heads, head_dim,
                     window, softcap, (1.0 / math.sqrt(head_dim)) if scale is None else scale,
                     kv_shared, capacity)
    sl = torch.as_tensor(seqlens, dtype=torch.int32).reshape(batch)
    return fp8_layer_inputs(spec, batch, sl, seed, device=device, spread=spread)
