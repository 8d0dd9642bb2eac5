"""Device-side failure path without a GPU fault: with GDATTN_FLAG_TEST_WITHHOLD_KV
every CTA leaves its first KV tile unloaded, so a real bounded pipeline wait
runs out (after about 2 s at the maximum SM clock).  The kernel must drain its
copies and tensor-core work, free tensor memory and return; the call reports
GDATTN_ERR_DEVICE_TIMEOUT, the context stays usable, and the same workspace,
re-initialised, then gives the oracle's result.  Every kernel path is covered:
the tcgen05 pair kernel (bf16 and fp8 caches), the 16-head kernel, the
CUDA-core kernel, and the multi-token and prefill kernels."""
import pytest
import torch

import oracle
import workloads
from decode_attention_09_b200 import binding
from gpu_helpers import GpuLayer, compare, oracle_for, require_gpu

pytestmark = pytest.mark.gpu

WITHHOLD = binding.GDATTN_FLAG_TEST_WITHHOLD_KV

# (B, Hq, Hkv, D, C, seqlens, window, kv_shared, flags)
CASES = {
    "pair_even": (2, 16, 8, 256, 256, [256, 256], 256, False, binding.GDATTN_FLAG_EVEN_UNITS),
    "pair_chunks": (2, 16, 8, 256, 200, [450, 130], 200, False, 0),
    "tc16_even": (2, 16, 1, 512, 512, [512, 512], 0, True, binding.GDATTN_FLAG_EVEN_UNITS),
    "tc16_sepv_chunks": (2, 16, 1, 512, 300, [300, 77], 0, False, 0),
    "core_g4": (2, 8, 2, 256, 90, [90, 33], 0, False, 0),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_expired_wait_is_reported_and_context_survives(name):
    require_gpu()
    B, Hq, Hkv, D, C, sl, w, shared, flags = CASES[name]
    inp = workloads.random_case(950 + sorted(CASES).index(name), B, Hq, Hkv, D, C, sl, window=w,
                                kv_shared=shared)
    o_ref, l_ref = oracle_for(inp)
    layer = GpuLayer(inp)
    layer.set_desc(binding.desc_from_spec(inp.spec, capacity=C, flags=flags | WITHHOLD))
    layer.run(check_status=False)  # guards still checked: a failing kernel writes nothing outside
    assert binding.check_device_status(layer.ws) == binding.GDATTN_ERR_DEVICE_TIMEOUT
    # the context is usable and the workspace, re-initialised, serves a normal call
    layer.desc = binding.desc_from_spec(inp.spec, capacity=C, flags=flags)
    binding.workspace_init(layer.ws)
    out, lse = layer.run()
    compare(out, lse, o_ref, l_ref, ulp_floor=True, what=f"{name} after a timeout")


def test_expired_wait_fp8():
    require_gpu()
    f8 = workloads.random_fp8_case(960, 2, 16, 8, 256, 192, [300, 77], window=192)
    s = f8.spec
    desc = binding.desc_from_spec(s, capacity=192, flags=WITHHOLD)
    dev = "cuda"
    args = (f8.q.to(dev), f8.k_codes.to(dev), f8.v_codes.to(dev), f8.k_scale.to(dev),
            f8.v_scale.to(dev), f8.seqlens.to(dev))
    ws = binding.alloc_workspace(2, 300, desc, dev)
    binding.decode_fp8(*args, desc, 300, workspace=ws)
    assert binding.check_device_status(ws) == binding.GDATTN_ERR_DEVICE_TIMEOUT
    binding.workspace_init(ws)
    out, lse = binding.decode_fp8(*args, binding.desc_from_spec(s, capacity=192), 300,
                                  workspace=ws)
    assert binding.check_device_status(ws) == binding.GDATTN_OK
    o_ref, l_ref = oracle.get().decode_fp8(f8.q, f8.k_codes, f8.v_codes, f8.k_scale, f8.v_scale,
                                           f8.seqlens, s.window, s.softcap, s.scale)
    torch.cuda.synchronize()
    compare(out, lse, o_ref, l_ref, ulp_floor=True, what="fp8 after a timeout")


# Multi-token steps on the pair geometry: (T, seqlens, capacity, window, flags):
# the single-pass kernel with units cut into parts (counted merge) and with
# flattened chunks, and flash prefill.
MULTI_CASES = {
    "verify_t4_even": (4, [600, 600], 600, 512, binding.GDATTN_FLAG_EVEN_UNITS),
    "verify_t2_chunks": (2, [700, 90], 300, 256, 0),
    "prefill_t64": (64, [200, 64], 200, 128, 0),
}


@pytest.mark.parametrize("name", sorted(MULTI_CASES))
def test_expired_wait_multi_token(name):
    require_gpu()
    T, sl, C, w, flags = MULTI_CASES[name]
    B = len(sl)
    inp = workloads.random_case(970 + sorted(MULTI_CASES).index(name), B, 16, 8, 256, C, sl,
                                window=w)
    g = torch.Generator().manual_seed(980 + sorted(MULTI_CASES).index(name))
    q = torch.randn((T, B, 16, 256), generator=g).to(torch.bfloat16)
    s = inp.spec
    dev = "cuda"
    desc = binding.desc_from_spec(s, capacity=C, flags=flags | WITHHOLD)
    ws = torch.empty(binding.multi_workspace_size(B, T, max(sl), desc), dtype=torch.uint8,
                     device=dev)
    binding.workspace_init(ws)
    args = (q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.seqlens.to(dev))
    binding.decode_multi(*args, desc, max(sl), workspace=ws)
    assert binding.check_device_status(ws) == binding.GDATTN_ERR_DEVICE_TIMEOUT
    binding.workspace_init(ws)
    out, lse = binding.decode_multi(*args, binding.desc_from_spec(s, capacity=C, flags=flags),
                                    max(sl), workspace=ws)
    assert binding.check_device_status(ws) == binding.GDATTN_OK
    o_ref, l_ref = oracle.get().decode_multi(q, inp.k, inp.v, inp.seqlens, s.window, s.softcap,
                                             s.scale)
    torch.cuda.synchronize()
    for t in range(T):
        compare(out[t], lse[t], o_ref[t], l_ref[t], ulp_floor=True,
                what=f"{name} token {t} after a timeout")
