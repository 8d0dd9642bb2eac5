"""Device-side failure path without a GPU fault: with GDATTN_FLAG_TEST_WITHHOLD_KV
every CTA leaves its first KV tile unloaded, so a real bounded pipeline wait
runs out (after about 2 s at the maximum SM clock).  The kernel must drain its
copies and tensor-core work, free tensor memory and return; the call reports
GDATTN_ERR_DEVICE_TIMEOUT, the context stays usable, and the same workspace,
re-initialised, then gives the oracle's result.  Every kernel path is covered:
the tcgen05 pair kernel (bf16 and fp8 caches), the 16-head kernel, and the
CUDA-core kernel."""
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
