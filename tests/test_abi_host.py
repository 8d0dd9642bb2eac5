"""The C ABI without a GPU: exports, struct layout and host-side argument checks.

Every call here is rejected by a host check before the library touches CUDA, so
these run on a machine with no GPU.  Fake device addresses are never
dereferenced.
"""
import ctypes
import os
import re
import subprocess

import pytest

from decode_attention_09_b200 import binding
from decode_attention_09_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdattn.h")

A = 0x100000  # a 16-byte-aligned fake device address (never dereferenced)


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return binding.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(gdattn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_api():
    names = declared_functions()
    for n in ("gdattn_decode", "gdattn_decode_fp8", "gdattn_decode_multi", "gdattn_combine",
              "gdattn_workspace_size", "gdattn_multi_workspace_size",
              "gdattn_workspace_init",
              "gdattn_plan_splits", "gdattn_plan_launches",
              "gdattn_check_device_status", "gdattn_status_string", "gdattn_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], check=True,
                         capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT\s+(gdattn_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for n in declared_functions():
        assert hasattr(lib, n)


def test_desc_layout_matches_c(tmp_path):
    """ctypes mirror of gdattn_layer_desc has the C compiler's size and offsets."""
    src = tmp_path / "layout.c"
    fields = [f for f, _ in binding.LayerDesc._fields_]
    body = "\n".join(f'printf("%zu\\n", offsetof(gdattn_layer_desc, {f}));' for f in fields)
    src.write_text("#include <stddef.h>\n#include <stdio.h>\n#include \"gdattn.h\"\n"
                   "int main(void){" + body + 'printf("%zu\\n", sizeof(gdattn_layer_desc));'
                   "return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe)], check=True)
    vals = [int(x) for x in subprocess.run([str(exe)], check=True, capture_output=True,
                                           text=True).stdout.split()]
    expect = [getattr(binding.LayerDesc, f).offset for f in fields] + [
        ctypes.sizeof(binding.LayerDesc)]
    assert vals == expect


def test_plain_c_client_links_and_gets_the_documented_statuses(lib, tmp_path):
    """tests/abi_client.c: a C99 program that includes only gdattn.h, links the
    shared library and checks the statuses of calls the host checks refuse."""
    pkg = os.path.dirname(binding.LIB_PATH)
    exe = tmp_path / "abi_client"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "abi_client.c"), "-o", str(exe),
                    f"-L{pkg}", "-lgdattn", f"-Wl,-rpath,{pkg}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr


def test_version_and_status_strings(lib):
    assert binding.version() == 100
    assert binding.status_string(0) == "GDATTN_OK"
    assert binding.status_string(binding.GDATTN_ERR_DEVICE_SEQLEN) == "GDATTN_ERR_DEVICE_SEQLEN"
    assert binding.status_string(999) == "GDATTN_UNKNOWN_STATUS"


def good_desc(**kw):
    d = dict(n_q_heads=16, n_kv_heads=8, head_dim=256, window=1024, softcap=0.0,
             scale=1 / 16, kv_shared=False, cache_capacity=1024)
    d.update(kw)
    return binding.make_desc(**d)


def call(desc, q=A, k=A, v=A, seqlens=A, batch=1, max_seqlen=8, out=A, lse=A, ws=A, ws_bytes=1 << 20):
    return binding.decode_raw(q, k, v, seqlens, batch, max_seqlen, desc, out, lse, ws, ws_bytes,
                              None)


@pytest.mark.parametrize("case,expect", [
    (dict(q=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(k=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(seqlens=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(out=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(v=None), binding.GDATTN_ERR_INVALID_ARG),  # separate V expected
    (dict(batch=0), binding.GDATTN_ERR_INVALID_ARG),
    (dict(max_seqlen=0), binding.GDATTN_ERR_INVALID_ARG),
    (dict(q=A + 8), binding.GDATTN_ERR_MISALIGNED),
    (dict(k=A + 2), binding.GDATTN_ERR_MISALIGNED),
    (dict(v=A + 4), binding.GDATTN_ERR_MISALIGNED),
    (dict(out=A + 8), binding.GDATTN_ERR_MISALIGNED),
    (dict(seqlens=A + 2), binding.GDATTN_ERR_MISALIGNED),
    (dict(lse=A + 1), binding.GDATTN_ERR_MISALIGNED),
    (dict(ws=None), binding.GDATTN_ERR_WORKSPACE),
    (dict(ws=A + 8), binding.GDATTN_ERR_MISALIGNED),
])
def test_decode_rejects_bad_pointers(lib, case, expect):
    assert call(good_desc(), **case) == expect


@pytest.mark.parametrize("desc_kw,expect", [
    (dict(n_q_heads=0), binding.GDATTN_ERR_INVALID_ARG),
    (dict(n_kv_heads=0), binding.GDATTN_ERR_INVALID_ARG),
    (dict(n_q_heads=12, n_kv_heads=8), binding.GDATTN_ERR_INVALID_ARG),
    (dict(head_dim=0), binding.GDATTN_ERR_INVALID_ARG),
    (dict(cache_capacity=0), binding.GDATTN_ERR_INVALID_ARG),
    (dict(window=-1), binding.GDATTN_ERR_INVALID_ARG),
    (dict(softcap=-1.0), binding.GDATTN_ERR_INVALID_ARG),
    (dict(softcap=float("nan")), binding.GDATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), binding.GDATTN_ERR_INVALID_ARG),
    (dict(split_ctas=-1), binding.GDATTN_ERR_INVALID_ARG),
    (dict(cache_batch_stride=100), binding.GDATTN_ERR_INVALID_ARG),  # < C*Hkv*D
    (dict(cache_batch_stride=1024 * 8 * 256 + 4), binding.GDATTN_ERR_INVALID_ARG),  # not % 8
    (dict(head_dim=128), binding.GDATTN_ERR_UNSUPPORTED),
    (dict(n_q_heads=64, n_kv_heads=8), binding.GDATTN_ERR_UNSUPPORTED),  # G = 8
    (dict(n_q_heads=64, n_kv_heads=16), binding.GDATTN_ERR_UNSUPPORTED),  # G = 4, Hkv = 16
])
def test_decode_rejects_bad_desc(lib, desc_kw, expect):
    assert call(good_desc(**desc_kw)) == expect


def test_kv_shared_requires_null_v(lib):
    d = good_desc(n_q_heads=16, n_kv_heads=1, head_dim=512, window=0, kv_shared=True)
    assert call(d, v=A) == binding.GDATTN_ERR_INVALID_ARG
    d.flags = 4  # undefined flag bit
    assert call(d, v=None) == binding.GDATTN_ERR_INVALID_ARG


def test_sixteen_head_groups_need_head_dim_512(lib):
    """8- and 16-head groups run on the tcgen05 16-head kernel at head_dim 512
    (K = V or separate V); at other head sizes no kernel serves them."""
    for g in (8, 16):
        d = good_desc(n_q_heads=g, n_kv_heads=1, head_dim=256, window=0, kv_shared=False)
        assert call(d) == binding.GDATTN_ERR_UNSUPPORTED
    d = good_desc(n_q_heads=12, n_kv_heads=1, head_dim=512, window=0, kv_shared=False)
    assert call(d) == binding.GDATTN_ERR_UNSUPPORTED  # G = 12


def test_unit_count_beyond_the_fixed_header_is_refused(lib):
    """The workspace header holds counters and epochs for 16384 (sequence, KV
    head) units; a call with more is refused before anything is enqueued."""
    assert call(good_desc(), batch=2049) == binding.GDATTN_ERR_UNSUPPORTED  # 16392 units
    assert binding.workspace_size(2049, 8, good_desc()) == 0
    core = good_desc(n_q_heads=4, n_kv_heads=1, head_dim=256, window=0)  # one unit per sequence
    assert call(core, v=A, batch=16385) == binding.GDATTN_ERR_UNSUPPORTED


def test_workspace_size_rejects_bad_args(lib):
    assert binding.workspace_size(0, 8, good_desc()) == 0
    assert binding.workspace_size(1, 8, good_desc(head_dim=128)) == 0
    assert lib.gdattn_workspace_size(1, 8, None) == 0
    assert binding.plan_splits(0, 8, good_desc()) == 0
    assert binding.plan_splits(1, 8, good_desc(n_q_heads=12)) == 0


def test_workspace_init_rejects_null(lib):
    assert lib.gdattn_workspace_init(None, 1024, None) == binding.GDATTN_ERR_WORKSPACE
    assert lib.gdattn_workspace_init(A, 16, None) == binding.GDATTN_ERR_WORKSPACE
    assert lib.gdattn_workspace_init(A + 8, 1024, None) == binding.GDATTN_ERR_MISALIGNED


@pytest.mark.parametrize("args,expect", [
    ((None, A, 1, 16, 2, 256, A, A), binding.GDATTN_ERR_INVALID_ARG),
    ((A, None, 1, 16, 2, 256, A, A), binding.GDATTN_ERR_INVALID_ARG),
    ((A, A, 1, 16, 2, 256, None, A), binding.GDATTN_ERR_INVALID_ARG),
    ((A, A, 0, 16, 2, 256, A, A), binding.GDATTN_ERR_INVALID_ARG),
    ((A, A, 1, 0, 2, 256, A, A), binding.GDATTN_ERR_INVALID_ARG),
    ((A, A, 1, 16, 0, 256, A, A), binding.GDATTN_ERR_INVALID_ARG),
    ((A, A, 1, 16, 2, 6, A, A), binding.GDATTN_ERR_INVALID_ARG),
    ((A, A, 1, 16, 2, 2048, A, A), binding.GDATTN_ERR_INVALID_ARG),
    ((A, A, 1, 16, 9000, 256, A, A), binding.GDATTN_ERR_INVALID_ARG),
    ((A + 4, A, 1, 16, 2, 256, A, A), binding.GDATTN_ERR_MISALIGNED),
    ((A, A + 2, 1, 16, 2, 256, A, A), binding.GDATTN_ERR_MISALIGNED),
    ((A, A, 1, 16, 2, 256, A + 8, A), binding.GDATTN_ERR_MISALIGNED),
])
def test_combine_rejects_bad_args(lib, args, expect):
    o, l, B, Hq, S, D, out, lse = args
    assert lib.gdattn_combine(o, l, B, Hq, S, D, out, lse, None) == expect


def test_decode_append_host_checks(lib):
    """gdattn_decode_append: the new rows' pointers are checked like the rest."""
    def app(desc, k_new=A, v_new=A, q=A, k=A, v=A, ws=A):
        return lib.gdattn_decode_append(q, k_new, v_new, k, v, A, 1, 8, ctypes.byref(desc), A, A,
                                        ws, 1 << 20, None)
    d = good_desc()
    assert app(d, k_new=None) == binding.GDATTN_ERR_INVALID_ARG
    assert app(d, v_new=None) == binding.GDATTN_ERR_INVALID_ARG      # separate V expected
    assert app(d, k_new=A + 8) == binding.GDATTN_ERR_MISALIGNED
    assert app(d, v_new=A + 4) == binding.GDATTN_ERR_MISALIGNED
    assert app(d, ws=None) == binding.GDATTN_ERR_WORKSPACE
    shared = good_desc(n_q_heads=16, n_kv_heads=1, head_dim=512, window=0, kv_shared=True)
    assert app(shared, v=None) == binding.GDATTN_ERR_INVALID_ARG     # K = V: no v_new
    assert app(shared, v=None, v_new=None, q=None) == binding.GDATTN_ERR_INVALID_ARG


def fp8_call(desc, q=A, kc=A, vc=A, ks=A, vs=A, seqlens=A, batch=1, max_seqlen=8, out=A, lse=A,
             ws=A, ws_bytes=1 << 20):
    return binding.decode_fp8_raw(q, kc, vc, ks, vs, seqlens, batch, max_seqlen, desc, out, lse,
                                  ws, ws_bytes, None)


@pytest.mark.parametrize("case,expect", [
    (dict(q=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(kc=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(vc=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(ks=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(vs=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(seqlens=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(out=None), binding.GDATTN_ERR_INVALID_ARG),
    (dict(batch=0), binding.GDATTN_ERR_INVALID_ARG),
    (dict(max_seqlen=0), binding.GDATTN_ERR_INVALID_ARG),
    (dict(q=A + 8), binding.GDATTN_ERR_MISALIGNED),
    (dict(kc=A + 1), binding.GDATTN_ERR_MISALIGNED),
    (dict(vc=A + 8), binding.GDATTN_ERR_MISALIGNED),
    (dict(ks=A + 2), binding.GDATTN_ERR_MISALIGNED),
    (dict(vs=A + 1), binding.GDATTN_ERR_MISALIGNED),
    (dict(out=A + 8), binding.GDATTN_ERR_MISALIGNED),
    (dict(lse=A + 2), binding.GDATTN_ERR_MISALIGNED),
    (dict(ws=None), binding.GDATTN_ERR_WORKSPACE),
    (dict(ws=A + 8), binding.GDATTN_ERR_MISALIGNED),
])
def test_decode_fp8_rejects_bad_pointers(lib, case, expect):
    """gdattn_decode_fp8: the codes need 16-byte alignment (TMA), the scales 4."""
    assert fp8_call(good_desc(), **case) == expect


@pytest.mark.parametrize("desc_kw,expect", [
    (dict(n_q_heads=16, n_kv_heads=1, head_dim=512, window=0, kv_shared=True),
     binding.GDATTN_ERR_UNSUPPORTED),                       # global geometry: bf16 only
    (dict(n_q_heads=8, n_kv_heads=8), binding.GDATTN_ERR_UNSUPPORTED),  # G = 1
    (dict(head_dim=512), binding.GDATTN_ERR_UNSUPPORTED),
    (dict(n_q_heads=12), binding.GDATTN_ERR_INVALID_ARG),
    (dict(cache_batch_stride=1024 * 8 * 256 + 8), binding.GDATTN_ERR_MISALIGNED),  # bytes % 16
])
def test_decode_fp8_rejects_bad_desc(lib, desc_kw, expect):
    assert fp8_call(good_desc(**desc_kw)) == expect


def test_decode_multi_host_checks(lib):
    """gdattn_decode_multi: token count, ring capacity and workspace checked on the host."""
    def multi(desc, T=2, max_seqlen=2048, ws=A, ws_bytes=1 << 24, q=A):
        return binding.decode_multi_raw(q, A, A, A, 1, T, max_seqlen, desc, A, A, ws, ws_bytes,
                                        None)
    d = good_desc(cache_capacity=1030)  # window 1024: room for T <= 7
    assert multi(d, T=0) == binding.GDATTN_ERR_INVALID_ARG
    assert multi(d, T=65) == binding.GDATTN_ERR_INVALID_ARG
    assert multi(d, T=8) == binding.GDATTN_ERR_INVALID_ARG      # C < w + T - 1
    assert multi(good_desc(), T=2) == binding.GDATTN_ERR_INVALID_ARG  # C = w: no room
    assert multi(d, T=2, ws=None) == binding.GDATTN_ERR_WORKSPACE
    assert multi(d, T=2, q=None) == binding.GDATTN_ERR_INVALID_ARG
    assert multi(d, T=2, q=A + 8) == binding.GDATTN_ERR_MISALIGNED
    assert binding.multi_workspace_size(1, 0, 8, good_desc()) == 0


def test_prompt_chunks_allowed_where_flash_prefill_runs(lib):
    """Token limits by geometry: up to 2^20 tokens on the pair geometry and on the
    global geometry with K = V (flash prefill), 64 elsewhere.  A chunk that passes
    the host checks reaches the workspace check (here: no workspace)."""
    def multi(desc, T, ws=None):
        return binding.decode_multi_raw(A, A, None if desc.kv_shared else A, A, 1, T, 1 << 21,
                                        desc, A, A, ws, 1 << 24, None)
    pair = good_desc(window=1024, cache_capacity=1 << 21)  # a cache that never wraps
    assert multi(pair, 65) == binding.GDATTN_ERR_WORKSPACE
    assert multi(pair, 1 << 20) == binding.GDATTN_ERR_WORKSPACE
    assert multi(pair, (1 << 20) + 1) == binding.GDATTN_ERR_INVALID_ARG
    glob = good_desc(n_q_heads=16, n_kv_heads=1, head_dim=512, window=0, kv_shared=True,
                     scale=512 ** -0.5, cache_capacity=1 << 21)
    assert multi(glob, 100) == binding.GDATTN_ERR_WORKSPACE
    sepv = good_desc(n_q_heads=16, n_kv_heads=1, head_dim=512, window=0, kv_shared=False,
                     scale=512 ** -0.5, cache_capacity=1 << 21)
    assert multi(sepv, 64) == binding.GDATTN_ERR_WORKSPACE
    assert multi(sepv, 65) == binding.GDATTN_ERR_INVALID_ARG
    core = good_desc(n_q_heads=8, n_kv_heads=2, head_dim=256, window=0,
                     cache_capacity=1 << 21)
    assert multi(core, 64) == binding.GDATTN_ERR_WORKSPACE
    assert multi(core, 65) == binding.GDATTN_ERR_INVALID_ARG
