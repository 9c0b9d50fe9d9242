"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments before anything is enqueued.

No test here launches a kernel: every call below carries an argument the
library must refuse on the host, so the same tests are safe on a GPU machine.
"""
import ctypes
import os
import re

import pytest
import torch

from llama_gqa_causal_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "llama_attn.h")

FAKE = 0x10000  # a 16-byte aligned non-null address; never dereferenced (calls are rejected first)


@pytest.fixture(scope="module")
def lib():
    build.build()
    return api.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(llama_\w+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert declared_functions() == sorted(api.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_abi_version_and_status_strings(lib):
    assert lib.llama_attn_abi_version() == 120
    assert api.status_string(0) == "ok"
    assert "invalid" in api.status_string(1)
    assert "unsupported" in api.status_string(2)
    assert "CUDA" in api.status_string(3)
    assert "timed out" in api.status_string(4)
    assert api.status_string(99) == "unknown status"


def test_workspace_sizes(lib):
    # prefill: rotated K in bf16 when RoPE is on, nothing otherwise / for fp32
    assert lib.llama_attn_prefill_workspace_bytes(1, 64, 8, 8192, 128, 1, 1) == 8192 * 8 * 128 * 2
    assert lib.llama_attn_prefill_workspace_bytes(1, 64, 8, 8192, 128, 1, 0) == 0
    assert lib.llama_attn_prefill_workspace_bytes(1, 4, 2, 64, 64, 0, 1) == 0
    # decode: one partial row of D + 4 floats per (b, head) and per (CTA, head of
    # an 8-head chunk) for up to 256 CTAs, then the chunk prefix over the batch
    # ([b + 1] int32 in 256-byte units); independent of the cache length
    def dec(b, H, D):
        return (b * H + 256 * 8) * (D + 4) * 4 + ((b + 1) * 4 + 255) // 256 * 256
    assert lib.llama_attn_decode_workspace_bytes(32, 64, 4096, 128) == dec(32, 64, 128)
    assert lib.llama_attn_decode_workspace_bytes(2, 4, 513, 64) == dec(2, 4, 64)
    assert lib.llama_attn_decode_workspace_bytes(2, 4, 1 << 20, 64) == dec(2, 4, 64)
    assert lib.llama_attn_decode_workspace_bytes(4096, 8, 64, 64) == dec(4096, 8, 64)
    assert lib.llama_attn_decode_workspace_bytes(0, 4, 513, 64) == 0


def _prefill(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, cos=None, sin=None, bsz=1, H=4, Hkv=2, S=64, D=64,
             scale=0.125, causal=1, out=FAKE, mask=None, dtype=1, ws=None, ws_bytes=0, stream=None)
    a.update(kw)
    return lib.llama_attn_prefill(a["q"], a["k"], a["v"], a["cos"], a["sin"], a["bsz"], a["H"],
                                  a["Hkv"], a["S"], a["D"], a["scale"], a["causal"], a["out"],
                                  a["mask"], a["dtype"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1),
    (dict(out=None), 1),
    (dict(v=None), 1),
    (dict(bsz=0), 1),
    (dict(S=0), 1),
    (dict(H=0), 1),
    (dict(H=6, Hkv=4), 1),            # n_heads % n_kv_heads != 0 (divisibility, as TP demands)
    (dict(D=63), 1),                  # odd head_dim: rotate-half needs pairs
    (dict(cos=FAKE), 1),              # cos without sin
    (dict(scale=float("nan")), 1),
    (dict(scale=float("inf")), 1),
    (dict(dtype=7), 1),
    (dict(q=FAKE + 8), 1),            # misaligned
    (dict(mask=FAKE + 4), 1),
    (dict(cos=FAKE, sin=FAKE, ws=None, ws_bytes=0), 1),        # RoPE needs the K workspace
    (dict(cos=FAKE, sin=FAKE, ws=FAKE, ws_bytes=64 * 2 * 64), 1),  # too small by half
    (dict(D=96), 2),                  # valid but no kernel for this head_dim
    (dict(D=256), 2),
])
def test_prefill_rejects(lib, kw, status):
    assert _prefill(lib, **kw) == status


def _decode(lib, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, lens=FAKE, cos=None, sin=None, bsz=2, H=8, Hkv=2, L=100,
             D=128, scale=0.1, out=FAKE, ws=FAKE, ws_bytes=1 << 30, dtype=1, stream=None)
    a.update(kw)
    return lib.llama_attn_decode(a["q"], a["kc"], a["vc"], a["lens"], a["cos"], a["sin"], a["bsz"],
                                 a["H"], a["Hkv"], a["L"], a["D"], a["scale"], a["out"], a["ws"],
                                 a["ws_bytes"], a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(lens=None), 1),
    (dict(kc=None), 1),
    (dict(L=0), 1),
    (dict(H=8, Hkv=3), 1),
    (dict(D=7), 1),
    (dict(sin=FAKE), 1),
    (dict(ws=None), 1),
    (dict(ws_bytes=100), 1),
    (dict(lens=FAKE + 2), 1),
    (dict(vc=FAKE + 4), 1),
    (dict(dtype=-1), 1),
    (dict(D=80), 2),
    (dict(bsz=4097), 2),
])
def test_decode_rejects(lib, kw, status):
    assert _decode(lib, **kw) == status


def _prefill_window(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, cos=None, sin=None, bsz=1, H=8, Hkv=2, S=100, D=128, scale=0.1,
             window=16, out=FAKE, dtype=1, ws=None, ws_bytes=0, stream=None)
    a.update(kw)
    return lib.llama_attn_prefill_window(a["q"], a["k"], a["v"], a["cos"], a["sin"], a["bsz"],
                                         a["H"], a["Hkv"], a["S"], a["D"], a["scale"], a["window"],
                                         a["out"], a["dtype"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(window=0), 1),
    (dict(window=-4), 1),
    (dict(q=None), 1),
    (dict(S=0), 1),
    (dict(H=8, Hkv=3), 1),
    (dict(out=FAKE + 2), 1),
    (dict(cos=FAKE), 1),                  # sin missing
    (dict(cos=FAKE, sin=FAKE), 1),        # RoPE needs the K-rotation workspace
    (dict(dtype=0), 2),
    (dict(D=96), 2),
])
def test_prefill_window_rejects(lib, kw, status):
    assert _prefill_window(lib, **kw) == status


def _prefill_varlen(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, cos=None, sin=None, lens=FAKE, bsz=2, H=8, Hkv=2, S=100, D=128,
             scale=0.1, causal=1, out=FAKE, dtype=1, ws=None, ws_bytes=0, stream=None)
    a.update(kw)
    return lib.llama_attn_prefill_varlen(a["q"], a["k"], a["v"], a["cos"], a["sin"], a["lens"],
                                         a["bsz"], a["H"], a["Hkv"], a["S"], a["D"], a["scale"],
                                         a["causal"], a["out"], a["dtype"], a["ws"], a["ws_bytes"],
                                         a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(lens=None), 1),
    (dict(lens=FAKE + 2), 1),
    (dict(q=None), 1),
    (dict(S=0), 1),
    (dict(H=8, Hkv=3), 1),
    (dict(cos=FAKE, sin=FAKE), 1),        # RoPE needs the K-rotation workspace
    (dict(dtype=0), 2),
    (dict(D=96), 2),
])
def test_prefill_varlen_rejects(lib, kw, status):
    assert _prefill_varlen(lib, **kw) == status


def _prefill_packed(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, cos=None, sin=None, cu=FAKE, n=3, T=300, maxlen=128, H=8,
             Hkv=2, D=128, scale=0.1, causal=1, out=FAKE, dtype=1, ws=None, ws_bytes=0,
             stream=None)
    a.update(kw)
    return lib.llama_attn_prefill_packed(a["q"], a["k"], a["v"], a["cos"], a["sin"], a["cu"],
                                         a["n"], a["T"], a["maxlen"], a["H"], a["Hkv"], a["D"],
                                         a["scale"], a["causal"], a["out"], a["dtype"], a["ws"],
                                         a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(cu=None), 1),
    (dict(cu=FAKE + 2), 1),
    (dict(T=0), 1),
    (dict(maxlen=0), 1),
    (dict(n=0), 1),
    (dict(H=8, Hkv=3), 1),
    (dict(cos=FAKE, sin=FAKE), 1),        # RoPE needs the K-rotation workspace
    (dict(dtype=0), 2),
    (dict(D=96), 2),
])
def test_prefill_packed_rejects(lib, kw, status):
    assert _prefill_packed(lib, **kw) == status


@pytest.mark.parametrize("args", [
    (FAKE, 1, 4, 64, 1e4, 0.0, FAKE, FAKE),    # alpha must be positive
    (FAKE, 1, 4, 64, 1e4, -2.0, FAKE, FAKE),
    (FAKE, 1, 4, 2, 1e4, 2.0, FAKE, FAKE),     # head_dim 2 has no D - 2
    (None, 1, 4, 64, 1e4, 2.0, FAKE, FAKE),
    (FAKE, 1, 4, 64, 1e300, 1e300, FAKE, FAKE),  # base overflows
])
def test_rope_table_ntk_rejects(lib, args):
    assert lib.llama_rope_table_ntk(*args, None) == 1


def _qkv(lib, **kw):
    a = dict(x=FAKE, w=FAKE, cos=None, sin=None, T=10, hidden=64, H=8, Hkv=2, D=128, q=FAKE, k=FAKE,
             v=FAKE, dtype=1, stream=None)
    a.update(kw)
    return lib.llama_attn_qkv_rope(a["x"], a["w"], a["cos"], a["sin"], a["T"], a["hidden"], a["H"],
                                   a["Hkv"], a["D"], a["q"], a["k"], a["v"], a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), 1), (dict(w=None), 1), (dict(v=None), 1),
    (dict(T=0), 1), (dict(hidden=0), 1), (dict(hidden=60), 1),
    (dict(H=8, Hkv=3), 1), (dict(cos=FAKE), 1), (dict(q=FAKE + 2), 1),
    (dict(dtype=0), 2), (dict(D=96), 2),
])
def test_qkv_rope_rejects(lib, kw, status):
    assert _qkv(lib, **kw) == status


@pytest.mark.parametrize("args,status", [
    ((None, FAKE, 10, 64, 64, FAKE, 1, None), 1),
    ((FAKE, FAKE, 0, 64, 64, FAKE, 1, None), 1),
    ((FAKE, FAKE, 10, 60, 64, FAKE, 1, None), 1),
    ((FAKE, FAKE, 10, 64, 65, FAKE, 1, None), 1),
    ((FAKE, FAKE, 10, 64, 64, FAKE + 4, 1, None), 1),
    ((FAKE, FAKE, 10, 64, 64, FAKE, 0, None), 2),
])
def test_out_proj_rejects(lib, args, status):
    assert lib.llama_attn_out_proj(*args) == status


def _decode_append(lib, **kw):
    a = dict(q=FAKE, kn=FAKE, vn=FAKE, kc=FAKE, vc=FAKE, lens=FAKE, cos=None, sin=None, bsz=2, H=8,
             Hkv=2, L=100, D=128, scale=0.1, out=FAKE, ws=FAKE, ws_bytes=1 << 30, dtype=1,
             stream=None)
    a.update(kw)
    return lib.llama_attn_decode_append(a["q"], a["kn"], a["vn"], a["kc"], a["vc"], a["lens"],
                                        a["cos"], a["sin"], a["bsz"], a["H"], a["Hkv"], a["L"],
                                        a["D"], a["scale"], a["out"], a["ws"], a["ws_bytes"],
                                        a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(kn=None), 1),
    (dict(vn=None), 1),
    (dict(kc=None), 1),
    (dict(vn=FAKE + 4), 1),
    (dict(kn=FAKE + 8), 1),
    (dict(L=0), 1),
    (dict(ws_bytes=100), 1),
    (dict(H=8, Hkv=3), 1),
    (dict(dtype=0), 2),
    (dict(D=80), 2),
    (dict(bsz=4097), 2),
])
def test_decode_append_rejects(lib, kw, status):
    assert _decode_append(lib, **kw) == status


@pytest.mark.parametrize("args", [
    (None, 1, 4, 64, 1e4, 1.0, FAKE, FAKE),
    (FAKE, 0, 4, 64, 1e4, 1.0, FAKE, FAKE),
    (FAKE, 1, 4, 63, 1e4, 1.0, FAKE, FAKE),
    (FAKE, 1, 4, 64, 0.0, 1.0, FAKE, FAKE),
    (FAKE, 1, 4, 64, 1e4, -2.0, FAKE, FAKE),
    (FAKE, 1, 4, 64, 1e4, 1.0, None, FAKE),
])
def test_rope_table_rejects(lib, args):
    assert lib.llama_rope_table(*args, None) == 1


def test_decode_noalloc_refuses_what_its_static_scratch_cannot_hold(lib):
    # 35.7 MB of partials needed (1024 x 64 heads); the library's fixed scratch is 16 MiB
    assert lib.llama_attn_decode_noalloc(FAKE, FAKE, FAKE, FAKE, None, None, 1024, 64, 8, 4096, 128,
                                         0.088, FAKE, 1, None) == 1
    # argument checks are the regular decode's
    assert lib.llama_attn_decode_noalloc(FAKE, FAKE, FAKE, None, None, None, 2, 8, 2, 100, 128,
                                         0.1, FAKE, 1, None) == 1


def test_python_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        api.prefill(q, q[:, :, :1], q[:, :, :1], causal=True)


def test_build_flags_target_sm100a():
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.FLAGS)


def test_loader_refuses_a_library_built_from_other_sources(lib, monkeypatch):
    # A library whose recorded source hash differs from the tree's sources
    # would run old kernels under new tests; the loader must refuse it.
    assert build.built_hash() == build.source_hash()
    monkeypatch.setattr(api, "_lib", None)
    monkeypatch.setattr(build, "built_hash", lambda: "0" * 64)
    with pytest.raises(RuntimeError, match="other sources"):
        api.load()
    monkeypatch.undo()
    assert api.load() is not None


def test_loader_fails_loudly_without_the_library(tmp_path, monkeypatch):
    # No CPU fallback: without the built library every entry point raises.
    monkeypatch.setattr(api, "_lib", None)
    monkeypatch.setattr(api, "LIB_PATH", str(tmp_path / "libllama_attn.so"))
    with pytest.raises(RuntimeError, match="is missing"):
        api.load()
    with pytest.raises(RuntimeError, match="is missing"):
        api.rope_table(torch.zeros(1, 4, dtype=torch.int64), 128)
    monkeypatch.undo()
    assert api.load() is not None


def _bf(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


@pytest.mark.parametrize("call,match", [
    (lambda: api.prefill(_bf(1, 8, 4, 64), _bf(1, 7, 2, 64), _bf(1, 8, 2, 64)), "k must have shape"),
    (lambda: api.prefill(_bf(1, 8, 4, 64), _bf(1, 8, 2, 64), _bf(1, 8, 2, 64).float()),
     "v must be torch.bfloat16"),
    (lambda: api.prefill(_bf(1, 8, 4, 64), _bf(1, 8, 2, 64), _bf(1, 8, 2, 64),
                         torch.zeros(1, 8, 64)), "both cos and sin"),
    (lambda: api.prefill(_bf(1, 8, 4, 64), _bf(1, 8, 2, 64), _bf(1, 8, 2, 64),
                         torch.zeros(1, 8, 32), torch.zeros(1, 8, 32)), "cos must hold 512"),
    (lambda: api.prefill(_bf(1, 8, 4, 64), _bf(1, 8, 2, 64), _bf(1, 8, 2, 64),
                         mask=torch.zeros(1, 1, 8, 7)), "mask must hold 64"),
    (lambda: api.prefill(_bf(1, 8, 4, 64), _bf(1, 8, 2, 64), _bf(1, 8, 2, 64),
                         out=_bf(1, 8, 128)), "out must hold 2048"),
    (lambda: api.prefill_window(_bf(1, 8, 4, 64), _bf(1, 8, 2, 64), _bf(1, 8, 1, 64), window=4),
     "v must have shape"),
    (lambda: api.prefill_varlen(_bf(2, 8, 4, 64), _bf(2, 8, 2, 64), _bf(2, 8, 2, 64),
                                torch.zeros(3, dtype=torch.int32)), "seq_lens must hold 2"),
    (lambda: api.prefill_packed(_bf(10, 4, 64), _bf(9, 2, 64), _bf(10, 2, 64),
                                torch.tensor([0, 10], dtype=torch.int32), 10), "k must have shape"),
    (lambda: api.decode(_bf(2, 8, 64), _bf(2, 2, 16, 64), _bf(2, 2, 15, 64),
                        torch.zeros(2, dtype=torch.int32)), "v_cache must have shape"),
    (lambda: api.decode(_bf(2, 8, 64), _bf(2, 2, 16, 64), _bf(2, 2, 16, 64),
                        torch.zeros(2, dtype=torch.int64)), "cache_lens must be torch.int32"),
    (lambda: api.decode_append(_bf(2, 8, 64), _bf(2, 2, 64), _bf(2, 2, 64), _bf(2, 2, 16, 64),
                               _bf(2, 2, 16, 64), torch.zeros(1, dtype=torch.int32)),
     "cache_lens must hold 2"),
    (lambda: api.decode_noalloc(_bf(2, 8, 64), _bf(2, 2, 16, 64), _bf(2, 2, 16, 64),
                                torch.zeros(2, dtype=torch.int32), out=_bf(2, 256)),
     "out must hold 1024"),
    (lambda: api.qkv_rope(_bf(5, 32), _bf(3 * 64, 32), 2, 1, 64), "w_qkv must have shape"),
    (lambda: api.out_proj(_bf(5, 32), _bf(16, 31)), "w_o must have shape"),
])
def test_python_binding_checks_tensor_sizes_before_any_launch(lib, call, match):
    # the C ABI sees only pointers: the binding refuses tensors that disagree
    # with the sizes it passes (checked before the device check, so on CPU here)
    with pytest.raises(ValueError, match=match):
        call()


def test_header_is_plain_c_and_links(lib, tmp_path):
    # the boundary is a C ABI: a strict C99 program includes the header, links
    # against the library and calls its host-only entry points
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(
        "#include <stdio.h>\n#include \"llama_attn.h\"\n"
        "int main(void) {\n"
        "  printf(\"%d|%s|%zu\\n\", llama_attn_abi_version(),\n"
        "         llama_attn_status_string(LLAMA_ERR_UNSUPPORTED),\n"
        "         llama_attn_decode_workspace_bytes(32, 64, 4096, 128));\n"
        "  return 0;\n}\n")
    libdir = os.path.dirname(build.LIB)
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", build.INCLUDE, str(src), "-L", libdir, "-lllama_attn",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.strip()
    version, status, ws = out.split("|")
    assert int(version) == lib.llama_attn_abi_version()
    assert status == api.status_string(api.LLAMA_ERR_UNSUPPORTED)
    assert int(ws) == api.decode_workspace_bytes(32, 64, 4096, 128)


@pytest.mark.parametrize("limit_us", [0, 1000001, 1 << 31])
def test_selftest_wait_timeout_rejects_limits_outside_its_range(lib, limit_us):
    assert lib.llama_attn_selftest_wait_timeout(limit_us, None) == api.LLAMA_ERR_INVALID_ARG
