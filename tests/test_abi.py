"""Host-side checks of the C ABI that need no GPU: the library builds and loads,
exports every entry point include/b200attn.h declares, and rejects bad
arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "b200attn.h")


@pytest.fixture(scope="module")
def lib():
    from bf16_causal_prefill_fwd_b200 import build
    build.build()
    from bf16_causal_prefill_fwd_b200 import _binding
    return _binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(b200attn_\w+)\s*\(", text, re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("b200attn_fwd", "b200attn_quantize_fp8", "b200attn_quantize_workspace_bytes",
                 "b200attn_check", "b200attn_strerror", "b200attn_version"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    from bf16_causal_prefill_fwd_b200 import LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r" T (b200attn_\w+)$", out, re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_version_and_strerror(lib):
    text = open(HEADER).read()
    ver = int(re.search(r"#define B200ATTN_VERSION (\d+)", text).group(1))
    assert lib.b200attn_version() == ver
    for code in (0, -1, -2, -3, -4, -5, 12345):
        assert isinstance(lib.b200attn_strerror(code), bytes)
    assert lib.b200attn_strerror(-4) != lib.b200attn_strerror(-1)


FAKE = 0x10000  # a 16-byte aligned non-NULL value; never dereferenced on these paths


def fwd(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, B=1, Hq=4, Hkv=2, N=64, dqk=128, dv=128, causal=1, dtype=0,
        qs=None, ks=None, vs=None, gran=0, scale=0.0, lse=None):
    return lib.b200attn_fwd(q, k, v, o, B, Hq, Hkv, N, dqk, dv, causal, dtype, qs, ks, vs, gran, scale, lse, None)


def test_fwd_rejects_bad_arguments_on_the_host(lib):
    assert fwd(lib, q=None) == -1
    assert fwd(lib, o=None) == -1
    assert fwd(lib, B=0) == -1
    assert fwd(lib, N=0) == -1
    assert fwd(lib, Hq=3, Hkv=2) == -1
    assert fwd(lib, causal=2) == -1
    assert fwd(lib, q=FAKE + 8) == -1                       # misaligned
    assert fwd(lib, lse=FAKE + 2) == -1                     # misaligned lse
    assert fwd(lib, dtype=1) == -1                          # FP8 without scales
    assert fwd(lib, scale=float("nan")) == -1


def test_fwd_reports_unsupported_shapes_on_the_host(lib):
    assert fwd(lib, dqk=64, dv=64) == -2
    assert fwd(lib, dqk=128, dv=192) == -2
    assert fwd(lib, dtype=7) == -2
    assert fwd(lib, dtype=1, qs=FAKE, ks=FAKE, vs=FAKE, gran=5) == -2
    # the kernels index (b, n, h) rows in 32 bits: B*N*max(Hq, Hkv) must stay below 2^31
    assert fwd(lib, B=1, N=1 << 26, Hq=32, Hkv=8) == -2
    assert fwd(lib, B=1 << 10, N=1 << 16, Hq=32, Hkv=8) == -2


def test_quantize_workspace_size(lib):
    assert lib.b200attn_quantize_workspace_bytes(1, 16384, 32, 128, 0) == 1 * 32 * 128 * 4
    assert lib.b200attn_quantize_workspace_bytes(2, 300, 8, 128, 0) == 2 * 8 * 3 * 4
    assert lib.b200attn_quantize_workspace_bytes(2, 300, 8, 128, 1) == 0
    assert lib.b200attn_quantize_workspace_bytes(0, 300, 8, 128, 0) == 0


def test_quantize_rejects_bad_arguments_on_the_host(lib):
    q = lib.b200attn_quantize_fp8
    assert q(None, FAKE, FAKE, 1, 10, 1, 128, 0, 0, FAKE, 64, None) == -1
    assert q(FAKE, FAKE, FAKE, 1, 0, 1, 128, 0, 0, FAKE, 64, None) == -1
    assert q(FAKE, FAKE, FAKE, 1, 10, 1, 64, 0, 0, FAKE, 64, None) == -2
    assert q(FAKE, FAKE, FAKE, 1, 10, 1, 128, 3, 0, FAKE, 64, None) == -2
    assert q(FAKE, FAKE, FAKE, 1, 10, 1, 128, 0, 2, FAKE, 64, None) == -1
    assert q(FAKE + 4, FAKE, FAKE, 1, 10, 1, 128, 0, 0, FAKE, 64, None) == -1
    assert q(FAKE, FAKE, FAKE, 1, 10, 1, 128, 0, 0, None, 0, None) == -5     # per-head needs a workspace
    assert q(FAKE, FAKE, FAKE, 1, 300, 2, 128, 0, 0, FAKE, 8, None) == -5    # too small
    assert q(FAKE, FAKE, FAKE, 1, 300, 65536, 128, 1, 0, None, 0, None) == -2  # more heads than a grid dimension
    assert q(FAKE, FAKE, FAKE, 65536, 300, 1, 128, 1, 0, None, 0, None) == -2  # batch beyond a grid dimension


def test_binding_refuses_cpu_tensors():
    import torch
    import bf16_causal_prefill_fwd_b200 as b
    x = torch.zeros(1, 8, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        b.attn_fwd(x, x, x)
    with pytest.raises(ValueError):
        b.quantize_fp8(x)


def test_package_has_no_oracle_dependency():
    """The product path never imports the oracle (it is test infrastructure)."""
    pkg = os.path.join(ROOT, "bf16_causal_prefill_fwd_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", text, re.M), f
                assert "attn_oracle" not in text and "liboracle" not in text, f


def qkv(lib, ptr=FAKE, B=1, N=256, Hq=4, Hkv=2, dqk=128, dv=128, gran=0, had=0, ws=FAKE, wsb=1 << 20):
    p = [ptr] * 9
    return lib.b200attn_quantize_qkv_fp8(*p, B, N, Hq, Hkv, dqk, dv, gran, had, ws, wsb, None)


def test_quantize_qkv_workspace_and_arguments_on_the_host(lib):
    # one partial absmax per 128-token block of every Q, K and V head
    assert lib.b200attn_quantize_qkv_workspace_bytes(2, 300, 4, 2, 0) == 2 * (4 + 2 * 2) * 3 * 4
    assert lib.b200attn_quantize_qkv_workspace_bytes(2, 300, 4, 2, 1) == 0
    assert lib.b200attn_quantize_qkv_workspace_bytes(0, 300, 4, 2, 0) == 0
    assert qkv(lib, ptr=None) == -1
    assert qkv(lib, ptr=FAKE + 4) == -1                     # misaligned
    assert qkv(lib, N=0) == -1
    assert qkv(lib, had=2) == -1
    assert qkv(lib, dqk=64) == -2
    assert qkv(lib, dv=192) == -2
    assert qkv(lib, gran=3) == -2
    assert qkv(lib, N=65536 * 128) == -2                    # more token blocks than a grid dimension holds
    assert qkv(lib, ws=None) == -5
    assert qkv(lib, wsb=8) == -5


def test_varlen_workspace_and_arguments_on_the_host(lib):
    # bounded from the sizes: 16-byte header, then Hq * (total // 256 + batch) units of 16 bytes
    assert lib.b200attn_fwd_varlen_workspace_bytes(3, 400, 4) == 16 + 16 * 4 * (400 // 256 + 3)
    assert lib.b200attn_fwd_varlen_workspace_bytes(0, 400, 4) == 0

    def call(cu=FAKE, batch=2, total=400, ws=FAKE, wsb=1 << 20, dtype=0, q=FAKE):
        return lib.b200attn_fwd_varlen(q, FAKE, FAKE, FAKE, cu, batch, total, 4, 2, 128, 128, 1,
                                       dtype, None, None, None, 0.0, None, ws, wsb, None)
    # cu_seqlens is read on the device only; what the host can check it checks
    assert call(cu=None) == -1
    assert call(cu=FAKE + 2) == -1                   # misaligned int array
    assert call(batch=0) == -1
    assert call(q=None) == -1
    assert call(dtype=1) == -1                       # FP8 without scales
    assert call(ws=None) == -5
    assert call(wsb=16) == -5
    assert call(total=(1 << 21) + 1) == -2           # above the device-side unit builder's limit
    assert call(total=0, q=None) == 0                # only empty sequences: nothing to do


def test_q_block_granularity_on_the_host(lib):
    # Q per 128-token block needs no partial absmax: only K's and V's
    assert lib.b200attn_quantize_qkv_workspace_bytes(2, 300, 4, 2, 2) == 2 * (2 * 2) * 3 * 4
    assert qkv(lib, gran=2, wsb=8) == -5
    assert fwd(lib, dtype=1, qs=FAKE, ks=FAKE, vs=FAKE, gran=3) == -2


def header_prototypes():
    """{name: (return C type, [parameter C types])} for every entry point in the header."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    protos = {}
    for ret, name, params in re.findall(r"((?:const\s+)?\w+\s*\**)\s*(b200attn_\w+)\s*\(([^)]*)\)\s*;", text):
        types = []
        for p in params.split(","):
            p = " ".join(p.split())
            if not p or p == "void":
                continue
            types.append(re.sub(r"\s*\b\w+$", "", p).replace(" *", "*"))   # drop the parameter name
        protos[name] = (" ".join(ret.split()).replace(" *", "*"), types)
    return protos


def ctype_of(c):
    if c.endswith("*"):
        base = c.replace("const", "").replace("*", "").strip()
        if base == "char":
            return ctypes.c_char_p
        return ctypes.c_void_p  # every pointer argument is a device (or caller-owned) address
    return {"int": ctypes.c_int, "float": ctypes.c_float, "size_t": ctypes.c_size_t}[c]


def test_binding_argtypes_match_header_prototypes(lib):
    """Every entry point the binding declares to ctypes has the header's parameter list:
    a wrong count or type would pass garbage to the library without an error."""
    protos = header_prototypes()
    assert set(protos) == set(declared_functions())
    checked = 0
    for name, (ret, params) in protos.items():
        fn = getattr(lib, name)
        if fn.argtypes is None:
            continue  # not declared by the binding (called only through raw ctypes in tests)
        assert list(fn.argtypes) == [ctype_of(p) for p in params], name
        assert fn.restype == ctype_of(ret), name
        checked += 1
    assert checked >= 10
