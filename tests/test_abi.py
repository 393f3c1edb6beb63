"""The C ABI on the CPU: the library loads, exports every function include/kvattn.h
declares, and rejects bad arguments on the host before any device work (no compute
call is made here: there is no GPU in this test)."""
import ctypes
import os
import re

import pytest

from mla_kv_cache_b200 import binding as kb
from mla_kv_cache_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build(quiet=True)
    return kb.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "kvattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvattn_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("kvattn_gqa_decode", "kvattn_mla_decode", "kvattn_status_string",
                     "kvattn_version", "kvattn_release_workspace"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in kb._SIGNATURES, f"binding lacks {name}"


def test_version_and_status_strings(lib):
    assert lib.kvattn_version() == 10000
    for code, name in [(0, "KVATTN_OK"), (1, "KVATTN_ERR_INVALID_ARG"), (2, "KVATTN_ERR_UNSUPPORTED"),
                       (3, "KVATTN_ERR_MISALIGNED"), (4, "KVATTN_ERR_CUDA"), (5, "KVATTN_ERR_NO_MEMORY")]:
        assert lib.kvattn_status_string(code).decode() == name
    assert lib.kvattn_status_string(99).decode() == "KVATTN_UNKNOWN_STATUS"


# Fake, never-dereferenced, 16-byte aligned "device" addresses far apart from each other.
A = 1 << 40


def gqa_args(**kw):
    args = dict(q=A, k=2 * A, v=3 * A, lens=4 * A, T=512, B=1, nq=8, nkv=2, d=64, scale=0.125,
                out=5 * A, lse=6 * A, stream=None)
    args.update(kw)
    return args


def call_gqa(lib, a):
    return lib.kvattn_gqa_decode(a["q"], a["k"], a["v"], a["lens"], a["T"], a["B"], a["nq"], a["nkv"],
                                 a["d"], a["scale"], a["out"], a["lse"], a["stream"])


@pytest.mark.parametrize("kw,expected", [
    (dict(q=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(k=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(v=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(lens=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(out=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(lse=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(B=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(B=-3), kb.KVATTN_ERR_INVALID_ARG),
    (dict(nq=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(nkv=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(nq=8, nkv=3), kb.KVATTN_ERR_INVALID_ARG),
    (dict(T=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), kb.KVATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), kb.KVATTN_ERR_INVALID_ARG),
    (dict(d=96), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(d=256), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(B=4097), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(B=4096, nkv=8, nq=8, T=1 << 16), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(q=A + 8), kb.KVATTN_ERR_MISALIGNED),
    (dict(k=2 * A + 2), kb.KVATTN_ERR_MISALIGNED),
    (dict(out=5 * A + 4), kb.KVATTN_ERR_MISALIGNED),
    (dict(lse=6 * A + 12), kb.KVATTN_ERR_MISALIGNED),
    (dict(out=2 * A + 64), kb.KVATTN_ERR_INVALID_ARG),      # output overlaps the K cache
    (dict(lse=A), kb.KVATTN_ERR_INVALID_ARG),              # lse overlaps q
])
def test_gqa_rejects_bad_arguments(lib, kw, expected):
    assert call_gqa(lib, gqa_args(**kw)) == expected


def mla_args(**kw):
    args = dict(ql=A, qr=2 * A, lat=3 * A, rope=4 * A, lens=5 * A, T=4096, B=2, H=128, dc=512, dr=64,
                scale=0.0722, out=6 * A, lse=7 * A, stream=None)
    args.update(kw)
    return args


def call_mla(lib, a):
    return lib.kvattn_mla_decode(a["ql"], a["qr"], a["lat"], a["rope"], a["lens"], a["T"], a["B"],
                                 a["H"], a["dc"], a["dr"], a["scale"], a["out"], a["lse"], a["stream"])


@pytest.mark.parametrize("kw,expected", [
    (dict(ql=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(rope=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(lse=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(B=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(H=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(T=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), kb.KVATTN_ERR_INVALID_ARG),
    (dict(H=129), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(dc=256), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(dr=32), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(B=5000), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(B=1025), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(lat=3 * A + 8), kb.KVATTN_ERR_MISALIGNED),
    (dict(out=3 * A), kb.KVATTN_ERR_INVALID_ARG),
])
def test_mla_rejects_bad_arguments(lib, kw, expected):
    assert call_mla(lib, mla_args(**kw)) == expected


def rope_args(**kw):
    args = dict(q=A, kn=2 * A, vn=3 * A, pos=4 * A, kc=5 * A, vc=7 * A, T=1024, B=2, nq=8, nkv=2, d=128,
                base=10000.0, inter=0, stream=None)
    args.update(kw)
    return args


def call_rope(lib, a):
    return lib.kvattn_rope_append(a["q"], a["kn"], a["vn"], a["pos"], a["kc"], a["vc"], a["T"], a["B"],
                                  a["nq"], a["nkv"], a["d"], a["base"], a["inter"], a["stream"])


@pytest.mark.parametrize("kw,expected", [
    (dict(q=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(pos=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(vc=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(B=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(nq=8, nkv=3), kb.KVATTN_ERR_INVALID_ARG),
    (dict(base=0.0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(base=float("nan")), kb.KVATTN_ERR_INVALID_ARG),
    (dict(d=127), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(d=2048), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(kc=5 * A + 4), kb.KVATTN_ERR_MISALIGNED),
    (dict(q=5 * A), kb.KVATTN_ERR_INVALID_ARG),            # q overlaps the K cache
    (dict(kn=7 * A + 64), kb.KVATTN_ERR_INVALID_ARG),      # the new key lies inside the V cache
])
def test_rope_append_rejects_bad_arguments(lib, kw, expected):
    assert call_rope(lib, rope_args(**kw)) == expected


@pytest.mark.parametrize("kw,expected", [
    (dict(dr=63), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(lat=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(rope=4 * A + 2), kb.KVATTN_ERR_MISALIGNED),
])
def test_mla_rope_append_rejects_bad_arguments(lib, kw, expected):
    a = dict(qr=A, ln=2 * A, rn=3 * A, pos=4 * A, lat=5 * A, rope=7 * A, T=1024, B=2, H=128, dc=512, dr=64)
    a.update(kw)
    st = lib.kvattn_mla_rope_append(a["qr"], a["ln"], a["rn"], a["pos"], a["lat"], a["rope"], a["T"], a["B"],
                                    a["H"], a["dc"], a["dr"], 10000.0, 0, None)
    assert st == expected


@pytest.mark.parametrize("kw,expected", [
    (dict(table=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(P=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(S=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(M=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(S=16), kb.KVATTN_ERR_UNSUPPORTED),       # pages must hold whole 64-row tiles
    (dict(S=96), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(d=96), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(table=6 * A + 4), kb.KVATTN_ERR_MISALIGNED),
    (dict(out=7 * A + 32), kb.KVATTN_ERR_INVALID_ARG),    # output overlaps the block table
])
def test_gqa_paged_rejects_bad_arguments(lib, kw, expected):
    a = dict(q=A, k=2 * A, v=3 * A, table=6 * A, lens=5 * A, P=64, S=128, M=8, B=2, nq=8, nkv=2, d=128,
             scale=0.088, out=7 * A, lse=8 * A)
    a.update(kw)
    if kw.get("out") == 7 * A + 32:
        a["table"] = 7 * A
    st = lib.kvattn_gqa_decode_paged(a["q"], a["k"], a["v"], a["table"], a["lens"], a["P"], a["S"], a["M"],
                                     a["B"], a["nq"], a["nkv"], a["d"], a["scale"], a["out"], a["lse"], None)
    assert st == expected


@pytest.mark.parametrize("kw,expected", [
    (dict(S=32), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(dc=256), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(table=0), kb.KVATTN_ERR_INVALID_ARG),
])
def test_mla_paged_rejects_bad_arguments(lib, kw, expected):
    a = dict(ql=A, qr=2 * A, lat=3 * A, rope=4 * A, table=5 * A, lens=6 * A, P=64, S=64, M=8, B=2, H=128,
             dc=512, dr=64, out=7 * A, lse=8 * A)
    a.update(kw)
    st = lib.kvattn_mla_decode_paged(a["ql"], a["qr"], a["lat"], a["rope"], a["table"], a["lens"], a["P"],
                                     a["S"], a["M"], a["B"], a["H"], a["dc"], a["dr"], 0.0722, a["out"],
                                     a["lse"], None)
    assert st == expected


@pytest.mark.parametrize("kw,expected", [
    (dict(L=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(L=513), kb.KVATTN_ERR_UNSUPPORTED),                # batch * q_len > 1024
    (dict(dc=256), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(e4m3=1, ls=0.0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(out=A + 16), kb.KVATTN_ERR_INVALID_ARG),           # output overlaps q_latent
])
def test_mla_multi_rejects_bad_arguments(lib, kw, expected):
    a = dict(ql=A, qr=2 * A, lat=3 * A, rope=4 * A, lens=5 * A, T=4096, B=2, L=4, H=128, dc=512, dr=64, e4m3=0,
             ls=1.0, rs=1.0, out=6 * A, lse=7 * A)
    a.update(kw)
    st = lib.kvattn_mla_decode_multi(a["ql"], a["qr"], a["lat"], a["rope"], a["lens"], a["T"], a["B"], a["L"], a["H"],
                                     a["dc"], a["dr"], 0.0722, a["e4m3"], a["ls"], a["rs"], a["out"], a["lse"], None)
    assert st == expected


@pytest.mark.parametrize("kw,expected", [
    (dict(L=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(window=-1), kb.KVATTN_ERR_INVALID_ARG),
    (dict(L=2049), kb.KVATTN_ERR_UNSUPPORTED),               # batch * q_len > 4096
    (dict(d=96), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(window=5, d=64), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(window=3, nq=128, nkv=1), kb.KVATTN_ERR_UNSUPPORTED),   # a window needs groups of <= 64
    (dict(q=A + 4), kb.KVATTN_ERR_MISALIGNED),
    (dict(out=A + 16), kb.KVATTN_ERR_INVALID_ARG),          # output overlaps q
])
def test_gqa_multi_rejects_bad_arguments(lib, kw, expected):
    a = dict(q=A, k=2 * A, v=3 * A, lens=4 * A, T=4096, B=2, L=4, nq=32, nkv=8, d=128, window=0,
             out=5 * A, lse=6 * A)
    a.update(kw)
    st = lib.kvattn_gqa_decode_multi(a["q"], a["k"], a["v"], a["lens"], a["T"], a["B"], a["L"], a["nq"], a["nkv"],
                                     a["d"], 0.088, a["window"], a["out"], a["lse"], None)
    assert st == expected


@pytest.mark.parametrize("kw,expected", [
    (dict(d=64), kb.KVATTN_ERR_UNSUPPORTED),                 # E4M3 path: head_dim 128 only
    (dict(nq=128, nkv=1), kb.KVATTN_ERR_UNSUPPORTED),        # groups of more than 64 heads
    (dict(L=2049), kb.KVATTN_ERR_UNSUPPORTED),               # batch * q_len > 4096
    (dict(ks=0.0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(vs=-1.0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(ks=float("inf")), kb.KVATTN_ERR_INVALID_ARG),
    (dict(vs=float("nan")), kb.KVATTN_ERR_INVALID_ARG),
    (dict(window=-2), kb.KVATTN_ERR_INVALID_ARG),
    (dict(k=2 * A + 8), kb.KVATTN_ERR_MISALIGNED),
    (dict(out=2 * A + 64), kb.KVATTN_ERR_INVALID_ARG),      # output inside the key cache
    (dict(k=0), kb.KVATTN_ERR_INVALID_ARG),
])
def test_gqa_fp8_rejects_bad_arguments(lib, kw, expected):
    a = dict(q=A, k=2 * A, v=3 * A, lens=4 * A, T=4096, B=2, L=1, nq=32, nkv=8, d=128, ks=0.01, vs=0.02,
             window=0, out=5 * A, lse=6 * A)
    a.update(kw)
    st = lib.kvattn_gqa_decode_fp8(a["q"], a["k"], a["v"], a["lens"], a["T"], a["B"], a["L"], a["nq"], a["nkv"],
                                   a["d"], 0.088, a["ks"], a["vs"], a["window"], a["out"], a["lse"], None)
    assert st == expected


@pytest.mark.parametrize("kw,expected", [
    (dict(S=64), kb.KVATTN_ERR_UNSUPPORTED),                 # pages of whole 128-token tiles
    (dict(d=64), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(table=0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(ks=0.0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(table=6 * A + 4), kb.KVATTN_ERR_MISALIGNED),
])
def test_gqa_fp8_paged_rejects_bad_arguments(lib, kw, expected):
    a = dict(q=A, k=2 * A, v=3 * A, table=6 * A, lens=5 * A, P=64, S=128, M=8, B=2, nq=8, nkv=2, d=128,
             ks=0.01, vs=0.02, out=7 * A, lse=8 * A)
    a.update(kw)
    st = lib.kvattn_gqa_decode_fp8_paged(a["q"], a["k"], a["v"], a["table"], a["lens"], a["P"], a["S"], a["M"],
                                         a["B"], a["nq"], a["nkv"], a["d"], 0.088, a["ks"], a["vs"], a["out"],
                                         a["lse"], None)
    assert st == expected


@pytest.mark.parametrize("kw,expected", [
    (dict(ks=0.0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(vs=float("inf")), kb.KVATTN_ERR_INVALID_ARG),
    (dict(d=7), kb.KVATTN_ERR_UNSUPPORTED),
    (dict(base=-1.0), kb.KVATTN_ERR_INVALID_ARG),
    (dict(kc=2 * A + 4), kb.KVATTN_ERR_MISALIGNED),
    (dict(vc=4 * A + 64), kb.KVATTN_ERR_INVALID_ARG),       # value cache inside the key cache
    (dict(q=0), kb.KVATTN_ERR_INVALID_ARG),
])
def test_rope_append_fp8_rejects_bad_arguments(lib, kw, expected):
    a = dict(q=A, kn=6 * A, vn=7 * A, pos=8 * A, kc=4 * A, vc=5 * A, T=1024, B=2, nq=8, nkv=2, d=128,
             base=10000.0, ks=0.01, vs=0.02)
    a.update(kw)
    st = lib.kvattn_rope_append_fp8(a["q"], a["kn"], a["vn"], a["pos"], a["kc"], a["vc"], a["T"], a["B"], a["nq"],
                                    a["nkv"], a["d"], a["base"], 0, a["ks"], a["vs"], None)
    assert st == expected


def test_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 8, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 2, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        kb.kvattn_gqa_decode(q, k, k, torch.zeros(1, dtype=torch.int32), 0.125)


def test_product_path_does_not_reference_the_oracle():
    """The library sources and the binding never name the oracle (no CPU fallback)."""
    pkg = os.path.join(ROOT, "mla_kv_cache_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "kvattn_oracle" not in text, f
