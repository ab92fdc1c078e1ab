"""The C ABI on the host: the library loads, exports every symbol the header declares,
rejects invalid arguments before touching the GPU, and the heuristic is sane."""
import ctypes
import os
import re
import subprocess

import pytest

import gqa_exact_attention_b200 as G

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa_attn.h")


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"GQA_API\s+[\w\s\*]+?\b(gqa_attn_\w+)\s*\(", txt)))


def test_header_declares_the_entry_points():
    assert declared_symbols() == sorted([
        "gqa_attn_fwd", "gqa_attn_choose", "gqa_attn_workspace_bytes",
        "gqa_attn_status_string", "gqa_attn_device_status", "gqa_attn_fwd_noalloc",
        "gqa_attn_fwd_kvcache", "gqa_attn_fwd_paged", "gqa_attn_fwd_fp8"])


def test_library_exports_every_declared_symbol():
    L = G.load()
    for name in declared_symbols():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", G.lib_path], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(declared_symbols()) <= exported
    # nothing else of ours leaks: the C ABI is the only interface
    ours = {s for s in exported if s.startswith("gqa")}
    assert ours == set(declared_symbols())


def test_header_compiles_as_c():
    src = f'#include "{HEADER}"\nint main(void) {{ return (int)GQA_OK; }}\n'
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-x", "c", "-", "-o", os.devnull],
                       input=src, text=True, capture_output=True)
    assert r.returncode == 0, r.stderr


NULL = None


def fwd_raw(q=16, k=16, v=16, out=16, lse=16, B=1, Sq=8, Sk=8, Hq=4, Hk=2, d=64, scale=0.125,
            causal=0, pack=-1, splits=0):
    L = G.load()
    return L.gqa_attn_fwd(q, k, v, out, lse, B, Sq, Sk, Hq, Hk, d, scale, causal, pack, splits, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), 1), (dict(k=NULL), 1), (dict(v=NULL), 1), (dict(out=NULL), 1), (dict(lse=NULL), 1),
    (dict(B=0), 2), (dict(Sq=0), 2), (dict(Sk=-1), 2), (dict(Hq=0), 2), (dict(Hk=0), 2),
    (dict(pack=2), 2), (dict(pack=-2), 2), (dict(splits=-1), 2),
    (dict(Hq=6, Hk=4), 3), (dict(Hq=5, Hk=2), 3),
    (dict(d=96), 4), (dict(d=256), 4), (dict(d=0), 4),
    (dict(q=24), 5), (dict(out=8), 5), (dict(lse=4), 5),
    (dict(scale=float("nan")), 2), (dict(scale=float("inf")), 2),
    (dict(Hq=256, Hk=1, pack=1), 2),
    (dict(B=1 << 16, Sq=1 << 12, Hq=1 << 4), 2),
])
def test_invalid_arguments_return_before_any_launch(kw, code):
    # the pointers are fake: validation must reject before anything dereferences them
    assert fwd_raw(**kw) == code
    assert G.gqa_attn_status_string(code)


def kvcache_raw(q=16, k=16, v=16, seqlens=NULL, out=16, out_dtype=0, lse=16, B=1, Sq=8, Sk=8,
                Hq=4, Hk=2, d=64, scale=0.125, causal=0, pack=-1, splits=0):
    L = G.load()
    return L.gqa_attn_fwd_kvcache(q, k, v, seqlens, out, out_dtype, lse, B, Sq, Sk, Hq, Hk, d,
                                  scale, causal, pack, splits, None)


@pytest.mark.parametrize("kw,code", [
    (dict(out_dtype=2), 2), (dict(out_dtype=-1), 2),
    (dict(q=NULL), 1), (dict(out=NULL), 1), (dict(lse=NULL), 1),
    (dict(seqlens=18), 5), (dict(out=8), 5),
    (dict(Hq=6, Hk=4), 3), (dict(d=96), 4), (dict(B=0), 2),
])
def test_kvcache_invalid_arguments(kw, code):
    # fake pointers again: rejected before any launch or dereference (a 4-byte-misaligned
    # cache_seqlens included)
    assert kvcache_raw(**kw) == code


def paged_raw(q=16, kp=16, vp=16, table=16, max_pages=4, seqlens=32, num_pages=8, page_size=16,
              out=16, out_dtype=0, lse=16, B=1, Sq=8, Hq=4, Hk=2, d=64, scale=0.125, causal=0,
              pack=-1, splits=0):
    L = G.load()
    return L.gqa_attn_fwd_paged(q, kp, vp, table, max_pages, seqlens, num_pages, page_size, out,
                                out_dtype, lse, B, Sq, Hq, Hk, d, scale, causal, pack, splits, None)


@pytest.mark.parametrize("kw,code", [
    (dict(out_dtype=2), 2), (dict(max_pages=0), 2), (dict(page_size=0), 2),
    (dict(page_size=8), 2), (dict(page_size=24), 2), (dict(page_size=96), 2), (dict(num_pages=0), 2),
    (dict(table=NULL), 1), (dict(seqlens=NULL), 1), (dict(kp=NULL), 1), (dict(out=NULL), 1),
    (dict(table=18), 5), (dict(kp=24), 5), (dict(seqlens=34), 5),
    (dict(Hq=6, Hk=4), 3), (dict(d=96), 4), (dict(B=0), 2),
    (dict(max_pages=1 << 20, page_size=1 << 12), 2),
    (dict(num_pages=1 << 20, page_size=1 << 10, Hk=4, Hq=4), 2),
])
def test_paged_invalid_arguments(kw, code):
    # fake pointers: every check happens on the host before anything is launched or read
    assert paged_raw(**kw) == code


def fp8_raw(q=16, k=16, v=16, qs=1.0, ks=1.0, vs=1.0, seqlens=NULL, out=16, out_dtype=0, lse=16,
            B=1, Sq=8, Sk=8, Hq=4, Hk=2, d=64, scale=0.125, causal=0, pack=-1, splits=0):
    L = G.load()
    return L.gqa_attn_fwd_fp8(q, k, v, qs, ks, vs, seqlens, out, out_dtype, lse, B, Sq, Sk, Hq,
                              Hk, d, scale, causal, pack, splits, None)


@pytest.mark.parametrize("kw,code", [
    (dict(qs=0.0), 2), (dict(ks=-1.0), 2), (dict(vs=float("inf")), 2), (dict(qs=float("nan")), 2),
    (dict(out_dtype=3), 2), (dict(q=NULL), 1), (dict(v=NULL), 1), (dict(lse=NULL), 1),
    (dict(q=24), 5), (dict(seqlens=18), 5), (dict(Hq=6, Hk=4), 3), (dict(d=96), 4), (dict(Sk=0), 2),
])
def test_fp8_invalid_arguments(kw, code):
    # fake pointers: rejected on the host before anything is launched or read
    assert fp8_raw(**kw) == code


def test_pages_head_constraint_example():
    """Hq must be a multiple of Hk (the pages' interface constraint); Hq=6, Hk=2 is valid."""
    L = G.load()
    pk, ns = ctypes.c_int(), ctypes.c_int()
    assert L.gqa_attn_choose(1, 128, 128, 6, 2, 64, 1, 148, ctypes.byref(pk), ctypes.byref(ns)) == 0
    assert L.gqa_attn_choose(1, 128, 128, 6, 4, 64, 1, 148, ctypes.byref(pk), ctypes.byref(ns)) == 3


def test_status_strings():
    for c in range(11):
        assert G.gqa_attn_status_string(c) != "unknown status"
    assert G.gqa_attn_status_string(42) == "unknown status"


def test_heuristic_pack():
    # decode: one position per sequence, 4 heads per group -> packed
    assert G.gqa_attn_choose(32, 1, 2048, 32, 8, 128, 0)[0] == 1
    # ragged short query (77 positions): packing pads fewer rows
    assert G.gqa_attn_choose(4, 77, 4096, 32, 8, 128, 0)[0] == 1
    # long prefill, tile-aligned (equal padded rows): causal packs (the two tiles of a
    # unit end on the same key block), non-causal does not
    assert G.gqa_attn_choose(64, 2048, 2048, 32, 8, 128, 1)[0] == 1
    assert G.gqa_attn_choose(64, 2048, 2048, 32, 8, 128, 0)[0] == 0
    # packing would pad more rows (g = 3: 42 positions per tile): no packing, causal or not
    assert G.gqa_attn_choose(2, 2048, 2048, 6, 2, 128, 1)[0] == 0
    # MHA never packs
    assert G.gqa_attn_choose(4, 77, 4096, 32, 32, 128, 0)[0] == 0


def test_heuristic_splits():
    # enough (batch, head, q-tile) units to fill 148 SMs -> no split
    assert G.gqa_attn_choose(64, 2048, 2048, 32, 8, 128, 1)[1] == 1
    assert G.gqa_attn_choose(16, 2048, 2048, 32, 8, 128, 0)[1] == 1
    # small decode batch -> split the key axis, bounded by the key blocks and 16
    # a decode batch whose (batch, kv-head) units nearly fill the SM slots: no split
    # (measured on B200: splitting B=32, Sk=8192 costs more than it spreads)
    assert G.gqa_attn_choose(32, 1, 8192, 32, 8, 128, 0)[1] == 1
    assert G.gqa_attn_choose(256, 1, 8192, 32, 8, 128, 0)[1] == 1
    # a small decode batch: split the key axis
    pk, ns = G.gqa_attn_choose(4, 1, 8192, 32, 8, 128, 0)
    assert 2 <= ns <= 16
    assert G.gqa_attn_choose(1, 1, 256, 32, 8, 128, 0)[1] <= 2
    assert G.gqa_attn_choose(1, 1, 1 << 20, 32, 8, 128, 0)[1] <= 16


def test_workspace_bytes():
    assert G.gqa_attn_workspace_bytes(2, 128, 128, 4, 2, 64, 0, 0, 1) == 0
    assert G.gqa_attn_workspace_bytes(2, 128, 512, 4, 2, 64, 0, 0, 2) == 2 * 2 * 4 * 128 * 65 * 4
    # clamped to the number of 128-key blocks
    assert G.gqa_attn_workspace_bytes(1, 1, 256, 4, 2, 128, 0, 1, 16) == 2 * 1 * 4 * 1 * 129 * 4


def test_no_gpu_is_an_error_not_a_fallback():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # valid arguments on a machine without a GPU: a CUDA error, never a CPU result
    assert fwd_raw() in (6, 8)
    assert kvcache_raw() in (6, 8)
    assert kvcache_raw(seqlens=32, out_dtype=1) in (6, 8)
    L = G.load()
    assert L.gqa_attn_fwd_noalloc(16, 16, 16, 16, 16, 1, 8, 8, 4, 2, 64, 0.125, 0, -1, 0, None) in (6, 8)
    assert paged_raw() in (6, 8)
    assert fp8_raw() in (6, 8)
