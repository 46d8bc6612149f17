"""The C ABI library: it loads without a GPU, exports every symbol the header
declares, and rejects invalid arguments on the host before launching anything.
No call here reaches a kernel."""
import ctypes
import os
import re

import pytest

import unified_sparse_attention_b200 as U
from unified_sparse_attention_b200 import binding as Bd

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "lserve.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lserve_[a-z_0-9]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert sorted(U.EXPORTED_SYMBOLS) == declared_functions()


def test_library_exports_every_declared_symbol():
    lib = U.load_library()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert U.lserve_version().count(".") == 2


def shape(B=1, S=1024, Hq=4, Hkv=2, d=64):
    return ctypes.byref(Bd.Shape(B, S, Hq, Hkv, d, 0.0))


FAKE = ctypes.c_void_p(1 << 20)   # 16-byte aligned, never dereferenced: validation fails first


def test_prefill_validation():
    lib = U.load_library()
    assert lib.lserve_prefill_workspace_size(shape(d=64)) > 0
    assert lib.lserve_prefill_workspace_size(shape(S=100)) == 0
    call = lambda shp, q=FAKE, ws=None, wsb=0, sink=64, local=256: lib.lserve_prefill(
        shp, q, FAKE, FAKE, FAKE, sink, local, None, FAKE, None, ws, wsb, None)
    assert call(shape(d=96)) == 2
    assert call(shape(S=1000)) == 2
    assert call(shape(Hq=3)) == 1
    assert call(shape(), q=None) == 1
    assert call(shape(), sink=-1) == 1
    bad_flag = Bd.Shape(1, 1024, 4, 2, 64, 0.0, 2)                 # lambda_tiles is 0 or 1
    assert call(ctypes.byref(bad_flag)) == 1
    assert call(shape(), q=ctypes.c_void_p((1 << 20) + 2)) == 1   # misaligned
    assert call(shape()) == 3                                      # no workspace
    need = lib.lserve_prefill_workspace_size(shape())
    assert call(shape(), ws=ctypes.c_void_p(1 << 20), wsb=need - 1) == 3
    assert call(shape(), ws=ctypes.c_void_p((1 << 20) + 16), wsb=need) == 3   # not 256-aligned
    assert "workspace" in U.lserve_last_error_string()


def decode_args(**kw):
    a = dict(B=2, Hq=8, Hkv=2, d=128, num_pages=64, maxP=32, q=1 << 20, k_pages=1 << 20, v_pages=1 << 20,
             page_table=1 << 20, seq_lens=1 << 20, stats=1 << 20, head_kind=1 << 20, sink=64, local=256,
             token_budget=512, scale=0.0)
    a.update(kw)
    return Bd.DecodeArgs(**a)


def test_decode_validation_and_capacity():
    lib = U.load_library()
    a = decode_args()
    assert lib.lserve_decode_max_selected(ctypes.byref(a)) == 8          # 512 / 64
    a = decode_args(token_budget=64, sink=64, local=256)
    assert lib.lserve_decode_max_selected(ctypes.byref(a)) == 1 + 4 + 1   # streaming bound
    assert lib.lserve_decode_workspace_size(ctypes.byref(decode_args())) > 0
    for bad, code in ((dict(d=96), 2), (dict(Hq=24), 2), (dict(token_budget=63), 1), (dict(Hq=7), 1),
                      (dict(sink=-1), 1), (dict(q=0), 1), (dict(stats=(1 << 20) + 8), 1)):
        a = decode_args(**bad)
        assert lib.lserve_decode_workspace_size(ctypes.byref(a)) == 0
        assert lib.lserve_decode(ctypes.byref(a), FAKE, None, None, None, None, 0, None) == code, bad
    a = decode_args()
    assert lib.lserve_decode(ctypes.byref(a), FAKE, None, None, None, None, 0, None) == 3


def test_page_stats_validation():
    lib = U.load_library()
    assert lib.lserve_update_page_stats(1, 2, 96, 4, FAKE, FAKE, 4, FAKE, 0, FAKE, FAKE, None) == 2
    assert lib.lserve_update_page_stats(1, 2, 64, 4, None, FAKE, 4, FAKE, 0, FAKE, FAKE, None) == 1
    assert lib.lserve_update_page_stats(1, 2, 64, 4, FAKE, FAKE, 4, FAKE, -1, FAKE, FAKE, None) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 64, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        U.lserve_prefill(q, q[:, :, :1], q[:, :, :1], torch.zeros(1, dtype=torch.uint8), 0, 64)


def test_int4_reuse_and_cra_validation():
    """The next rows' entry points refuse bad arguments on the host, before any
    launch: INT4 quantiser and decode, selection reuse, CRA."""
    lib = U.load_library()
    bad16 = ctypes.c_void_p((1 << 20) + 8)   # not 16-byte aligned
    q = lib.lserve_quantize_pages_int4
    #           B  Hkv  d  NP  k     v     table maxP lens first kind  kq    kpar  vq    vpar  stats stream
    assert q(1, 2, 96, 4, FAKE, FAKE, FAKE, 4, FAKE, 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert q(1, 2, 64, 4, FAKE, FAKE, FAKE, 4, FAKE, -1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert q(1, 2, 64, 4, FAKE, FAKE, FAKE, 4, FAKE, 0, FAKE, None, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert q(1, 2, 64, 4, FAKE, FAKE, FAKE, 4, FAKE, 0, FAKE, bad16, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert q(0, 2, 64, 4, FAKE, FAKE, FAKE, 4, FAKE, 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1

    d4 = lib.lserve_decode_int4
    a = decode_args()
    assert d4(ctypes.byref(a), None, FAKE, FAKE, None, None, None, FAKE, 1 << 30, None) == 1      # no kpar
    assert d4(ctypes.byref(a), FAKE, bad16, FAKE, None, None, None, FAKE, 1 << 30, None) == 1     # misaligned vpar
    assert d4(ctypes.byref(decode_args(d=96)), FAKE, FAKE, FAKE, None, None, None, FAKE, 1 << 30, None) == 2
    assert d4(ctypes.byref(a), FAKE, FAKE, FAKE, None, None, None, None, 0, None) == 3           # no workspace
    # one size query covers the bf16 and the INT4 plans
    assert lib.lserve_decode_workspace_size(ctypes.byref(a)) > 0

    r = lib.lserve_decode_reuse
    a = decode_args(stats=0)   # reuse reads no summaries
    assert r(ctypes.byref(a), None, FAKE, FAKE, None, None, None, FAKE, 1 << 30, None) == 1      # no sel_in
    assert r(ctypes.byref(a), FAKE, FAKE, FAKE, None, None, None, None, 0, None) == 3            # no workspace

    assert lib.lserve_cra_workspace_size(shape(S=1000)) == 0   # S not a multiple of 64
    assert lib.lserve_cra_workspace_size(shape()) > 0
    assert lib.lserve_cra(shape(d=96), FAKE, FAKE, FAKE, FAKE, 0, 64, None, None, FAKE, FAKE, 1 << 30, None) == 2


def test_vslash_validation():
    lib = U.load_library()
    assert lib.lserve_vslash_workspace_size(shape(), 1) > 0
    assert lib.lserve_vslash_workspace_size(shape(), 0) == 0
    call = lambda shp, stride=1, tau=0.9, ws=None, wsb=0: lib.lserve_build_vslash_mask(
        shp, FAKE, FAKE, FAKE, stride, tau, FAKE, None, None, None, ws, wsb, None)
    assert call(shape(), stride=0) == 1
    assert call(shape(), tau=1.5) == 1
    assert call(shape(), tau=float("nan")) == 1
    assert call(shape(Hq=18, Hkv=2)) == 2          # Hq/Hkv = 9 > 8
    assert call(shape(d=96)) == 2
    assert call(shape()) == 3                      # no workspace
    assert "vslash" in U.lserve_last_error_string()
