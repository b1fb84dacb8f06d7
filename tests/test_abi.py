"""The C ABI: the library builds, loads, exports every declared entry point, and
rejects bad arguments on the host before touching the GPU."""
import ctypes
import os
import re

import pytest

import sparse_mixture_experts_07_b200 as moe
from sparse_mixture_experts_07_b200 import build as moe_build
from sparse_mixture_experts_07_b200.moe import MoEShape

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.load_library()


def declared_entry_points():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", text)
    return names


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for n in ("moe_route", "moe_permute", "moe_forward", "moe_combine", "moe_workspace_size",
              "moe_status_str"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_entry_points():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in moe.moe.STATUS.items():
        assert lib.moe_status_str(code).decode() == name
    assert lib.moe_status_str(99).decode() == "MOE_ERR_UNKNOWN"


def _shape(**kw):
    base = dict(T=64, H=128, I=256, E=8, k=2, n_shared=0, I_shared=0, routed_scale=1.0,
                dtype=moe.MOE_BF16)
    base.update(kw)
    return MoEShape(**base)


def _ws(lib, s):
    n = ctypes.c_size_t(0)
    rc = lib.moe_workspace_size(ctypes.byref(s), ctypes.byref(n))
    return rc, n.value


@pytest.mark.parametrize("kw,expected", [
    (dict(k=9), 1), (dict(k=0), 1), (dict(E=0), 1), (dict(T=-1), 1), (dict(H=0), 1),
    (dict(n_shared=1, I_shared=0), 1), (dict(dtype=7), 1),
    (dict(E=300, k=2), 2), (dict(k=17, E=64), 2), (dict(n_shared=9, I_shared=64), 2),
    (dict(H=100), 2), (dict(I=100), 2), (dict(n_shared=1, I_shared=36), 2),
    (dict(H=100, dtype=moe.MOE_F32), 0), (dict(T=0), 0),
])
def test_shape_validation(lib, kw, expected):
    rc, _ = _ws(lib, _shape(**kw))
    assert rc == expected


def test_workspace_size_grows_with_tokens(lib):
    sizes = [_ws(lib, _shape(T=t))[1] for t in (1, 64, 1000, 4096)]
    assert sizes == sorted(sizes) and sizes[0] > 0
    _, with_shared = _ws(lib, _shape(n_shared=2, I_shared=128))
    assert with_shared > _ws(lib, _shape())[1]


def test_null_pointers_rejected_before_launch(lib):
    s = _shape()
    p = ctypes.c_void_p(16)   # never dereferenced: validation fails first
    assert lib.moe_route(ctypes.byref(s), None, p, None, None, p, p, None, None) == 1
    assert lib.moe_route(ctypes.byref(s), p, None, None, None, p, p, None, None) == 1
    assert lib.moe_permute(ctypes.byref(s), p, None, p, p, p, None, p, 1 << 30, None) == 1
    assert lib.moe_forward(ctypes.byref(s), p, p, p, p, None, p, None, None, p, None, p,
                           1 << 30, None) == 1
    sh = _shape(n_shared=2, I_shared=128)
    assert lib.moe_forward(ctypes.byref(sh), p, p, p, p, p, p, None, None, p, None, p,
                           1 << 30, None) == 1
    assert lib.moe_combine(ctypes.byref(s), None, p, p, None) == 1
    assert lib.moe_route(None, p, p, None, None, p, p, None, None) == 1
    # moe_route_permute: x, w_router, topk_idx, topk_w, counts, offsets, perm, inv
    args = [p, p, None, None, None, p, p, p, p, p, p, None, p, 1 << 30, None]
    for i in (0, 1, 5, 6, 7, 8, 9, 10):
        a = list(args)
        a[i] = None
        assert lib.moe_route_permute(ctypes.byref(s), *a) == 1, i


def test_small_workspace_rejected(lib):
    s = _shape()
    rc, need = _ws(lib, s)
    p = ctypes.c_void_p(256)
    assert lib.moe_permute(ctypes.byref(s), p, p, p, p, p, None, p, need - 1, None) == 3
    assert lib.moe_permute(ctypes.byref(s), p, p, p, p, p, None, None, need, None) == 3
    assert lib.moe_forward(ctypes.byref(s), p, p, p, p, p, p, None, None, p, None, p,
                           need - 1, None) == 3
    for ws, n in ((p, need - 1), (None, need)):
        assert lib.moe_route_permute(ctypes.byref(s), p, p, None, None, None, p, p, p, p, p, p,
                                     None, ws, n, None) == 3


def test_misaligned_bf16_pointers_rejected(lib):
    s = _shape()
    _, need = _ws(lib, s)
    ok, bad = ctypes.c_void_p(4096), ctypes.c_void_p(4096 + 2)
    assert lib.moe_forward(ctypes.byref(s), bad, ok, ok, ok, ok, ok, None, None, ok, None, ok,
                           need, None) == 2
    assert lib.moe_combine(ctypes.byref(s), bad, ok, ok, None) == 2


def _split_size(lib, s):
    n = ctypes.c_size_t(0)
    rc = lib.moe_router_split_size(ctypes.byref(s), ctypes.byref(n))
    return rc, n.value


@pytest.mark.parametrize("E,rows", [(1, 32), (8, 32), (9, 48), (16, 48), (17, 96), (32, 96), (40, 192),
                                    (64, 192)])
def test_router_split_size(lib, E, rows):
    # N = 3 E_PAD rounded up to 16, E_PAD in {8, 16, 32, 64}; bf16 rows of H
    assert _split_size(lib, _shape(E=E, k=1, H=256)) == (0, rows * 256 * 2)


def test_router_split_size_zero_where_the_tensor_core_router_does_not_apply(lib):
    assert _split_size(lib, _shape(dtype=moe.MOE_F32)) == (0, 0)
    assert _split_size(lib, _shape(E=65)) == (0, 0)
    assert _split_size(lib, _shape(k=0))[0] == 1


def test_shared_merge_argument_checks(lib):
    """moe_shared_merge rejects a shape without shared experts, NULL pointers
    and invalid shapes before any copy is enqueued."""
    p = ctypes.c_void_p(4096)
    s = _shape(n_shared=2, I_shared=64)
    args = [p, p, p, p]
    for i in range(4):
        a = list(args)
        a[i] = None
        assert lib.moe_shared_merge(ctypes.byref(s), *a, None) == 1
    none = _shape(n_shared=0, I_shared=0)
    assert lib.moe_shared_merge(ctypes.byref(none), *args, None) == 1
    assert lib.moe_shared_merge(ctypes.byref(_shape(n_shared=2, I_shared=0)), *args, None) == 1
    assert lib.moe_shared_merge(ctypes.byref(_shape(n_shared=2, I_shared=60)), *args, None) == 2
    assert lib.moe_shared_merge(None, *args, None) == 1


def test_shared_merge_binding_checks_shapes(lib):
    """The binding rejects shared-expert tensors of the wrong shape or layout
    before it calls the library."""
    import torch
    shape = moe.Shape(T=4, H=16, I=8, E=4, k=2, n_shared=2, I_shared=8)
    gu = torch.zeros(2, 16, 16, dtype=torch.bfloat16)
    dn = torch.zeros(2, 16, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        moe.shared_merge(shape, gu[:, :8], dn)
    with pytest.raises(ValueError):
        moe.shared_merge(shape, gu, dn.transpose(1, 2).contiguous())
    with pytest.raises(ValueError):
        moe.shared_merge(shape, gu, torch.zeros(2, 8, 16, dtype=torch.bfloat16).transpose(1, 2))


def test_router_split_argument_checks(lib):
    s = _shape(E=8, H=128)
    _, need = _split_size(lib, s)
    ok, bad = ctypes.c_void_p(4096), ctypes.c_void_p(4096 + 4)
    assert lib.moe_router_split(ctypes.byref(s), None, ok, need, None) == 1
    assert lib.moe_router_split(ctypes.byref(s), ok, None, need, None) == 1
    assert lib.moe_router_split(ctypes.byref(s), ok, ok, need - 1, None) == 3
    assert lib.moe_router_split(ctypes.byref(s), bad, ok, need, None) == 2
    assert lib.moe_router_split(ctypes.byref(s), ok, bad, need, None) == 2
    f32 = _shape(dtype=moe.MOE_F32)
    assert lib.moe_router_split(ctypes.byref(f32), ok, ok, 1 << 20, None) == 2
    p = ctypes.c_void_p(16)
    assert lib.moe_route_split(ctypes.byref(s), None, p, p, None, None, p, p, None, None) == 1
    assert lib.moe_route_split(ctypes.byref(s), p, None, p, None, None, p, p, None, None) == 1
    big = _shape(T=4096, E=8)
    assert lib.moe_route_split(ctypes.byref(big), bad, ok, ok, None, None, ok, ok, None,
                               None) == 2
    assert lib.moe_route_split(ctypes.byref(big), ok, ok, bad, None, None, ok, ok, None,
                               None) == 2


def test_forward_mxfp4_argument_checks(lib):
    ok = ctypes.c_void_p(4096)
    s = _shape(T=4, H=256, I=128)
    _, need = _ws(lib, s)

    def call(shape, ws_bytes=need, x=ok, q=ok, ws=ok):
        return lib.moe_forward_mxfp4(ctypes.byref(shape), x, ok, ok, ok, q, ok, ok, ok, ok,
                                     None, ws, ws_bytes, None)
    assert call(_shape(T=65, H=256, I=128)) == 2             # decode batches only (T <= 64)
    assert call(_shape(T=4, H=256, I=128, n_shared=1, I_shared=64)) == 2
    assert call(_shape(T=4, H=136, I=128)) == 2              # H not a multiple of 32
    assert call(_shape(T=4, H=256, I=136)) == 2
    assert call(_shape(T=4, H=256, I=128, dtype=moe.MOE_F32)) == 2
    assert call(s, q=None) == 1
    assert call(s, x=None) == 1
    assert call(s, ws_bytes=need - 1) == 3
    assert call(s, ws=None) == 3
    assert call(s, x=ctypes.c_void_p(4096 + 8)) == 2
    # scale arrays are read in aligned 4-byte words
    assert lib.moe_forward_mxfp4(ctypes.byref(s), ok, ok, ok, ok, ok, ctypes.c_void_p(4096 + 2),
                                 ok, ok, ok, None, ok, need, None) == 2
    assert call(_shape(T=0, H=256, I=128), x=None, q=None, ws=None, ws_bytes=0) == 0


def test_zero_tokens_is_a_no_op(lib):
    s = _shape(T=0)
    assert lib.moe_route(ctypes.byref(s), None, None, None, None, None, None, None, None) == 0
    assert lib.moe_forward(ctypes.byref(s), None, None, None, None, None, None, None, None,
                           None, None, None, 0, None) == 0
    assert lib.moe_combine(ctypes.byref(s), None, None, None, None) == 0


def test_missing_library_fails_loudly(tmp_path):
    import importlib
    m = importlib.import_module("sparse_mixture_experts_07_b200.moe")
    saved = m._lib
    m._lib = None
    try:
        with pytest.raises(RuntimeError, match="not built"):
            m.load_library(str(tmp_path / "libmoe.so"))
    finally:
        m._lib = saved


@pytest.mark.parametrize("kw", [
    dict(k=9), dict(E=0), dict(T=-1), dict(dtype=7), dict(n_shared=1, I_shared=0),
    dict(E=300, k=2), dict(n_shared=9, I_shared=64), dict(H=100), dict(I=100),
    dict(n_shared=1, I_shared=36), dict(T=1 << 30, k=2, n_shared=2, I_shared=64),
])
def test_noalloc_permute_validates_shapes_like_permute(lib, kw):
    """moe_permute_noalloc applies moe_permute's shape checks (before its own
    scratch limit), so both return the same status on an invalid shape."""
    s = _shape(**kw)
    p = ctypes.c_void_p(256)     # never dereferenced: validation fails first
    lib.moe_permute_noalloc.argtypes = [ctypes.POINTER(MoEShape)] + [ctypes.c_void_p] * 7
    lib.moe_permute_noalloc.restype = ctypes.c_int
    want = lib.moe_permute(ctypes.byref(s), p, p, p, p, p, None, p, 1 << 40, None)
    got = lib.moe_permute_noalloc(ctypes.byref(s), p, p, p, p, p, None, None)
    assert want != 0 and got == want


@pytest.mark.parametrize("n_group,topk_group", [(3, 1), (4, 0), (4, 5), (8, 1), (64, 1), (0, 1)])
def test_noaux_rejects_bad_group_arguments(lib, n_group, topk_group):
    """E % n_group != 0, topk_group outside [1, n_group], k above the kept
    experts, n_group above 32: MOE_ERR_INVALID_ARG before any launch."""
    s = _shape(T=4, E=16, k=4)
    p = ctypes.c_void_p(256)
    f = lib.moe_route_noaux_tc
    f.argtypes = [ctypes.POINTER(MoEShape), ctypes.c_int32, ctypes.c_int32] + \
        [ctypes.c_void_p] * 9
    f.restype = ctypes.c_int
    assert f(ctypes.byref(s), n_group, topk_group, p, p, None, None, p, p, p, None, None) == 1
    # valid groups, but the logits buffer the selection reads is required
    assert f(ctypes.byref(s), 4, 2, p, p, None, None, None, p, p, None, None) == 1


def _prepared_size(lib, s):
    n = ctypes.c_size_t(0)
    rc = lib.moe_mxfp4_prepared_size(ctypes.byref(s), ctypes.byref(n))
    return rc, n.value


def _prepared_bytes(H, I, E):
    """Scale atoms of both GEMMs, then codes padded to 128-weight rows where
    H or I needs it; each part rounded up to 256 bytes."""
    def a256(v):
        return (v + 255) // 256 * 256
    def c128(v):
        return -(-v // 128)
    parts = [512 * E * (I // 64) * c128(H), 512 * E * c128(H) * c128(I),
             E * 2 * I * c128(H) * 64 if H % 128 else 0, E * H * c128(I) * 64 if I % 128 else 0]
    return sum(a256(p) for p in parts)


@pytest.mark.parametrize("H,I,E", [(4096, 6400, 16), (2880, 2880, 32), (320, 192, 3),
                                   (288, 128, 8), (256, 96, 8)])
def test_mxfp4_prepared_size(lib, H, I, E):
    want = _prepared_bytes(H, I, E) if H % 64 == 0 and I % 64 == 0 else 0
    assert _prepared_size(lib, _shape(H=H, I=I, E=E, k=2, T=8)) == (0, want)
    if (H, I, E) == (4096, 6400, 16):
        assert want == 512 * 16 * (100 * 32 + 32 * 50)       # no padded codes


def test_mxfp4_prepared_argument_checks(lib):
    s = _shape(H=320, I=192, E=4, k=2, T=8)
    _, need = _prepared_size(lib, s)
    ok, bad = ctypes.c_void_p(4096), ctypes.c_void_p(4096 + 8)
    assert lib.moe_mxfp4_prepare(ctypes.byref(s), None, ok, ok, ok, ok, need, None) == 1
    assert lib.moe_mxfp4_prepare(ctypes.byref(s), ok, ok, ok, ok, ok, need - 1, None) == 3
    assert lib.moe_mxfp4_prepare(ctypes.byref(s), ok, ok, ok, ok, bad, need, None) == 2
    odd = _shape(H=288, I=192, E=4, k=2, T=8)
    assert lib.moe_mxfp4_prepare(ctypes.byref(odd), ok, ok, ok, ok, ok, 1 << 30, None) == 2
    _, ws = _ws(lib, s)
    # x, offsets, perm, topk_w, gate_up_q, down_q, prepared, y_slots
    args = [ok, ok, ok, ok, ok, ok, ok, ok, None, ok, ws, None]
    for i in range(8):
        a = list(args)
        a[i] = None
        assert lib.moe_forward_mxfp4_prepared(ctypes.byref(s), *a) == 1, i
    a = list(args)
    a[9] = None
    assert lib.moe_forward_mxfp4_prepared(ctypes.byref(s), *a) == 3
    assert lib.moe_forward_mxfp4_prepared(ctypes.byref(odd), *args) == 2
    long_batch = _shape(H=320, I=192, E=4, k=2, T=65)
    assert lib.moe_forward_mxfp4_prepared(ctypes.byref(long_batch), *args) == 2
