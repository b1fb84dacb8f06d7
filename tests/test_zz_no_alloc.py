"""moe_permute_noalloc: the dispatch plan without a caller-provided workspace.

Some callers cannot allocate device memory (a plugin whose host framework
owns every allocation and passes in only inputs and outputs; a latency-bound
path where a cudaMalloc could synchronise the device).  For them the library
keeps the plan's scratch in its own static device memory.  This file checks
that entry point, called through the C ABI, against moe_permute on two calls
in a row.  Both plans are above 65536 slots, so both take the three-launch
path that uses the static array: the first (120000 slots, 59 blocks x 64
experts) fills 3776 entries of it, the second (72000 slots, 36 blocks x 32
experts) reuses a prefix of the array that the first left dirty.  It sorts
last so that a failure here stops a -x run only after every other test has
run.
"""
import ctypes

import pytest
import torch

import sparse_mixture_experts_07_b200 as moe
from sparse_mixture_experts_07_b200.moe import MoEShape

pytestmark = pytest.mark.gpu


def _noalloc(lib):
    f = lib.moe_permute_noalloc
    P = ctypes.c_void_p
    f.argtypes = [ctypes.POINTER(MoEShape), P, P, P, P, P, P, P]
    f.restype = ctypes.c_int
    return f


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _random_topk(T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    scores = torch.rand(T, E, generator=g)
    return torch.topk(scores, k, dim=1).indices.to(torch.int32).cuda()


def test_noalloc_permute_matches_workspace_permute(cuda_ok):
    lib = moe.load_library()
    f = _noalloc(lib)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for T, E, k, seed in ((20000, 64, 6, 1), (12000, 32, 6, 2)):
        assert T * k > 65536    # the path that uses the static array
        shape = moe.Shape(T=T, H=128, I=128, E=E, k=k)
        idx = _random_topk(T, E, k, seed)
        ws = moe.alloc_workspace(shape)
        err_ref = torch.zeros(1, dtype=torch.int32, device="cuda")
        ref = moe.permute(shape, idx, ws, err_ref)

        counts = torch.full((E,), -1, dtype=torch.int32, device="cuda")
        offsets = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
        perm = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
        inv = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = f(ctypes.byref(shape.c()), _ptr(idx), _ptr(counts), _ptr(offsets), _ptr(perm),
               _ptr(inv), _ptr(err), stream)
        assert rc == 0, moe.moe.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        assert err.item() == 0 and err_ref.item() == 0
        for got, want in zip((counts, offsets, perm, inv), ref):
            assert torch.equal(got, want)
        assert int(counts.sum()) == T * k


def test_noalloc_rejects_plans_beyond_its_scratch(cuda_ok):
    lib = moe.load_library()
    f = _noalloc(lib)
    # ceil(T*k / 2048) * E > 262144 int32 of static scratch
    shape = moe.Shape(T=2_000_000, H=128, I=128, E=256, k=4)
    p = ctypes.c_void_p(256)
    rc = f(ctypes.byref(shape.c()), p, p, p, p, p, None, None)
    assert rc == 2   # MOE_ERR_UNSUPPORTED, before any launch
