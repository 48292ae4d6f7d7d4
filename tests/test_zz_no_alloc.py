"""pbs_permute_noalloc against pbs_permute, through the C ABI.

pbs_permute_noalloc exists for callers that cannot allocate device memory
when they call (their device memory is reserved by another allocator, or
their plugin interface gives a kernel no workspace).  It keeps its scratch in
a fixed array inside the library, so this test checks that two calls in a
row -- the second one seeing the first call's leftovers in that array --
both give exactly the permutation of the workspace-based entry point.  This
file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import permuted_block_sparse_b200 as pbs
from permuted_block_sparse_b200 import _binding as bd
from permuted_block_sparse_b200 import synth

pytestmark = pytest.mark.gpu


def _noalloc(lib):
    fn = lib.pbs_permute_noalloc
    P = ctypes.POINTER(bd.PbsTensor)
    fn.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def _case(seed, B, Hq, Hkv, N, d, blk, seg, n_sink):
    w = synth.Workload("noalloc", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, blk=blk, seg=seg, mode="topk",
                       stripe_frac=0.01, seed=seed)
    Q, K, V, _ = synth.make_inputs(w)
    Qd = torch.from_numpy(Q).to(torch.bfloat16).cuda()
    Kd = torch.from_numpy(K).to(torch.bfloat16).cuda()
    return Qd, Kd


def test_noalloc_matches_workspace_entry_point_twice():
    lib = pbs.load()
    fn = _noalloc(lib)
    stream = torch.cuda.current_stream().cuda_stream
    cases = [
        (0, 1, 8, 2, 8192, 128, 128, 1024, 0),     # first call: scratch holds nothing yet
        (7, 2, 4, 4, 4096, 64, 64, 512, 64),       # second call: scratch holds the first call's data
    ]
    for (seed, B, Hq, Hkv, N, d, blk, seg, n_sink) in cases:
        Qd, Kd = _case(seed, B, Hq, Hkv, N, d, blk, seg, n_sink)
        ref = pbs.pbs_permute(Qd, Kd, blk, seg, n_sink)
        out = torch.full_like(ref, -1)
        q, k = bd.describe(Qd), bd.describe(Kd)
        rc = fn(ctypes.byref(q), ctypes.byref(k), blk, seg, n_sink, out.data_ptr(), stream)
        assert rc == 0, lib.pbs_get_last_error()
        pbs.pbs_check_device()
        assert torch.equal(out, ref), (seed, B, Hq, Hkv, N)


def test_noalloc_at_exactly_its_scratch_size():
    """B * Hkv * D = 512 * 128 = 65536 floats fills the static scratch
    exactly: still served, and equal to the workspace entry point."""
    lib = pbs.load()
    fn = _noalloc(lib)
    stream = torch.cuda.current_stream().cuda_stream
    Qd, Kd = _case(3, 1, 512, 512, 256, 128, 128, 256, 0)
    ref = pbs.pbs_permute(Qd, Kd, 128, 256, 0)
    out = torch.full_like(ref, -1)
    q, k = bd.describe(Qd), bd.describe(Kd)
    rc = fn(ctypes.byref(q), ctypes.byref(k), 128, 256, 0, out.data_ptr(), stream)
    assert rc == 0, lib.pbs_get_last_error()
    pbs.pbs_check_device()
    assert torch.equal(out, ref)
    # one KV head more (65536 + 128 floats) is refused before any launch
    Qd, Kd = _case(3, 1, 513, 513, 128, 128, 128, 128, 0)
    q, k = bd.describe(Qd), bd.describe(Kd)
    out = torch.full((1, 513, 128), -1, dtype=torch.int32, device="cuda")
    rc = fn(ctypes.byref(q), ctypes.byref(k), 128, 128, 0, out.data_ptr(), stream)
    assert rc == -3
    assert int(out.min()) == -1 and int(out.max()) == -1


def test_noalloc_rejects_inputs_beyond_its_scratch():
    lib = pbs.load()
    fn = _noalloc(lib)
    # B * Hkv * D = 4 * 130 * 128 > 65536 floats: refused before any launch
    q = bd.PbsTensor(0x1000, 4, 130, 256, 128, 130 * 256 * 128, 256 * 128, 128)
    k = bd.PbsTensor(0x1000, 4, 130, 256, 128, 130 * 256 * 128, 256 * 128, 128)
    rc = fn(ctypes.byref(q), ctypes.byref(k), 128, 256, 0, ctypes.c_void_p(0x2000), None)
    assert rc == -3
    assert b"65536" in lib.pbs_get_last_error()
