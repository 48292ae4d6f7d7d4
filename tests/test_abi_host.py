"""Host-only checks of the C ABI: the library loads, exports every function
include/pbs.h declares, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import subprocess
import re

import pytest

import permuted_block_sparse_b200 as pbs
from permuted_block_sparse_b200 import _binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


def _declared():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(pbs_[a-z0-9_]+)\s*\(", text):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    from permuted_block_sparse_b200 import build
    build.build()
    return pbs.load()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert {"pbs_permute", "pbs_select", "pbs_attn_fwd"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(bd.EXPORTS) <= declared


def test_version_and_last_error(lib):
    assert "sm_100a" in pbs.version()
    assert lib.pbs_get_last_error() is not None


def _desc(B=1, H=2, N=256, D=128, ptr=0x1000):
    return bd.PbsTensor(ptr, B, H, N, D, H * N * D, N * D, D)


@pytest.mark.parametrize("mutate,code", [
    (dict(ptr=0), -1),                 # null data
    (dict(D=96), -2),                  # unsupported head dim
    (dict(ptr=0x1008), -2),            # misaligned
])
def test_permute_rejects_bad_tensors(lib, mutate, code):
    kw = dict(B=1, H=2, N=256, D=128, ptr=0x1000)
    kw.update(mutate)
    q = _desc(**kw)
    k = _desc(B=1, H=1, N=256, D=kw["D"])
    rc = lib.pbs_permute(ctypes.byref(q), ctypes.byref(k), 128, 256, 0, ctypes.c_void_p(0x2000),
                         ctypes.c_void_p(0x4000), 1 << 20, None)
    assert rc == code
    assert lib.pbs_get_last_error()


def test_geometry_checks(lib):
    q, k = _desc(H=4), _desc(H=3)
    rc = lib.pbs_permute(ctypes.byref(q), ctypes.byref(k), 128, 256, 0, ctypes.c_void_p(0x2000),
                         ctypes.c_void_p(0x4000), 1 << 20, None)
    assert rc == -1 and b"multiple" in lib.pbs_get_last_error()
    q, k = _desc(H=2), _desc(H=1)
    for blk, seg, code in ((96, 192, -2), (128, 192, -1), (128, 16384, -2)):
        rc = lib.pbs_permute(ctypes.byref(q), ctypes.byref(k), blk, seg, 0, ctypes.c_void_p(0x2000),
                             ctypes.c_void_p(0x4000), 1 << 20, None)
        assert rc == code, (blk, seg)
    # workspace too small / misaligned
    rc = lib.pbs_permute(ctypes.byref(q), ctypes.byref(k), 128, 256, 0, ctypes.c_void_p(0x2000),
                         ctypes.c_void_p(0x4000), 16, None)
    assert rc == -1
    rc = lib.pbs_permute(ctypes.byref(q), ctypes.byref(k), 128, 256, 0, ctypes.c_void_p(0x2000),
                         ctypes.c_void_p(0x4010), 1 << 20, None)
    assert rc == -1


def test_select_capacity_and_errors(lib):
    # 128K, 10 % density, one sink block: budget 100 at block 992 minus 1 own block
    assert pbs.select_capacity(131072, 128, 4096, "topk", 0.10, 0, 128) == 99
    assert pbs.select_capacity(32768, 128, 2048, "tau", 0.95) == 240
    assert pbs.select_capacity(1024, 64, 256, "topk", 1.0) == 12
    q, k = _desc(H=2, N=1024), _desc(H=1, N=1024)
    cap = pbs.select_capacity(1024, 128, 256, "topk", 0.5)
    rc = lib.pbs_select(ctypes.byref(q), ctypes.byref(k), ctypes.c_void_p(0x2000), 128, 256, 0, 0.5, 0, 0,
                        ctypes.c_void_p(0x3000), ctypes.c_void_p(0x5000), cap - 1, ctypes.c_void_p(0x4000),
                        1 << 30, None)
    assert rc == -3
    rc = lib.pbs_select(ctypes.byref(q), ctypes.byref(k), ctypes.c_void_p(0x2000), 128, 256, 7, 0.5, 0, 0,
                        ctypes.c_void_p(0x3000), ctypes.c_void_p(0x5000), cap, ctypes.c_void_p(0x4000),
                        1 << 30, None)
    assert rc == -1


def test_workspace_sizes(lib):
    q, k = _desc(B=1, H=32, N=131072), _desc(B=1, H=8, N=131072)
    assert lib.pbs_workspace_size(0, ctypes.byref(q), ctypes.byref(k), 128, 4096) == 8 * 128 * 4
    nb = 1024
    # pooled query blocks, pooled permuted and natural key blocks, inverse
    # permutation, block-score matrix
    expect = 32 * nb * 128 * 4 + 2 * 8 * nb * 128 * 4 + 8 * 131072 * 4 + 32 * nb * nb * 4
    assert lib.pbs_workspace_size(1, ctypes.byref(q), ctypes.byref(k), 128, 4096) == expect


def test_attn_rejects_mismatched_output(lib):
    q, k, v = _desc(H=2), _desc(H=1), _desc(H=1)
    o = _desc(H=2, N=128)
    rc = lib.pbs_attn_fwd(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.c_void_p(0x2000),
                          ctypes.c_void_p(0x3000), ctypes.c_void_p(0x5000), 4, 128, 256, None, 0.088,
                          ctypes.byref(o), None, None, None, 0, None)
    assert rc == -1 and b"O shape" in lib.pbs_get_last_error()
    o = _desc(H=2)
    rc = lib.pbs_attn_fwd(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.c_void_p(0x2000),
                          ctypes.c_void_p(0x3000), ctypes.c_void_p(0x5000), 4, 128, 256, None, -1.0,
                          ctypes.byref(o), None, None, None, 0, None)
    assert rc == -1


def test_early_stop_and_score_order_argument_checks(lib):
    q, k, v, o = _desc(H=2), _desc(H=1), _desc(H=1), _desc(H=2)
    for tau in (-0.1, float("nan"), float("inf")):
        rc = lib.pbs_attn_fwd_early_stop(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v),
                                         ctypes.c_void_p(0x2000), ctypes.c_void_p(0x3000),
                                         ctypes.c_void_p(0x5000), 4, 128, 256, tau, 0.088, ctypes.byref(o),
                                         None, None, None)
        assert rc == -1 and b"stop_tau" in lib.pbs_get_last_error(), tau
    # the visiting-order flag leaves the capacity unchanged; other flag bits are refused
    assert (lib.pbs_select_capacity(32768, 128, 2048, 0x10 | 0, 0.3, 0, 0)
            == lib.pbs_select_capacity(32768, 128, 2048, 0, 0.3, 0, 0))
    q, k = _desc(H=2, N=1024), _desc(H=1, N=1024)
    cap = pbs.select_capacity(1024, 128, 256, "topk", 0.5)
    rc = lib.pbs_select(ctypes.byref(q), ctypes.byref(k), ctypes.c_void_p(0x2000), 128, 256, 0x40, 0.5, 0, 0,
                        ctypes.c_void_p(0x3000), ctypes.c_void_p(0x5000), cap, ctypes.c_void_p(0x4000),
                        1 << 30, None)
    assert rc == -1


def test_segmented_permutation_host_checks(lib):
    q, k, v, o = _desc(H=2), _desc(H=1), _desc(H=1), _desc(H=2)
    # general entry point: unknown flags, and a gate together with early stopping
    rc = lib.pbs_attn_fwd_ex(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.c_void_p(0x2000),
                             ctypes.c_void_p(0x3000), ctypes.c_void_p(0x5000), 4, 128, 256, 8, None, 0.0, 0.088,
                             ctypes.byref(o), None, None, None)
    assert rc == -1 and b"flags" in lib.pbs_get_last_error()
    rc = lib.pbs_attn_fwd_ex(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.c_void_p(0x2000),
                             ctypes.c_void_p(0x3000), ctypes.c_void_p(0x5000), 4, 128, 256, 1,
                             ctypes.c_void_p(0x6000), 0.1, 0.088, ctypes.byref(o), None, None, None)
    assert rc == -2
    # workspaces: fp64 pooled query per (b, KV head, segment); select holds one
    # pooled-key matrix and one inverse permutation per query segment
    Q, K = _desc(B=1, H=32, N=32768), _desc(B=1, H=8, N=32768)
    nseg, nb = 32768 // 2048, 32768 // 128
    assert lib.pbs_workspace_size(3, ctypes.byref(Q), ctypes.byref(K), 128, 2048) == 8 * nseg * 128 * 8
    expect = (32 * nb * 128 * 4 + 8 * nseg * nb * 128 * 4 + 8 * nb * 128 * 4 + 8 * nseg * 32768 * 4
              + 32 * nb * nb * 4)
    assert lib.pbs_workspace_size(4, ctypes.byref(Q), ctypes.byref(K), 128, 2048) == expect
    # a null permutation is refused before anything runs
    rc = lib.pbs_permute_segmented(ctypes.byref(Q), ctypes.byref(K), 128, 2048, 0, None,
                                   ctypes.c_void_p(0x4000), 1 << 30, None)
    assert rc == -1


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        pbs.pbs_permute(x, x, 64, 128)


def test_sample_selector_host_checks(lib):
    """PBS_SELECT_SAMPLE: a null permutation is accepted (it reads none);
    the visiting-order and per-segment flags, a non-positive CIA target and
    a too-small capacity are refused before anything runs; the capacity is
    every candidate block; the workspace holds fp64 column and slash scores
    and two bitmaps per (b, query head)."""
    SAMPLE = 2
    q, k = _desc(H=2, N=1024), _desc(H=1, N=1024)
    cap = pbs.select_capacity(1024, 128, 256, "sample", 0.9)
    assert cap == pbs.select_capacity(1024, 128, 256, "tau", 0.9) == 6
    args = (ctypes.c_void_p(0x3000), ctypes.c_void_p(0x5000))
    for mode, target, c, code in ((SAMPLE | 0x10, 0.9, cap, -2), (SAMPLE | 0x20, 0.9, cap, -2),
                                  (SAMPLE, 0.0, cap, -1), (SAMPLE, -1.0, cap, -1),
                                  (SAMPLE, float("nan"), cap, -1), (SAMPLE, 0.9, cap - 1, -3)):
        rc = lib.pbs_select(ctypes.byref(q), ctypes.byref(k), None, 128, 256, mode, target, 0, 0, *args, c,
                            ctypes.c_void_p(0x4000), 1 << 30, None)
        assert rc == code, (mode, target, c, rc)
    # broadcast views (a zero head stride over two heads) cannot be read by TMA
    qb = _desc(H=2, N=1024)
    qb.sH = 0
    rc = lib.pbs_select(ctypes.byref(qb), ctypes.byref(k), None, 128, 256, SAMPLE, 0.9, 0, 0, *args, cap,
                        ctypes.c_void_p(0x4000), 1 << 30, None)
    assert rc == -2 and b"broadcast" in lib.pbs_get_last_error()
    # grids above 2^31 CTAs are refused on the host
    big_q, big_k = _desc(B=65535, H=65535, N=128 * 8192), _desc(B=65535, H=1, N=128 * 8192)
    rc = lib.pbs_select(ctypes.byref(big_q), ctypes.byref(big_k), None, 128, 128, SAMPLE, 0.9, 0, 0, *args,
                        8192, ctypes.c_void_p(0x4000), 1 << 62, None)
    assert rc == -2 and b"2^31" in lib.pbs_get_last_error(), rc
    # other modes still need a permutation
    rc = lib.pbs_select(ctypes.byref(q), ctypes.byref(k), None, 128, 256, 0, 0.5, 0, 0, *args, cap,
                        ctypes.c_void_p(0x4000), 1 << 30, None)
    assert rc == -1 and b"perm" in lib.pbs_get_last_error()
    Q, K = _desc(B=1, H=32, N=32768), _desc(B=1, H=8, N=32768)
    words = 32768 // 32
    expect = 2 * 32 * 32768 * 8 + 2 * 32 * words * 4
    assert lib.pbs_workspace_size(pbs.PBS_OP_SELECT_SAMPLE, ctypes.byref(Q), ctypes.byref(K), 128, 2048) == expect


def test_binding_rejects_unknown_selection_mode(lib):
    with pytest.raises(ValueError):
        pbs.select_capacity(1024, 128, 256, "bogus", 0.5)


def _c_prototypes():
    """name -> list of parameter type strings, from include/pbs.h."""
    import re
    text = open(os.path.join(ROOT, "include", "pbs.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    protos = {}
    for m in re.finditer(r"(?:^|\n)\s*(?:const\s+)?\w+\s*\*?\s*(pbs_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        params = [" ".join(x.split()) for x in m.group(2).split(",")]
        types = []
        for prm in params:
            if prm in ("", "void"):
                continue
            t = re.sub(r"\b\w+$", "", prm).strip()      # drop the parameter name
            types.append(t.replace(" *", "*"))
        protos[m.group(1)] = types
    return protos


def _ctype_of(c_type):
    import ctypes
    if "pbs_tensor*" in c_type:
        return ctypes.POINTER(bd.PbsTensor)
    if c_type.endswith("*"):
        return ctypes.c_void_p
    return {"int": ctypes.c_int, "int64_t": ctypes.c_int64, "double": ctypes.c_double, "float": ctypes.c_float,
            "size_t": ctypes.c_size_t, "unsigned": ctypes.c_uint}[c_type]


def test_binding_signatures_match_the_header(lib):
    """Every ctypes declaration in the binding has the header's parameter
    list (count and C types), so drift between the two fails here."""
    protos = _c_prototypes()
    assert set(bd.EXPORTS) <= set(protos)
    checked = 0
    for name, types in protos.items():
        fn = getattr(lib, name)
        if fn.argtypes is None:
            continue
        want = [_ctype_of(t) for t in types]
        assert len(fn.argtypes) == len(want), name
        for got, exp in zip(fn.argtypes, want):
            assert got == exp or (exp is __import__("ctypes").c_void_p and got.__name__.startswith("LP_")), (name, got, exp)
        checked += 1
    assert checked >= 12


def test_c_caller_compiles_against_the_header_and_runs(tmp_path):
    """tests/c_abi/abi_check.c includes include/pbs.h, is compiled as C and
    linked against libpbs.so; every call is rejected on the host with its
    documented status."""
    import shutil
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path / "abi_check")
    libdir = os.path.dirname(bd.LIB_PATH)
    build = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                            os.path.join(ROOT, "tests", "c_abi", "abi_check.c"), "-o", exe, "-L", libdir, "-l:libpbs.so",
                            "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and "abi ok" in run.stdout, run.stdout + run.stderr
