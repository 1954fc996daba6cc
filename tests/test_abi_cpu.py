"""The C-ABI library without a GPU: it loads, exports every declared entry point,
validates arguments on the host, and plans launches (host arithmetic only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dyt.h")


def _lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location("dyt_build", os.path.join(ROOT, "elementwise_reduction_b200",
                                                                            "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import elementwise_reduction_b200 as dyt
    return dyt


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dyt_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for f in ("dyt_forward", "dyt_backward", "dyt_backward_workspace_bytes", "dyt_status_string",
              "dyt_last_launch_info", "dyt_plan_query", "dyt_forward_ex", "dyt_backward_ex"):
        assert f in names


def test_backward_takes_beta_after_gamma():
    # dyt_backward(x, dy, alpha, gamma, beta, dx, dgamma, dbeta, dalpha, M, N, ...)
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    for name in ("dyt_backward", "dyt_backward_strided", "dyt_backward_noalloc", "dyt_backward_ex"):
        m = re.search(r"dyt_status\s+" + name + r"\s*\(([^)]*)\)", text)
        assert m, name
        params = [p.strip().split()[-1].lstrip("*") for p in m.group(1).split(",")]
        assert params[params.index("gamma") + 1] == "beta", (name, params)
        assert params.index("beta") < params.index("dx"), (name, params)


def test_library_exports_every_declared_function():
    dyt = _lib()
    lib = ctypes.CDLL(dyt._abi.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/dyt.h but not exported"


def test_host_validation_without_a_device():
    dyt = _lib()
    # negative sizes, bad dtypes and null pointers are rejected before any CUDA call
    assert dyt.dyt_forward(0, 0, 0, 0, 0, -1, 4, 0, 0, None) == 1
    assert dyt.dyt_forward(0, 0, 0, 0, 0, 4, -1, 0, 0, None) == 1
    assert dyt.dyt_forward(0, 0, 0, 0, 0, 4, 4, 7, 0, None) == 2
    assert dyt.dyt_forward(0, 0, 0, 0, 0, 4, 4, 0, 3, None) == 2
    assert dyt.dyt_forward(0, 0, 0, 0, 0, 4, 4, 0, 0, None) == 1          # null pointers
    assert dyt.dyt_forward(0, 0, 0, 0, 0, 4, 2**31, 0, 0, None) == 1      # N beyond int32
    assert dyt.dyt_forward(0, 0, 0, 0, 0, 2**62, 2**20, 0, 0, None) == 1  # M*N*size overflows
    assert dyt.dyt_forward(0, 0, 0, 0, 0, 0, 5, 0, 0, None) == 0          # empty: nothing to do
    assert dyt.dyt_last_launch_info()["kernels"] == 0
    assert dyt.dyt_backward(0, 0, 0, 0, None, 0, 0, 0, 0, 3, 3, 0, 0, 0, 0, None) == 1  # null dalpha
    assert dyt.dyt_backward(0, 0, 0, 0, None, 0, 0, 0, 1, 3, 3, 1, 0, 0, 0, None) == 1  # null dgamma/dbeta
    assert dyt.dyt_backward(0, 0, 0, 0, None, 0, 0, 0, 0, -3, 3, 0, 0, 0, 0, None) == 1
    assert dyt.dyt_backward(0, 0, 0, 0, None, 0, 0, 0, 0, 3, 3, 0, 5, 0, 0, None) == 2  # bad param dtype
    # one dtype per parameter: each code is checked
    for bad in ((3, 0, 0), (0, 3, 0), (0, 0, -1)):
        assert dyt.dyt_forward_ex(0, 4, 0, 0, 0, 0, 4, 4, 4, 0, *bad, None) == 2
        assert dyt.dyt_backward_ex(0, 4, 0, 4, 0, 0, None, 0, 4, 0, 0, 0, 4, 4, 0, *bad, 0, 0, None) == 2
    assert dyt.dyt_forward_ex(0, 4, 0, 0, 0, 0, 4, 0, 4, 1, 1, 2, 0, None) == 0  # empty: nothing to do
    assert dyt.dyt_backward_noalloc(0, 0, 0, 0, None, 0, 0, 0, 0, -1, 3, 0, 0, None) == 1
    # stage 1 and the finalize of several ranks
    st, lay = dyt.dyt_backward_partials(0, 4, 0, 4, 0, 0, 0, 4, 0, 4, 0, 0, 0, 0, 0, None)
    assert st == 0 and lay["rows"] == 0 and lay["dalpha_parts"] == 0      # no rows: no partials
    assert dyt.dyt_backward_partials(0, 4, 0, 4, 0, 0, 0, 4, -1, 4, 0, 0, 0, 0, 0, None)[0] == 1
    assert dyt.dyt_backward_partials(0, 4, 0, 4, 0, 0, 0, 4, 3, 4, 0, 7, 0, 0, 0, None)[0] == 2
    empty = {"bytes": 0, "off_dgamma": 0, "off_dbeta": 0, "off_dalpha": 0, "rows": 0, "dalpha_parts": 0}
    assert dyt.dyt_finalize_partials([], [], 4, 1, 1, 1, 0, 0, 0, None) == 1                # no ranks
    assert dyt.dyt_finalize_partials([0] * 9, [empty] * 9, 4, 1, 1, 1, 0, 0, 0, None) == 1   # more than 8
    assert dyt.dyt_finalize_partials([0], [empty], 4, 1, 1, 1, 0, 5, 0, None) == 2          # bad dtype
    assert dyt.dyt_finalize_partials([0], [empty], 4, 0, 1, 1, 0, 0, 0, None) == 1          # null dgamma
    bad = dict(empty, rows=3, bytes=64)                                                     # partials past `bytes`
    assert dyt.dyt_finalize_partials([16], [bad], 4, 1, 1, 1, 0, 0, 0, None) == 1
    assert dyt.dyt_finalize_partials([0], [dict(empty, rows=1, bytes=1 << 20)], 4, 1, 1, 1, 0, 0, 0, None) == 1
    # row pitches below N, or byte offsets beyond int64, are rejected
    assert dyt.dyt_forward_strided(0, 3, 0, 0, 0, 0, 4, 5, 4, 0, 0, None) == 1                  # ldx < N
    assert dyt.dyt_forward_strided(0, 4, 0, 0, 0, 0, 3, 5, 4, 0, 0, None) == 1                  # ldy < N
    assert dyt.dyt_forward_strided(0, 2**61, 0, 0, 0, 0, 4, 5, 4, 0, 0, None) == 1              # offsets overflow
    assert dyt.dyt_backward_strided(0, 4, 0, 2, 0, 0, None, 0, 4, 0, 0, 1, 5, 4, 0, 0, 0, 0, None) == 1  # lddy < N
    assert dyt.dyt_backward_strided(0, 4, 0, 4, 0, 0, None, 0, 3, 0, 0, 1, 5, 4, 0, 0, 0, 0, None) == 1  # lddx < N
    assert dyt.dyt_forward_strided(0, 9, 0, 0, 0, 0, 9, 0, 4, 0, 0, None) == 0                  # empty
    assert dyt.dyt_backward_workspace_bytes(-1, 3, 0, 0) == 0
    assert dyt.dyt_backward_workspace_bytes(0, 3, 0, 0) == 0
    from elementwise_reduction_b200 import _abi
    assert _abi.dyt_backward_workspace_bytes_strided(-1, 3, 3, 3, 3, 0, 0) == 0
    assert _abi.dyt_backward_workspace_bytes_strided(0, 3, 5, 5, 5, 0, 0) == 0   # empty: no workspace
    assert _abi.dyt_backward_workspace_bytes_strided(4, 3, 5, 5, 5, 9, 0) == 0   # bad dtype
    for s in range(5):
        assert dyt.dyt_status_string(s).startswith("DYT_")
    assert dyt.dyt_status_string(99) == "DYT_ERR_UNKNOWN"


def test_pointers_must_hold_whole_elements():
    # Every pointer is checked before anything runs, so fake device addresses
    # suffice: a tensor off its element boundary is an argument error.
    dyt = _lib()
    A, W = 1 << 20, 1 << 20  # 16-byte aligned stand-ins (W: the workspace)
    assert dyt.dyt_forward(A + 1, A, A, A, A, 4, 8, 1, 0, None) == 1                 # bf16 x one byte off
    assert dyt.dyt_forward(A, A, A, A, A + 3, 4, 8, 1, 0, None) == 1                 # bf16 y
    assert dyt.dyt_forward(A, A, A + 2, A, A, 4, 8, 1, 0, None) == 1                 # fp32 gamma
    assert dyt.dyt_forward(A, A, A, A + 6, A, 4, 8, 1, 0, None) == 1                 # fp32 beta
    assert dyt.dyt_forward_ex(A, 8, A + 1, A, A, A, 8, 4, 8, 1, 1, 0, 0, None) == 1  # bf16 alpha
    bw = lambda x=A, dy=A, al=A, ga=A, dx=A, dg=A, db=A, da=A: dyt.dyt_backward(
        x, dy, al, ga, None, dx, dg, db, da, 4, 8, 1, 0, W, 1 << 20, None)
    assert bw(x=A + 1) == 1 and bw(dy=A + 1) == 1 and bw(dx=A + 1) == 1   # bf16 activations
    assert bw(al=A + 2) == 1 and bw(ga=A + 2) == 1                        # fp32 parameters
    assert bw(dg=A + 2) == 1 and bw(db=A + 2) == 1 and bw(da=A + 2) == 1  # fp32 gradients
    empty = {"bytes": 0, "off_dgamma": 0, "off_dbeta": 0, "off_dalpha": 0, "rows": 0, "dalpha_parts": 0}
    assert dyt.dyt_finalize_partials([W], [empty], 4, A + 2, A, A, 0, 0, 0, None) == 1
    assert dyt.dyt_finalize_partials([W], [empty], 4, A, A, A + 1, 1, 1, 1, None) == 1  # bf16 dalpha


@pytest.mark.parametrize("M,N,xd", [(1024, 64, 0), (65537, 32, 1), (100003, 17, 0), (100003, 100, 0),
                                    (100003, 255, 0), (16384, 4096, 1), (32768, 8192, 1), (1, 1, 0),
                                    (3, 70000, 2), (10**7, 8, 1), (5, 513, 0), (7, 3, 1), (1, 17, 0),
                                    (100003, 4097, 1), (4099, 1001, 0)])
@pytest.mark.parametrize("layout,shift", [(0, 0), (1, 0), (2, 0), (2, 1), (2, -1), (3, 0), (3, 1), (3, -1),
                                          (4, 0), (4, 1)])
@pytest.mark.parametrize("sms,occ", [(148, 1), (148, 2), (7, 1)])
def test_launch_plan_invariants(M, N, xd, layout, shift, sms, occ):
    dyt = _lib()
    size = 4 if xd == 0 else 2
    sh = shift % (16 // size) if layout >= 2 else 0
    p = dyt.dyt_plan_query(M, N, xd, 0, 1, layout, sms, occ, shift=sh)
    vec = p["vec"]
    pk = p["pack_rows"]
    # strided rows of whole-vector pitches, off a boundary or of a ragged N:
    # the row frame
    rf = layout == 4 or (layout == 3 and (sh != 0 or N % (16 // size) != 0))
    # every tensor at the output's offset sh > 0 and N a multiple of the
    # vector: the first vector-column also holds each row's last sh elements
    wrap = layout == 3 and sh != 0 and N % (16 // size) == 0
    # adjacent rows always take the 16-byte kernels (packed when N is ragged);
    # tensors off 16-byte boundaries the shifted ones; strided rows of
    # whole-vector pitches too
    assert bool(p["async_stages"]) == (layout != 0)
    assert p["shifted"] == (3 if wrap else 2 if rf else 1 if layout == 2 else 0) and p["shift"] == sh
    if p["async_stages"]:    # per-thread copy ring: 16-byte vectors, one per thread
        assert vec == 16 // size
        # a ragged N on adjacent rows is streamed in packs of vec rows (exactly
        # N vectors each)
        assert pk == (vec if N % vec and layout in (1, 2) else 1)
        ctas = sms             # the 16-byte kernels run one CTA per SM
    else:
        assert vec == 1 and pk == 1
        ctas = sms * occ
    # pitch of a (packed) row; the row frame: a row's vectors from position sh
    Np = N if wrap else -(-(N + sh) // vec) * vec if rf else pk * N
    Mp = -(-(M * N + sh) // Np) if layout == 2 else -(-M // pk)  # (packed) rows; shifted: the matrix from position sh
    nv = Np // vec
    B = p["block"]
    # the backward over narrow rows (at most 32 vectors) runs 256-thread CTAs with 8-slot rings
    assert B == (1024 if not p["async_stages"] else 256 if nv <= 32 else 512) and p["kernels"] == 2
    if p["async_stages"]:
        assert p["async_stages"] == (8 if B == 256 else 6)
    assert 1 <= p["grid"] <= ctas                  # persistent 1D grid: never beyond one wave
    if p["path"] == 1:                             # row-tiled: several rows per CTA step
        assert p["row_lanes"] == B // nv >= 2 and p["col_chunks"] == 1
    else:                                          # row-per-CTA: columns across the CTA
        assert p["row_lanes"] == 1 and p["col_chunks"] == -(-nv // B)
    if p["async_stages"]:
        assert p["rows_per_step"] == p["row_lanes"] * pk
    items = p["row_groups"] * p["col_chunks"]
    assert p["grid"] <= items
    # every lane visits at most 2048 (packed) rows per group: the kernels' exact
    # multiply-high row counts need it
    rows_per_group = -(-Mp // p["row_groups"])
    assert -(-rows_per_group // p["row_lanes"]) <= 2048
    # every CTA gets the same number of work items, unless there are more
    # column chunks than CTAs
    if p["col_chunks"] <= ctas:
        assert items % p["grid"] == 0
        assert p["grid"] > ctas // 2 or p["grid"] == items
    # workspace: binary64 dgamma and dbeta partials per group and row position
    # (pack_rows x N of them) + binary64 dalpha per CTA
    al = lambda v: (v + 15) // 16 * 16
    assert p["workspace_bytes"] == 2 * al(p["row_groups"] * pk * N * 8) + al(p["grid"] * 8)


def test_plans_whose_counts_overflow_are_rejected():
    dyt = _lib()
    # 2^40 rows of 5000 unaligned fp32 columns: 5 column chunks of 1024 threads
    # and groups of at most 2048 rows would need about 2.7e9 work items, more
    # than an int holds
    with pytest.raises(dyt.DytError) as e:
        dyt.dyt_plan_query(2**40, 5000, 0, 0, 1, 0, 148, 1)
    assert e.value.status == 1
    p = dyt.dyt_plan_query(2**20, 300, 0, 0, 1, 0, 148, 1)
    assert p["row_lanes"] == 3 and p["row_groups"] == -(-(-(-2**20 // (3 * 2048))) // 148) * 148


def test_page_narrow_widths_take_the_row_tiled_path():
    dyt = _lib()
    for N in (16, 17, 32, 64, 100, 128, 255, 256):
        for xd in (0, 1, 2):
            p = dyt.dyt_plan_query(65537, N, xd, 0, 1, 1, 148, 1)
            assert p["path"] == 1 and p["rows_per_step"] > 1
    assert dyt.dyt_plan_query(32768, 8192, 1, 0, 1, 1, 148, 1)["path"] == 2


def test_multiply_high_quotients_are_exact():
    # The kernels divide by the row-lane count RL (2..1024) with a host constant
    # m = ceil(2^32 / RL): q = (n * m) >> 32. Groups hold at most 2048 RL rows,
    # so n < 2049 RL + RL; every quotient in that range must be exact (checked
    # at and around each multiple of RL, where an error would first show).
    import numpy as np
    for RL in range(2, 1025):
        m = ((1 << 32) + RL - 1) // RL
        k = np.arange(0, 2051, dtype=np.uint64)
        n = np.concatenate([k * RL, k * RL + RL - 1, np.maximum(k * RL, 1) - 1]).astype(np.uint64)
        n = n[n < 2050 * RL]
        q = (n * np.uint64(m)) >> np.uint64(32)
        assert np.array_equal(q, n // np.uint64(RL)), RL


def test_package_refuses_to_load_without_the_cuda_library(tmp_path):
    # A copy of the Python package with no libdyt.so next to it must fail on
    # import: there is no fallback implementation to run instead.
    import shutil
    import subprocess
    import sys
    pkg = os.path.join(ROOT, "elementwise_reduction_b200")
    dst = tmp_path / "elementwise_reduction_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "csrc", "__pycache__"))
    r = subprocess.run([sys.executable, "-c", "import elementwise_reduction_b200"], cwd=tmp_path,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "libdyt.so is missing" in r.stderr


def test_binding_scratch_size_matches_the_header():
    # The Python binding keeps its own copy of DYT_NOALLOC_SCRATCH_BYTES (ctypes
    # cannot read a #define); it must equal the header's value.
    dyt = _lib()
    text = open(HEADER).read()
    m = re.search(r"#define\s+DYT_NOALLOC_SCRATCH_BYTES\s+\(([^)]*)\)", text)
    assert m, "DYT_NOALLOC_SCRATCH_BYTES not found in include/dyt.h"
    value = eval(re.sub(r"(\d+)u\b", r"\1", m.group(1)), {"__builtins__": {}})
    assert value == dyt._abi.NOALLOC_SCRATCH_BYTES
