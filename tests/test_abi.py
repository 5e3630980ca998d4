"""The C ABI without a GPU: exported symbols, struct layout, host-side checks.

Every call below fails its argument or workspace checks before any CUDA call,
so it runs on a machine without a GPU.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mlg.h")


@pytest.fixture(scope="module")
def mlg():
    from neighbour_graph_attention_b200 import build

    build.build()
    from neighbour_graph_attention_b200 import mlg as m

    return m


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(mlg_[a-z_0-9]+)\s*\(", text, re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(mlg):
    names = _declared_functions()
    assert {"mlg_build_csr", "mlg_block_attention", "mlg_forward"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", mlg.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)$", out, re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(mlg.lib(), n)


def test_struct_layout_matches_c(mlg, tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "mlg.h"\n'
        "int main(void){\n"
        ' printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(mlg_system), offsetof(mlg_system, coords),'
        " offsetof(mlg_system, n_types), offsetof(mlg_system, box), offsetof(mlg_system, pbc),"
        " sizeof(mlg_csr));\n"
        ' printf("%zu %zu\\n", offsetof(mlg_csr, sw), offsetof(mlg_csr, status));\n'
        " return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src),
                           "-o", str(exe)])
    lines = subprocess.check_output([str(exe)], text=True).split("\n")
    a = list(map(int, lines[0].split()))
    b = list(map(int, lines[1].split()))
    S, C = mlg.mlg_system, mlg.mlg_csr
    assert a == [ctypes.sizeof(S), S.coords.offset, S.n_types.offset, S.box.offset,
                 S.pbc.offset, ctypes.sizeof(C)]
    assert b == [C.sw.offset, C.status.offset]


def test_status_strings(mlg):
    for code in range(7):
        assert mlg.mlg_status_string(code).startswith("MLG_")
    assert "unknown" in mlg.mlg_status_string(99)
    assert mlg.mlg_version() >= 100


FAKE = 0x1000  # a non-null device address that no host check dereferences


def _fake_csr(mlg, capacity=100):
    c = mlg.mlg_csr()
    c.capacity = capacity
    for name in ("row_ptr", "src", "shift", "vec", "dist", "sw", "n_edges", "n_truncated",
                 "status"):
        setattr(c, name, FAKE)
    return c


def _sys(mlg, n=64, box=None, pbc=(1, 1, 1)):
    s = mlg.mlg_system()
    s.n_atoms = n
    s.coords = FAKE
    s.types = None
    s.n_types = 0
    s.box[:] = list(np.ravel(np.diag([10.0] * 3) if box is None else box))
    s.pbc[:] = list(pbc)
    return s


def _build(mlg, sys_, rcut=4.0, r_on=3.5, nnei=40, csr=None, ws=None, ws_bytes=0):
    csr = csr or _fake_csr(mlg)
    return mlg.lib().mlg_build_csr(ctypes.byref(sys_), rcut, r_on, nnei, ctypes.byref(csr),
                                   ws, ws_bytes, None)


def test_host_argument_checks(mlg):
    assert _build(mlg, _sys(mlg, n=0)) == mlg.MLG_ERR_INVALID_ARG
    assert _build(mlg, _sys(mlg), rcut=-1.0) == mlg.MLG_ERR_INVALID_ARG
    assert _build(mlg, _sys(mlg), r_on=4.0) == mlg.MLG_ERR_INVALID_ARG      # r_on >= rcut
    assert _build(mlg, _sys(mlg), nnei=0) == mlg.MLG_ERR_INVALID_ARG
    assert _build(mlg, _sys(mlg), nnei=257) == mlg.MLG_ERR_UNSUPPORTED
    bad_box = np.diag([10.0] * 3); bad_box[0, 1] = 1.0
    assert _build(mlg, _sys(mlg, box=bad_box)) == mlg.MLG_ERR_UNSUPPORTED   # sheared cell
    nan_box = np.diag([10.0, np.nan, 10.0])
    assert _build(mlg, _sys(mlg, box=nan_box)) == mlg.MLG_ERR_INVALID_ARG
    zero_len = np.diag([10.0, 0.0, 10.0])
    assert _build(mlg, _sys(mlg, box=zero_len)) == mlg.MLG_ERR_INVALID_ARG
    # an open axis ignores its box row: a zero row is fine there
    assert _build(mlg, _sys(mlg, box=zero_len, pbc=(1, 0, 1))) == mlg.MLG_ERR_WORKSPACE
    assert _build(mlg, _sys(mlg), csr=_fake_csr(mlg, capacity=-1)) == mlg.MLG_ERR_CAPACITY
    c = _fake_csr(mlg); c.row_ptr = None
    assert _build(mlg, _sys(mlg), csr=c) == mlg.MLG_ERR_INVALID_ARG
    # a box far smaller than rcut: stencil beyond the supported reach
    assert _build(mlg, _sys(mlg, box=np.diag([0.05] * 3)), rcut=4.0) == mlg.MLG_ERR_UNSUPPORTED


def test_workspace_checks(mlg):
    s = _sys(mlg)
    need = mlg.mlg_build_csr_workspace_bytes(64, 4.0, np.diag([10.0] * 3), [1, 1, 1])
    assert need > 0
    assert _build(mlg, s, ws=None, ws_bytes=need) == mlg.MLG_ERR_WORKSPACE
    assert _build(mlg, s, ws=FAKE * 16, ws_bytes=need - 1) == mlg.MLG_ERR_WORKSPACE
    assert _build(mlg, s, ws=FAKE * 16 + 8, ws_bytes=need) == mlg.MLG_ERR_WORKSPACE  # misaligned
    assert mlg.mlg_build_csr_workspace_bytes(0, 4.0, np.diag([10.0] * 3), [1, 1, 1]) == 0
    # open axes: the cell budget bounds the workspace whatever the coordinates
    # (about 100 bytes per atom, plus 516 for the count-to-fill key stash of
    # the kernel chain: 5,964 atoms is past the one-launch build)
    w_open = mlg.mlg_build_csr_workspace_bytes(5964, 5.0, np.zeros((3, 3)), [0, 0, 0])
    assert 5964 * 516 < w_open < 5964 * 1000
    # forward adds one ping-pong feature buffer for >= 2 layers
    f1 = mlg.mlg_forward_workspace_bytes(64, 4.0, np.diag([10.0] * 3), [1, 1, 1], 1000, 32, 1, 1)
    f2 = mlg.mlg_forward_workspace_bytes(64, 4.0, np.diag([10.0] * 3), [1, 1, 1], 1000, 32, 2, 1)
    assert f1 == need and f2 >= need + 1000 * 32 * 8


def test_attention_argument_checks(mlg):
    lib = mlg.lib()
    c = _fake_csr(mlg)
    call = lambda **k: lib.mlg_block_attention(
        ctypes.byref(c), k.get("n", 10), k.get("nnei", 40), k.get("ch", 32), k.get("heads", 4),
        k.get("dtype", 1), k.get("gin", FAKE), k.get("gout", FAKE * 2), FAKE, FAKE, FAKE,
        None, 0, None)
    assert call(heads=3) == mlg.MLG_ERR_INVALID_ARG          # channels % heads != 0
    assert call(gin=None) == mlg.MLG_ERR_INVALID_ARG
    assert call(gout=FAKE) == mlg.MLG_ERR_INVALID_ARG        # aliasing in/out
    assert call(dtype=7) == mlg.MLG_ERR_INVALID_ARG
    assert call(ch=512, heads=8) == mlg.MLG_ERR_UNSUPPORTED
    assert call(ch=256, heads=2) == mlg.MLG_ERR_UNSUPPORTED  # head size 128 > 64
    assert call(nnei=300) == mlg.MLG_ERR_UNSUPPORTED
    assert call(n=-1) == mlg.MLG_ERR_INVALID_ARG


def test_product_path_fails_loudly_without_library(tmp_path):
    # the binding has no fallback: a missing library is an import error
    code = (
        "import importlib.util, sys\n"
        f"spec = importlib.util.spec_from_file_location('m', r'{ROOT}/neighbour_graph_attention_b200/mlg.py')\n"
        "m = importlib.util.module_from_spec(spec)\n"
        "import os\n"
        "os.path.exists = lambda p: False\n"
        "try:\n"
        "    spec.loader.exec_module(m)\n"
        "except ImportError as e:\n"
        "    print('IMPORT_ERROR', 'no CPU fallback' in str(e))\n")
    out = subprocess.run(["python", "-c", code], capture_output=True, text=True)
    assert "IMPORT_ERROR True" in out.stdout, out.stdout + out.stderr


def test_batch_workspace_and_checks(mlg):
    """Host side of the batched build: workspace sizes and argument checks
    (no kernel runs: every call below fails a host check)."""
    lib = mlg.lib()
    a, b = _sys(mlg, 64), _sys(mlg, 200, box=np.zeros((3, 3)), pbc=(0, 0, 0))
    empty = _sys(mlg, 0)
    one_a = mlg.mlg_build_csr_workspace_bytes(64, 4.0, np.diag([10.0] * 3), [1, 1, 1])
    one_b = mlg.mlg_build_csr_workspace_bytes(200, 4.0, np.zeros((3, 3)), [0, 0, 0])
    both = mlg.mlg_build_csr_batch_workspace_bytes([a, empty, b], 4.0)
    assert both >= one_a + one_b                       # each system's own workspace, plus counts
    assert mlg.mlg_build_csr_batch_workspace_bytes([], 4.0) > 0
    assert mlg.mlg_build_csr_batch_workspace_bytes([a], -1.0) == 0
    assert mlg.mlg_build_csr_batch_workspace_bytes([_sys(mlg, -3)], 4.0) == 0
    arr = mlg._system_array([a, b])
    csr = _fake_csr(mlg)
    call = lambda n=2, rcut=4.0, r_on=3.5, nnei=40, ws=None, nb=0: lib.mlg_build_csr_batch(
        arr, n, rcut, r_on, nnei, ctypes.byref(csr), ws, nb, None)
    assert call(ws=None, nb=both) == mlg.MLG_ERR_WORKSPACE
    assert call(ws=FAKE * 16, nb=both - 1) == mlg.MLG_ERR_WORKSPACE
    assert call(n=-1, ws=FAKE * 16, nb=both) == mlg.MLG_ERR_INVALID_ARG
    assert call(r_on=5.0, ws=FAKE * 16, nb=both) == mlg.MLG_ERR_INVALID_ARG
    assert call(nnei=999, ws=FAKE * 16, nb=both) == mlg.MLG_ERR_UNSUPPORTED


def test_local_and_smooth_argument_checks(mlg):
    """Host checks of the local and slot-occupancy attention calls.  Every
    call below returns before a kernel is launched (a host check fails, or
    there is no centre), so fake device pointers are never dereferenced."""
    lib = mlg.lib()
    c = _fake_csr(mlg)
    smooth = lambda **k: lib.mlg_block_attention_smooth(
        ctypes.byref(c), k.get("n", 10), k.get("nnei", 40), k.get("ch", 32), k.get("heads", 4),
        k.get("dtype", 1), k.get("gin", FAKE), k.get("gout", FAKE * 2), k.get("wq", FAKE),
        FAKE, FAKE, None)
    assert smooth(heads=3) == mlg.MLG_ERR_INVALID_ARG
    assert smooth(gout=FAKE) == mlg.MLG_ERR_INVALID_ARG      # aliasing in/out
    assert smooth(wq=None) == mlg.MLG_ERR_INVALID_ARG
    assert smooth(nnei=300) == mlg.MLG_ERR_UNSUPPORTED
    assert smooth(dtype=5) == mlg.MLG_ERR_INVALID_ARG
    assert smooth(n=0) == mlg.MLG_OK                          # nothing to do, nothing launched
    local = lambda **k: lib.mlg_local_attention(
        ctypes.byref(c), k.get("n", 10), k.get("nnei", 40), k.get("ch", 32), k.get("heads", 4),
        k.get("dtype", 1), k.get("h", FAKE * 3), k.get("gin", FAKE), k.get("out", FAKE * 2),
        FAKE, FAKE, k.get("wv", FAKE), None)
    assert local(h=None) == mlg.MLG_ERR_INVALID_ARG
    assert local(h=FAKE * 2) == mlg.MLG_ERR_INVALID_ARG      # query rows alias the output
    assert local(wv=None) == mlg.MLG_ERR_INVALID_ARG
    assert local(ch=64, heads=5) == mlg.MLG_ERR_INVALID_ARG
    assert local(ch=512, heads=8) == mlg.MLG_ERR_UNSUPPORTED
    assert local(n=-2) == mlg.MLG_ERR_INVALID_ARG
    assert local(n=0) == mlg.MLG_OK


def _prototypes():
    """name -> (return type, [parameter types]) for every function the header declares."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    protos = {}
    for m in re.finditer(r"^\s*((?:const\s+)?[a-z_0-9]+\s*\*?)\s*(mlg_[a-z_0-9]+)\s*\(([^)]*)\)\s*;",
                         text, re.M):
        ret, name, params = m.group(1), m.group(2), m.group(3).strip()
        plist = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
        protos[name] = (ret.strip(), plist)
    return protos


def _c_kind(decl):
    """The ctypes class of a C declaration (a parameter or a return type);
    int and the int-sized enum are 32-bit here, like int32_t."""
    decl = re.sub(r"\bconst\b", "", decl)
    if "*" in decl or "[" in decl or re.search(r"\bmlg_stream_t\b", decl):
        return "ptr"
    for ctype, kind in (("int64_t", "i64"), ("int32_t", "i32"), ("size_t", "size"),
                        ("double", "f64"), ("mlg_dtype", "i32"), ("int", "i32"), ("void", None)):
        if re.search(r"\b%s\b" % ctype, decl):
            return kind
    raise AssertionError("unclassified C type: " + decl)


def _ct_kind(t):
    if t is None:
        return None
    if t in (ctypes.c_void_p, ctypes.c_char_p) or issubclass(t, ctypes._Pointer):
        return "ptr"
    kinds = {ctypes.c_int64: "i64", ctypes.c_size_t: "size", ctypes.c_double: "f64",
             ctypes.c_int32: "i32", ctypes.c_int: "i32"}
    return kinds.get(t, repr(t))


def test_binding_signatures_match_header(mlg):
    # each ctypes declaration of the binding has the header's parameter count
    # and widths, so a call through Python marshals what the C side reads
    protos = _prototypes()
    assert set(protos) == set(_declared_functions())
    lib = mlg.lib()
    for name, (ret, params) in sorted(protos.items()):
        fn = getattr(lib, name)
        assert fn.argtypes is not None, name + ": no argtypes in the binding"
        want = [_c_kind(p) for p in params]
        got = [_ct_kind(t) for t in fn.argtypes]
        assert got == want, (name, got, want)
        want_ret = "ptr" if "*" in ret else _c_kind(ret)
        assert _ct_kind(fn.restype) == want_ret, (name, fn.restype, ret)


def test_forward_launch_counts(mlg):
    """The kernel launches of one mlg_forward, as the benchmark counts them
    (a host-side plan, no GPU):
      diamond-64:    one-launch build + c = 128 head-group attention (1 layer)    = 2
      diamond-512:   one-launch build + one fused launch for all 6 layers        = 2
      Fe BCC 65,536: init, bin, cell scan, scatter, count, row scan (3), fill,
                     + fused tile and the generic kernel for rows over 128       = 11
      protein 5,964: init, bounding box, bin, cell scan (3), scatter, count,
                     row scan, fill, + head-group kernel per layer (2)           = 12
      Fe BCC 524,288: init, bin, cell scan (3), scatter, count, row scan (3),
                     fill, + the tcgen05-logits kernel for rows up to 64 and the
                     fused tile for rows of 65-128                               = 13"""
    from neighbour_graph_attention_b200 import configs as C

    want = {1: 2, 2: 2, 3: 11, 4: 12, 5: 13}
    for key, n in want.items():
        w = C.workload(key)
        L = w.a * w.cells if w.periodic else 0.0
        box = np.diag([L] * 3) if w.periodic else np.zeros((3, 3))
        pbc = [1, 1, 1] if w.periodic else [0, 0, 0]
        dt = mlg.MLG_F64 if w.dtype == "f64" else mlg.MLG_F32
        got = mlg.mlg_forward_launch_count(w.n_atoms, w.rcut, box, pbc, w.nnei_max, w.channels,
                                           w.heads, w.n_layers, dt)
        assert got == n, (w.name, got, n)


def test_recorded_attention_traffic_names_the_launched_kernels(mlg):
    """bench.py reports a stored DRAM capture as roofline.traffic only while
    the library still launches the kernels it was taken on: each record must
    name exactly what mlg_attention_kernels() returns for its workload, so that
    a kernel change makes the stale figure drop out (and this test fail)."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from neighbour_graph_attention_b200 import configs as C

    assert bench.ATTN_TRAFFIC
    for key, (name, traffic) in bench.ATTN_TRAFFIC.items():
        w = C.workload(key)
        dt = mlg.MLG_F64 if w.dtype == "f64" else mlg.MLG_F32
        launched = mlg.mlg_attention_kernels(w.nnei_max, w.channels, w.heads, w.n_layers, dt)
        assert launched == name, (key, launched, name)
        assert traffic > 0


def test_workspace_holds_the_key_stash_only_for_the_kernel_chain(mlg):
    """Systems past the one-launch build get 516 bytes per atom more (the
    count-to-fill key stash: 64 keys of 8 bytes and a count); the one-launch
    build needs none."""
    L64 = 2.855 * 32
    chain = mlg.mlg_build_csr_workspace_bytes(65536, 6.0, np.diag([L64] * 3), [1, 1, 1])
    assert chain > 65536 * 516
    small = mlg.mlg_build_csr_workspace_bytes(512, 2.4, np.diag([3.567 * 4] * 3), [1, 1, 1])
    assert 0 < small < 512 * 516
