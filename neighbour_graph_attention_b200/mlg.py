"""Thin ctypes binding of libmlg.so (include/mlg.h).

Argument marshalling only: every step of the neighbour-graph hot path runs in
the library's CUDA kernels. Torch tensors provide device memory and streams.
There is no fallback: if ``libmlg.so`` is missing, importing this module
raises.

Names match the C ABI: :func:`mlg_build_csr`, :func:`mlg_build_csr_batch`,
:func:`mlg_block_attention`, :func:`mlg_attention_stack`, :func:`mlg_forward`,
:func:`mlg_local_attention`, :func:`mlg_block_attention_smooth`, the
``*_workspace_bytes`` queries and :func:`mlg_status_string`. :class:`Csr`
bundles the caller-owned CSR buffers. Descriptors (:func:`make_system`,
``Csr.struct()``) hold raw device addresses: the tensors behind them must
outlive every call that uses them.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmlg.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m neighbour_graph_attention_b200.build` "
        "(nvcc, sm_100a). There is no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)

MLG_OK = 0
MLG_ERR_INVALID_ARG = 1
MLG_ERR_WORKSPACE = 2
MLG_ERR_CAPACITY = 3
MLG_ERR_INPUT_DATA = 4
MLG_ERR_UNSUPPORTED = 5
MLG_ERR_CUDA = 6

MLG_STATUS_NONFINITE_COORD = 1
MLG_STATUS_TYPE_RANGE = 2
MLG_STATUS_CAPACITY = 4
MLG_STATUS_IMAGE_RANGE = 8
MLG_STATUS_TIES = 16
MLG_STATUS_INTERNAL = 32
MLG_STATUS_TIMEOUT = 64
MLG_STATUS_ROW_TOO_LONG = 128
MLG_STATUS_LIST_INCOMPLETE = 256

MLG_F32 = 0
MLG_F64 = 1

_c_i64, _c_i32, _c_dbl, _c_sz, _p = (ctypes.c_int64, ctypes.c_int32, ctypes.c_double,
                                     ctypes.c_size_t, ctypes.c_void_p)


class mlg_system(ctypes.Structure):
    _fields_ = [("n_atoms", _c_i64), ("coords", _p), ("types", _p), ("n_types", _c_i32),
                ("box", _c_dbl * 9), ("pbc", ctypes.c_uint8 * 3)]


class mlg_csr(ctypes.Structure):
    _fields_ = [("capacity", _c_i64), ("row_ptr", _p), ("src", _p), ("shift", _p), ("vec", _p),
                ("dist", _p), ("sw", _p), ("n_edges", _p), ("n_truncated", _p), ("status", _p)]


class mlg_verlet_list(ctypes.Structure):
    _fields_ = [("cand", mlg_csr), ("coords_ref", _p), ("state", _p), ("n_builds", _p)]


_lib.mlg_build_csr_workspace_bytes.restype = _c_sz
_lib.mlg_build_csr_workspace_bytes.argtypes = [_c_i64, _c_dbl, _p, _p]
_lib.mlg_build_csr.restype = ctypes.c_int
_lib.mlg_build_csr.argtypes = [ctypes.POINTER(mlg_system), _c_dbl, _c_dbl, _c_i32,
                               ctypes.POINTER(mlg_csr), _p, _c_sz, _p]
_lib.mlg_attention_workspace_bytes.restype = _c_sz
_lib.mlg_attention_workspace_bytes.argtypes = [_c_i64, _c_i32, _c_i32, _c_i32, ctypes.c_int]
_lib.mlg_block_attention.restype = ctypes.c_int
_lib.mlg_block_attention.argtypes = [ctypes.POINTER(mlg_csr), _c_i64, _c_i32, _c_i32, _c_i32,
                                     ctypes.c_int, _p, _p, _p, _p, _p, _p, _c_sz, _p]
_lib.mlg_forward_workspace_bytes.restype = _c_sz
_lib.mlg_forward_workspace_bytes.argtypes = [_c_i64, _c_dbl, _p, _p, _c_i64, _c_i32, _c_i32,
                                             ctypes.c_int]
_lib.mlg_forward.restype = ctypes.c_int
_lib.mlg_forward.argtypes = [ctypes.POINTER(mlg_system), _c_dbl, _c_dbl, _c_i32, _c_i32, _c_i32,
                             _c_i32, ctypes.c_int, ctypes.POINTER(_p), _p, _p,
                             ctypes.POINTER(mlg_csr), _p, _c_sz, _p]
_lib.mlg_build_csr_noalloc.restype = ctypes.c_int
_lib.mlg_build_csr_noalloc.argtypes = [ctypes.POINTER(mlg_system), _c_dbl, _c_dbl, _c_i32,
                                       ctypes.POINTER(mlg_csr), _p]
_lib.mlg_forward_launch_count.restype = ctypes.c_int
_lib.mlg_forward_launch_count.argtypes = [_c_i64, _c_dbl, _p, _p, _c_i32, _c_i32, _c_i32, _c_i32,
                                          ctypes.c_int]
_lib.mlg_attention_stack_workspace_bytes.restype = _c_sz
_lib.mlg_attention_stack_workspace_bytes.argtypes = [_c_i64, _c_i32, _c_i32, ctypes.c_int]
_lib.mlg_attention_stack.restype = ctypes.c_int
_lib.mlg_attention_stack.argtypes = [ctypes.POINTER(mlg_csr), _c_i64, _c_i32, _c_i32, _c_i32,
                                     _c_i32, ctypes.c_int, ctypes.POINTER(_p), _p, _p, _p, _c_sz,
                                     _p]
_lib.mlg_attention_stack_smooth.restype = ctypes.c_int
_lib.mlg_attention_stack_smooth.argtypes = [ctypes.POINTER(mlg_csr), _c_i64, _c_i32, _c_i32,
                                            _c_i32, _c_i32, ctypes.c_int, ctypes.POINTER(_p), _p,
                                            _p, _p, _c_sz, _p]
_lib.mlg_build_csr_batch_workspace_bytes.restype = _c_sz
_lib.mlg_build_csr_batch_workspace_bytes.argtypes = [ctypes.POINTER(mlg_system), _c_i32, _c_dbl]
_lib.mlg_build_csr_batch.restype = ctypes.c_int
_lib.mlg_build_csr_batch.argtypes = [ctypes.POINTER(mlg_system), _c_i32, _c_dbl, _c_dbl, _c_i32,
                                     ctypes.POINTER(mlg_csr), _p, _c_sz, _p]
_lib.mlg_block_attention_smooth.restype = ctypes.c_int
_lib.mlg_block_attention_smooth.argtypes = [ctypes.POINTER(mlg_csr), _c_i64, _c_i32, _c_i32,
                                            _c_i32, ctypes.c_int, _p, _p, _p, _p, _p, _p]
_lib.mlg_local_attention.restype = ctypes.c_int
_lib.mlg_local_attention.argtypes = [ctypes.POINTER(mlg_csr), _c_i64, _c_i32, _c_i32, _c_i32,
                                     ctypes.c_int, _p, _p, _p, _p, _p, _p, _p]
_lib.mlg_exp2_neg.restype = ctypes.c_int
_lib.mlg_exp2_neg.argtypes = [_p, _p, _c_i64, _p]
_lib.mlg_verlet_workspace_bytes.restype = _c_sz
_lib.mlg_verlet_workspace_bytes.argtypes = [_c_i64, _c_dbl, _c_dbl, _p, _p]
_lib.mlg_verlet_step.restype = ctypes.c_int
_lib.mlg_verlet_step.argtypes = [ctypes.POINTER(mlg_system), _c_dbl, _c_dbl, _c_dbl, _c_i32,
                                 ctypes.POINTER(mlg_verlet_list), ctypes.POINTER(mlg_csr), _p,
                                 _c_sz, _p]
_lib.mlg_build_csr_wait_test.restype = ctypes.c_int
_lib.mlg_build_csr_wait_test.argtypes = [ctypes.POINTER(mlg_system), _c_dbl, _c_dbl, _c_i32,
                                         ctypes.POINTER(mlg_csr), _p, _c_sz, _c_i32, _p]
_lib.mlg_attention_kernels.restype = ctypes.c_char_p
_lib.mlg_attention_kernels.argtypes = [_c_i32, _c_i32, _c_i32, _c_i32, ctypes.c_int]
_lib.mlg_status_string.restype = ctypes.c_char_p
_lib.mlg_status_string.argtypes = [ctypes.c_int]
_lib.mlg_version.restype = ctypes.c_int
_lib.mlg_version.argtypes = []


class MlgError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {mlg_status_string(code)}")
        self.code = code


def lib() -> ctypes.CDLL:
    return _lib


def mlg_status_string(code: int) -> str:
    return _lib.mlg_status_string(int(code)).decode()


def mlg_exp2_neg(y, out, stream=None, check: bool = True) -> int:
    """out = 2^y elementwise by the fp64 attention's device exponential
    (diagnostics; y, out: device float64 tensors of equal length)."""
    rc = _lib.mlg_exp2_neg(_ptr(y), _ptr(out), int(y.numel()), _stream_handle(stream))
    if check and rc != MLG_OK:
        raise MlgError(rc, "mlg_exp2_neg")
    return rc


def mlg_attention_kernels(nnei_max: int, channels: int, heads: int, n_layers: int,
                          dtype: int) -> str:
    """The kernels mlg_attention_stack launches for this shape."""
    return _lib.mlg_attention_kernels(int(nnei_max), int(channels), int(heads), int(n_layers),
                                      int(dtype)).decode()


def mlg_version() -> int:
    return _lib.mlg_version()


def _ptr(t) -> int | None:
    if t is None:
        return None
    return int(t.data_ptr())


def _stream_handle(stream) -> int | None:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def _box_pbc(box, pbc):
    b = np.ascontiguousarray(np.asarray(box, dtype=np.float64).reshape(9))
    q = np.ascontiguousarray(np.asarray(pbc, dtype=np.uint8).reshape(3))
    return b, q


def make_system(coords, box, pbc, types=None, n_types: int = 0) -> mlg_system:
    """Fill an ``mlg_system`` from a CUDA float64 [N][3] tensor and host box/pbc."""
    b, q = _box_pbc(box, pbc)
    s = mlg_system()
    s.n_atoms = int(coords.shape[0])
    s.coords = _ptr(coords)
    s.types = _ptr(types)
    s.n_types = int(n_types)
    s.box[:] = b.tolist()
    s.pbc[:] = q.tolist()
    return s


@dataclass
class Csr:
    """Caller-owned device buffers of the destination CSR (torch tensors)."""

    capacity: int
    row_ptr: object
    src: object
    shift: object
    vec: object
    dist: object
    sw: object
    n_edges: object
    n_truncated: object
    status: object

    @classmethod
    def empty(cls, n_atoms: int, capacity: int, device="cuda"):
        import torch
        cap = max(int(capacity), 0)
        z = dict(device=device)
        return cls(cap, torch.zeros(n_atoms + 1, dtype=torch.int64, **z),
                   torch.zeros(max(cap, 1), dtype=torch.int32, **z),
                   torch.zeros((max(cap, 1), 3), dtype=torch.int32, **z),
                   torch.zeros((max(cap, 1), 3), dtype=torch.float64, **z),
                   torch.zeros(max(cap, 1), dtype=torch.float64, **z),
                   torch.zeros(max(cap, 1), dtype=torch.float64, **z),
                   torch.zeros(1, dtype=torch.int64, **z), torch.zeros(1, dtype=torch.int64, **z),
                   torch.zeros(1, dtype=torch.int32, **z))

    def struct(self) -> mlg_csr:
        c = mlg_csr()
        c.capacity = int(self.capacity)
        for name in ("row_ptr", "src", "shift", "vec", "dist", "sw", "n_edges", "n_truncated",
                     "status"):
            setattr(c, name, _ptr(getattr(self, name)))
        return c


def mlg_build_csr_workspace_bytes(n_atoms: int, rcut: float, box, pbc) -> int:
    b, q = _box_pbc(box, pbc)
    return int(_lib.mlg_build_csr_workspace_bytes(int(n_atoms), float(rcut),
                                                  b.ctypes.data, q.ctypes.data))


def mlg_attention_workspace_bytes(n_centres: int, nnei_max: int, channels: int, heads: int,
                                  dtype: int) -> int:
    return int(_lib.mlg_attention_workspace_bytes(int(n_centres), int(nnei_max), int(channels),
                                                  int(heads), int(dtype)))


def mlg_forward_workspace_bytes(n_atoms: int, rcut: float, box, pbc, capacity: int,
                                channels: int, n_layers: int, dtype: int) -> int:
    b, q = _box_pbc(box, pbc)
    return int(_lib.mlg_forward_workspace_bytes(int(n_atoms), float(rcut), b.ctypes.data,
                                                q.ctypes.data, int(capacity), int(channels),
                                                int(n_layers), int(dtype)))


def mlg_forward_launch_count(n_atoms: int, rcut: float, box, pbc, nnei_max: int,
                             channels: int, heads: int, n_layers: int, dtype: int) -> int:
    b, q = _box_pbc(box, pbc)
    return int(_lib.mlg_forward_launch_count(int(n_atoms), float(rcut), b.ctypes.data,
                                             q.ctypes.data, int(nnei_max), int(channels),
                                             int(heads), int(n_layers), int(dtype)))


def mlg_attention_stack_workspace_bytes(capacity: int, channels: int, n_layers: int,
                                        dtype: int) -> int:
    return int(_lib.mlg_attention_stack_workspace_bytes(int(capacity), int(channels),
                                                        int(n_layers), int(dtype)))


def mlg_attention_stack(csr: Csr, n_centres: int, nnei_max: int, channels: int, heads: int,
                        n_layers: int, dtype: int, W, G_in, G_out, ws=None,
                        ws_bytes: int | None = None, stream=None, check: bool = True) -> int:
    """Launch ``n_layers`` fused attention layers. ``W``: 3 * n_layers device tensors."""
    ptrs = (_p * len(W))(*[_ptr(w) for w in W])
    c = csr.struct()
    nbytes = 0 if ws is None else (int(ws.numel() * ws.element_size()) if ws_bytes is None
                                   else int(ws_bytes))
    code = _lib.mlg_attention_stack(ctypes.byref(c), int(n_centres), int(nnei_max),
                                    int(channels), int(heads), int(n_layers), int(dtype), ptrs,
                                    _ptr(G_in), _ptr(G_out), _ptr(ws), nbytes,
                                    _stream_handle(stream))
    return _check(code, "mlg_attention_stack", check)


def mlg_attention_stack_smooth(csr: Csr, n_centres: int, nnei_max: int, channels: int,
                               heads: int, n_layers: int, dtype: int, W, G_in, G_out, ws=None,
                               ws_bytes: int | None = None, stream=None,
                               check: bool = True) -> int:
    """``mlg_attention_stack`` with the slot-occupancy softmax in every layer."""
    ptrs = (_p * len(W))(*[_ptr(w) for w in W])
    c = csr.struct()
    nbytes = 0 if ws is None else (int(ws.numel() * ws.element_size()) if ws_bytes is None
                                   else int(ws_bytes))
    code = _lib.mlg_attention_stack_smooth(ctypes.byref(c), int(n_centres), int(nnei_max),
                                           int(channels), int(heads), int(n_layers),
                                           int(dtype), ptrs, _ptr(G_in), _ptr(G_out), _ptr(ws),
                                           nbytes, _stream_handle(stream))
    return _check(code, "mlg_attention_stack_smooth", check)


def _check(code: int, where: str, check: bool):
    if check and code != MLG_OK:
        raise MlgError(code, where)
    return code


def mlg_build_csr(system: mlg_system, rcut: float, r_on: float, nnei_max: int, csr: Csr,
                  ws, ws_bytes: int | None = None, stream=None, check: bool = True) -> int:
    """Launch the CSR build on ``stream`` (default: torch's current stream)."""
    c = csr.struct()
    nbytes = int(ws.numel() * ws.element_size()) if ws_bytes is None else int(ws_bytes)
    code = _lib.mlg_build_csr(ctypes.byref(system), float(rcut), float(r_on), int(nnei_max),
                              ctypes.byref(c), _ptr(ws), nbytes, _stream_handle(stream))
    return _check(code, "mlg_build_csr", check)


@dataclass
class VerletList:
    """Caller-owned device buffers of a Verlet candidate list (torch tensors):
    the candidate CSR at rcut + skin, the coordinates it was built at, its
    state word (zero: no valid list yet) and a counter of its builds."""

    cand: Csr
    coords_ref: object
    state: object
    n_builds: object

    @classmethod
    def empty(cls, n_atoms: int, capacity: int, device="cuda"):
        import torch
        return cls(Csr.empty(n_atoms, capacity, device=device),
                   torch.zeros((max(n_atoms, 1), 3), dtype=torch.float64, device=device),
                   torch.zeros(1, dtype=torch.int32, device=device),
                   torch.zeros(1, dtype=torch.int64, device=device))

    def struct(self) -> mlg_verlet_list:
        v = mlg_verlet_list()
        v.cand = self.cand.struct()
        v.coords_ref = _ptr(self.coords_ref)
        v.state = _ptr(self.state)
        v.n_builds = _ptr(self.n_builds)
        return v


def mlg_verlet_workspace_bytes(n_atoms: int, rcut: float, skin: float, box, pbc) -> int:
    b, q = _box_pbc(box, pbc)
    return int(_lib.mlg_verlet_workspace_bytes(int(n_atoms), float(rcut), float(skin),
                                               b.ctypes.data, q.ctypes.data))


def mlg_verlet_step(system: mlg_system, rcut: float, r_on: float, skin: float, nnei_max: int,
                    vlist: VerletList, out: Csr, ws, ws_bytes: int | None = None, stream=None,
                    check: bool = True) -> int:
    """One step's CSR through the Verlet list (rebuilt on the device when some
    atom has moved skin / 2 or more), written to ``out``."""
    v = vlist.struct()
    c = out.struct()
    nbytes = int(ws.numel() * ws.element_size()) if ws_bytes is None else int(ws_bytes)
    code = _lib.mlg_verlet_step(ctypes.byref(system), float(rcut), float(r_on), float(skin),
                                int(nnei_max), ctypes.byref(v), ctypes.byref(c), _ptr(ws),
                                nbytes, _stream_handle(stream))
    return _check(code, "mlg_verlet_step", check)


def mlg_build_csr_wait_test(system: mlg_system, rcut: float, r_on: float, nnei_max: int,
                            csr: Csr, ws, polls: int, stream=None, check: bool = True) -> int:
    """Diagnostics: the one-launch build with its bounded waits made to run
    out after ``polls`` polls (the device status then has MLG_STATUS_TIMEOUT)."""
    c = csr.struct()
    nbytes = int(ws.numel() * ws.element_size())
    code = _lib.mlg_build_csr_wait_test(ctypes.byref(system), float(rcut), float(r_on),
                                        int(nnei_max), ctypes.byref(c), _ptr(ws), nbytes,
                                        int(polls), _stream_handle(stream))
    return _check(code, "mlg_build_csr_wait_test", check)


MLG_NOALLOC_SCRATCH_BYTES = 8 << 20


def mlg_build_csr_noalloc(system: mlg_system, rcut: float, r_on: float, nnei_max: int,
                          csr: Csr, stream=None, check: bool = True) -> int:
    """The CSR build with the library's built-in scratch array: no workspace, no
    allocation (for callers that cannot allocate; see include/mlg.h). Calls
    that overlap on the GPU share that array and race, so order them."""
    c = csr.struct()
    code = _lib.mlg_build_csr_noalloc(ctypes.byref(system), float(rcut), float(r_on),
                                      int(nnei_max), ctypes.byref(c), _stream_handle(stream))
    return _check(code, "mlg_build_csr_noalloc", check)


def mlg_block_attention(csr: Csr, n_centres: int, nnei_max: int, channels: int, heads: int,
                        dtype: int, G_in, G_out, Wq, Wk, Wv, ws=None, ws_bytes: int = 0,
                        stream=None, check: bool = True) -> int:
    """Launch one block-dense attention layer on ``stream``."""
    c = csr.struct()
    code = _lib.mlg_block_attention(ctypes.byref(c), int(n_centres), int(nnei_max),
                                    int(channels), int(heads), int(dtype), _ptr(G_in),
                                    _ptr(G_out), _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(ws),
                                    int(ws_bytes), _stream_handle(stream))
    return _check(code, "mlg_block_attention", check)


def mlg_block_attention_smooth(csr: Csr, n_centres: int, nnei_max: int, channels: int,
                               heads: int, dtype: int, G_in, G_out, Wq, Wk, Wv, stream=None,
                               check: bool = True) -> int:
    """Launch one attention layer with the slot-occupancy (smooth) softmax."""
    c = csr.struct()
    code = _lib.mlg_block_attention_smooth(ctypes.byref(c), int(n_centres), int(nnei_max),
                                           int(channels), int(heads), int(dtype), _ptr(G_in),
                                           _ptr(G_out), _ptr(Wq), _ptr(Wk), _ptr(Wv),
                                           _stream_handle(stream))
    return _check(code, "mlg_block_attention_smooth", check)


def _system_array(systems):
    arr = (mlg_system * max(len(systems), 1))()
    for k, s in enumerate(systems):
        arr[k] = s
    return arr


def mlg_build_csr_batch_workspace_bytes(systems, rcut: float) -> int:
    """Workspace bytes of mlg_build_csr_batch for these mlg_system descriptors."""
    return _lib.mlg_build_csr_batch_workspace_bytes(_system_array(systems), len(systems),
                                                    float(rcut))


def mlg_build_csr_batch(systems, rcut: float, r_on: float, nnei_max: int, csr: Csr, ws,
                        ws_bytes: int | None = None, stream=None, check: bool = True) -> int:
    """Launch the build of one CSR over several systems (``systems``: a list of
    mlg_system descriptors, e.g. from make_system)."""
    c = csr.struct()
    nb = ws.numel() * ws.element_size() if ws_bytes is None else int(ws_bytes)
    code = _lib.mlg_build_csr_batch(_system_array(systems), len(systems), float(rcut),
                                    float(r_on), int(nnei_max), ctypes.byref(c), _ptr(ws), nb,
                                    _stream_handle(stream))
    return _check(code, "mlg_build_csr_batch", check)


def mlg_local_attention(csr: Csr, n_centres: int, nnei_max: int, channels: int, heads: int,
                        dtype: int, H_in, G_in, out, Wq, Wk, Wv, stream=None,
                        check: bool = True) -> int:
    """Launch local attention (one query per centre from ``H_in``; keys and
    values from the centre's edges in ``G_in``) on ``stream``."""
    c = csr.struct()
    code = _lib.mlg_local_attention(ctypes.byref(c), int(n_centres), int(nnei_max),
                                    int(channels), int(heads), int(dtype), _ptr(H_in),
                                    _ptr(G_in), _ptr(out), _ptr(Wq), _ptr(Wk), _ptr(Wv),
                                    _stream_handle(stream))
    return _check(code, "mlg_local_attention", check)


def mlg_forward(system: mlg_system, rcut: float, r_on: float, nnei_max: int, channels: int,
                heads: int, n_layers: int, dtype: int, W, G0, G_out, csr: Csr, ws,
                ws_bytes: int | None = None, stream=None, check: bool = True) -> int:
    """Launch build + ``n_layers`` attention layers. ``W``: 3 * n_layers device tensors."""
    ptrs = (_p * len(W))(*[_ptr(w) for w in W])
    c = csr.struct()
    nbytes = int(ws.numel() * ws.element_size()) if ws_bytes is None else int(ws_bytes)
    code = _lib.mlg_forward(ctypes.byref(system), float(rcut), float(r_on), int(nnei_max),
                            int(channels), int(heads), int(n_layers), int(dtype), ptrs,
                            _ptr(G0), _ptr(G_out), ctypes.byref(c), _ptr(ws), nbytes,
                            _stream_handle(stream))
    return _check(code, "mlg_forward", check)


def workspace(nbytes: int, device="cuda"):
    """A 256-byte aligned device workspace tensor of at least ``nbytes``."""
    import torch
    t = torch.empty(max(int(nbytes), 1) + 256, dtype=torch.uint8, device=device)
    off = (-t.data_ptr()) % 256
    return t[off: off + max(int(nbytes), 1)]
