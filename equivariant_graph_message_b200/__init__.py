"""Equivariant message-passing convolution for NVIDIA B200 (sm_100a).

Thin ctypes binding of libe3conv.so (C ABI in include/e3conv.h).  This
module only marshals arguments: every step of the convolution, the CSR
indexing and the row gather run in the library's CUDA kernels.  PyTorch is
used for device memory and streams only.  There is no CPU fallback: if the
library is missing, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libe3conv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -c 'import __graft_entry__ as g; g.build()'` "
                      "or `python -m equivariant_graph_message_b200._build`")

_lib = ctypes.CDLL(LIB_PATH)

F32, F16 = 0, 1
NORM = {"SQRT_DIM_OUT": 0, "NONE": 1}
ERR_BAD_INDEX = 8

_c_int_p = ctypes.POINTER(ctypes.c_int)
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64


def _sig(name, restype, *argtypes):
    fn = getattr(_lib, name)
    fn.restype = restype
    fn.argtypes = list(argtypes)
    return fn


_create = _sig("e3conv_create", ctypes.c_int, ctypes.POINTER(_vp), ctypes.c_char_p,
               ctypes.c_char_p, ctypes.c_char_p, ctypes.c_double, ctypes.c_int)
_destroy = _sig("e3conv_destroy", None, _vp)
_set_dtype = _sig("e3conv_set_input_dtype", ctypes.c_int, _vp, ctypes.c_int)
_set_launch = _sig("e3conv_set_launch_config", ctypes.c_int, _vp, ctypes.c_int, ctypes.c_int,
                   ctypes.c_int)
_query = _sig("e3conv_query", ctypes.c_int, _vp, *([_c_int_p] * 5))
_path = _sig("e3conv_path", ctypes.c_int, _vp, ctypes.c_int, *([_c_int_p] * 7))
_num_outputs = _sig("e3conv_num_outputs", ctypes.c_int, _vp, _c_int_p)
_output_irrep = _sig("e3conv_output_irrep", ctypes.c_int, _vp, ctypes.c_int, *([_c_int_p] * 3))
_cg = _sig("e3conv_cg", ctypes.c_int, _vp, ctypes.c_int, ctypes.POINTER(ctypes.c_double))
_kernel_info = _sig("e3conv_kernel_info", ctypes.c_int, _vp, ctypes.c_int, *([_c_int_p] * 8))
_set_option = _sig("e3conv_set_option", ctypes.c_int, _vp, ctypes.c_int, ctypes.c_int)
OPT_CONTRACT_FIRST = 1
OPT_TENSOR_CORES = 2
OPT_PATH_SPLIT = 3
OPT_EDGE_VECTORS = 4
OPT_A_LAYOUT = 5
OPT_COPY_GROUP = 6
OPT_DIRECT_PIPELINE = 7
OPT_BACKWARD_PARTS = 8
_get_option = _sig("e3conv_get_option", ctypes.c_int, _vp, ctypes.c_int, _c_int_p)
_sh_host = _sig("e3conv_spherical_harmonics", ctypes.c_int, _vp, ctypes.POINTER(ctypes.c_double),
                ctypes.POINTER(ctypes.c_double))
_kernel_log = _sig("e3conv_kernel_log", ctypes.c_int, _vp, ctypes.c_int, ctypes.c_char_p,
                   ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t))
_edge_sh = _sig("e3conv_edge_harmonics", ctypes.c_int, _vp, _vp, _i64, _vp, _vp)
_kernel_source = _sig("e3conv_kernel_source", ctypes.c_int, _vp, ctypes.c_int, ctypes.c_char_p,
                      ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t))
_forward = _sig("e3conv_forward", ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp)
_forward_rows = _sig("e3conv_forward_rows", ctypes.c_int, _vp, _vp, _i64, _vp, _vp, _vp, _vp,
                     _i64, _i64, _vp, _vp)
_check = _sig("e3conv_check", ctypes.c_int, _vp, _vp)
_backward = _sig("e3conv_backward", ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                 _i64, _vp, _vp, _vp, _vp, _vp)
_prepare_backward = _sig("e3conv_prepare_backward", ctypes.c_int, _vp)
_backward_source = _sig("e3conv_backward_source", ctypes.c_int, _vp, ctypes.c_int, ctypes.c_char_p,
                        ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t))
_partition = _sig("e3conv_partition_rows", ctypes.c_int, _vp, _i64, ctypes.c_int, _vp)
_set_radial = _sig("e3conv_set_radial_mlp", ctypes.c_int, _vp, ctypes.c_int, ctypes.c_double,
                   ctypes.c_int, ctypes.c_int, _vp, _vp, _vp)
_radial_scalars = _sig("e3conv_radial_scalars", ctypes.c_int, _vp, _vp, _i64, _vp, _vp)
_lin_create = _sig("e3conv_linear_create", ctypes.c_int, ctypes.POINTER(_vp), ctypes.c_char_p,
                   ctypes.c_char_p, ctypes.c_double)
_lin_destroy = _sig("e3conv_linear_destroy", None, _vp)
_lin_query = _sig("e3conv_linear_query", ctypes.c_int, _vp, *([_c_int_p] * 5))
_lin_set = _sig("e3conv_linear_set_weights", ctypes.c_int, _vp, _vp)
_lin_forward = _sig("e3conv_linear_forward", ctypes.c_int, _vp, _vp, _i64, _vp, _vp)
_lin_check = _sig("e3conv_linear_check", ctypes.c_int, _vp, _vp)
_lin_uses_tma = _sig("e3conv_linear_uses_tma", ctypes.c_int, _vp, _c_int_p)
_lin_set_tma = _sig("e3conv_linear_set_tma", ctypes.c_int, _vp, ctypes.c_int)
_csr_ws = _sig("e3conv_csr_workspace_size", ctypes.c_int, _i64, _i64,
               ctypes.POINTER(ctypes.c_size_t))
_build_csr = _sig("e3conv_build_csr", ctypes.c_int, _vp, _i64, _i64, _vp, _vp, _vp,
                  ctypes.c_size_t, _vp)
_csr_check = _sig("e3conv_csr_check", ctypes.c_int, _vp, _vp)
_csr_count = _sig("e3conv_csr_kernel_count", ctypes.c_int, _i64, _i64, _c_int_p)
_build_csr_noalloc = _sig("e3conv_build_csr_noalloc", ctypes.c_int, _vp, _i64, _i64, _vp, _vp, _vp)
_permute = _sig("e3conv_permute_rows", ctypes.c_int, _vp, _i64, _vp, _i64, _i64, _vp, _vp, _vp)
_strerror = _sig("e3conv_strerror", ctypes.c_char_p, ctypes.c_int)
_last_error = _sig("e3conv_last_error", ctypes.c_char_p)
_version = _sig("e3conv_version", ctypes.c_int)

EXPORTED = ["e3conv_create", "e3conv_destroy", "e3conv_set_input_dtype",
            "e3conv_set_launch_config", "e3conv_set_option", "e3conv_get_option",
            "e3conv_spherical_harmonics", "e3conv_edge_harmonics", "e3conv_query", "e3conv_path", "e3conv_num_outputs",
            "e3conv_output_irrep", "e3conv_cg", "e3conv_kernel_info", "e3conv_kernel_source", "e3conv_kernel_log",
            "e3conv_forward", "e3conv_forward_rows", "e3conv_check", "e3conv_partition_rows",
            "e3conv_backward", "e3conv_prepare_backward", "e3conv_backward_source",
            "e3conv_set_radial_mlp", "e3conv_radial_scalars", "e3conv_linear_create",
            "e3conv_linear_destroy", "e3conv_linear_query", "e3conv_linear_set_weights",
            "e3conv_linear_forward", "e3conv_linear_check", "e3conv_linear_uses_tma",
            "e3conv_linear_set_tma", "e3conv_csr_workspace_size", "e3conv_build_csr",
            "e3conv_csr_check", "e3conv_build_csr_noalloc", "e3conv_csr_kernel_count", "e3conv_permute_rows", "e3conv_strerror", "e3conv_last_error",
            "e3conv_version"]


class E3ConvError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = _last_error().decode(errors="replace")
        super().__init__(f"{where}: {_strerror(code).decode()} ({code}): {msg}")


def _ok(code: int, where: str):
    if code != 0:
        raise E3ConvError(code, where)


def version() -> int:
    return _version()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _require(name, t, device=None, dtype=None, numel=None):
    """Checks a tensor handed to the library: a contiguous CUDA tensor (on `device`), of
    `dtype` and with at least `numel` elements.  Host tensors never reach a kernel."""
    if not getattr(t, "is_cuda", False):
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} has {t.numel()} elements, needs {numel}")


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


@dataclass(frozen=True)
class PathInfo:
    l1: int
    p1: int
    l2: int
    l3: int
    p3: int
    x_off: int
    out_off: int


class Conv:
    """One plan of the convolution (e3conv_create / e3conv_forward)."""

    def __init__(self, irreps_node: str, irreps_sh: str, irreps_out: str,
                 avg_num_neighbors: float, normalization: str = "SQRT_DIM_OUT",
                 dtype: str = "f32"):
        h = _vp()
        _ok(_create(ctypes.byref(h), irreps_node.encode(), irreps_sh.encode(),
                    irreps_out.encode(), float(avg_num_neighbors), NORM[normalization]),
            "e3conv_create")
        self._h = h
        vals = [ctypes.c_int() for _ in range(5)]
        _ok(_query(h, *[ctypes.byref(v) for v in vals]), "e3conv_query")
        self.C, self.nx, self.ny, self.nout, self.num_paths = (v.value for v in vals)
        self.dtype = "f32"
        if dtype != "f32":
            self.set_dtype(dtype)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and _destroy is not None:   # (module globals may be gone at interpreter exit)
            _destroy(h)
            self._h = None

    def close(self):
        self.__del__()

    # ---- plan inspection
    @property
    def paths(self) -> list[PathInfo]:
        out = []
        for p in range(self.num_paths):
            v = [ctypes.c_int() for _ in range(7)]
            _ok(_path(self._h, p, *[ctypes.byref(x) for x in v]), "e3conv_path")
            out.append(PathInfo(*(x.value for x in v)))
        return out

    @property
    def outputs(self) -> list[tuple[int, int, int]]:
        n = ctypes.c_int()
        _ok(_num_outputs(self._h, ctypes.byref(n)), "e3conv_num_outputs")
        res = []
        for k in range(n.value):
            v = [ctypes.c_int() for _ in range(3)]
            _ok(_output_irrep(self._h, k, *[ctypes.byref(x) for x in v]), "e3conv_output_irrep")
            res.append(tuple(x.value for x in v))
        return res

    def cg(self, p: int) -> np.ndarray:
        q = self.paths[p]
        shape = (2 * q.l1 + 1, 2 * q.l2 + 1, 2 * q.l3 + 1)
        buf = np.zeros(int(np.prod(shape)), dtype=np.float64)
        _ok(_cg(self._h, p, buf.ctypes.data_as(ctypes.POINTER(ctypes.c_double))), "e3conv_cg")
        return buf.reshape(shape)

    def set_dtype(self, dtype: str):
        _ok(_set_dtype(self._h, {"f32": F32, "f16": F16}[dtype]), "e3conv_set_input_dtype")
        self.dtype = dtype

    def set_launch_config(self, channels_per_lane: int = 0, block_threads: int = 0,
                          stages: int = -1):
        _ok(_set_launch(self._h, channels_per_lane, block_threads, stages),
            "e3conv_set_launch_config")

    def set_contract_first(self, value: int = -1):
        _ok(_set_option(self._h, OPT_CONTRACT_FIRST, value), "e3conv_set_option")

    def set_tensor_cores(self, value: int = -1):
        _ok(_set_option(self._h, OPT_TENSOR_CORES, value), "e3conv_set_option")

    def set_path_split(self, value: int = -1):
        _ok(_set_option(self._h, OPT_PATH_SPLIT, value), "e3conv_set_option")

    def set_direct_pipeline(self, value: int = -1):
        _ok(_set_option(self._h, OPT_DIRECT_PIPELINE, value), "e3conv_set_option")

    def set_backward_parts(self, value: int = -1):
        """Launches of each staged backward kernel (-1 automatic, 1 .. 4)."""
        _ok(_set_option(self._h, OPT_BACKWARD_PARTS, value), "e3conv_set_option")

    def set_copy_group(self, value: int = -1):
        _ok(_set_option(self._h, OPT_COPY_GROUP, value), "e3conv_set_option")

    def set_a_layout(self, value: int = -1):
        _ok(_set_option(self._h, OPT_A_LAYOUT, value), "e3conv_set_option")

    def set_edge_vectors(self, value: int = 1):
        """1: the forward's Y argument holds edge vectors float32 [E][4]; harmonics in-kernel."""
        _ok(_set_option(self._h, OPT_EDGE_VECTORS, value), "e3conv_set_option")

    @property
    def edge_vectors(self) -> bool:
        v = ctypes.c_int()
        _ok(_get_option(self._h, OPT_EDGE_VECTORS, ctypes.byref(v)), "e3conv_get_option")
        return v.value == 1

    def spherical_harmonics(self, vec) -> np.ndarray:
        """The plan's harmonics of vec / |vec| (host evaluation of the kernel's polynomials)."""
        v = np.ascontiguousarray(np.asarray(vec, dtype=np.float64).reshape(3))
        out = np.zeros(self.ny)
        _ok(_sh_host(self._h, v.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                     out.ctypes.data_as(ctypes.POINTER(ctypes.c_double))),
            "e3conv_spherical_harmonics")
        return out

    def edge_harmonics(self, edge_vectors, out=None, stream=None):
        """Y [E][ny] (plan dtype) from edge vectors float32 [E][4] on the device."""
        import torch
        _require("edge_vectors", edge_vectors, dtype=torch.float32)
        E = edge_vectors.shape[0]
        if tuple(edge_vectors.shape) != (E, 4):
            raise ValueError("edge_vectors must be [E][4]")
        want = torch.float16 if self.dtype == "f16" else torch.float32
        if out is None:
            out = torch.empty((E, self.ny), dtype=want, device=edge_vectors.device)
        else:
            _require("out", out, edge_vectors.device, want, E * self.ny)
        _ok(_edge_sh(self._h, _ptr(edge_vectors) if E else None, E, _ptr(out) if E else None,
                     _stream_handle(stream)), "e3conv_edge_harmonics")
        return out

    def kernel_info(self, dtype: str | None = None) -> dict:
        v = [ctypes.c_int() for _ in range(8)]
        _ok(_kernel_info(self._h, {"f32": F32, "f16": F16}[dtype or self.dtype],
                         *[ctypes.byref(x) for x in v]), "e3conv_kernel_info")
        keys = ["channels_per_lane", "lanes_per_tile", "block_threads", "stages", "contract_first",
                "tensor_cores", "registers", "local_bytes"]
        return dict(zip(keys, (x.value for x in v)))

    def kernel_log(self, dtype: str | None = None) -> str:
        """The launch-shape search's compile attempts and the kept compile's NVRTC log."""
        d = {"f32": F32, "f16": F16}[dtype or self.dtype]
        n = ctypes.c_size_t()
        _ok(_kernel_log(self._h, d, None, 0, ctypes.byref(n)), "e3conv_kernel_log")
        buf = ctypes.create_string_buffer(n.value)
        _ok(_kernel_log(self._h, d, buf, n.value, ctypes.byref(n)), "e3conv_kernel_log")
        return buf.value.decode()

    def kernel_source(self, dtype: str | None = None) -> str:
        d = {"f32": F32, "f16": F16}[dtype or self.dtype]
        n = ctypes.c_size_t()
        _ok(_kernel_source(self._h, d, None, 0, ctypes.byref(n)), "e3conv_kernel_source")
        buf = ctypes.create_string_buffer(n.value)
        _ok(_kernel_source(self._h, d, buf, n.value, ctypes.byref(n)), "e3conv_kernel_source")
        return buf.value.decode()

    # ---- device calls
    def _check_inputs(self, x, Y, s, senders, row_ptr):
        import torch
        N = x.shape[0]
        E = senders.shape[0]
        want = torch.float16 if self.dtype == "f16" else torch.float32
        _require("x", x, dtype=want)
        dev = x.device
        vec = self.edge_vectors
        _require("Y", Y, dev, torch.float32 if vec else want)
        _require("s", s, dev, want)
        _require("senders", senders, dev, torch.int32)
        _require("row_ptr", row_ptr, dev, torch.int32)
        if tuple(x.shape) != (N, self.nx, self.C):
            raise ValueError(f"x shape {tuple(x.shape)} != {(N, self.nx, self.C)}")
        if tuple(Y.shape) != ((E, 4) if vec else (E, self.ny)):
            raise ValueError("Y shape does not match the plan (edge vectors: [E][4])")
        if tuple(s.shape) != (E, self.num_paths, self.C):
            raise ValueError("s shape does not match the plan")

    def forward(self, x, Y, s, senders, row_ptr, out=None, stream=None):
        """out[N][nout][C] float32 from receiver-sorted edges (torch CUDA tensors)."""
        import torch
        N = x.shape[0]
        E = senders.shape[0]
        dev = x.device
        self._check_inputs(x, Y, s, senders, row_ptr)
        if row_ptr.shape[0] != N + 1:
            raise ValueError("row_ptr must have num_nodes + 1 entries")
        if out is None:
            out = torch.empty((N, self.nout, self.C), dtype=torch.float32, device=dev)
        else:
            _require("out", out, dev, torch.float32, N * self.nout * self.C)
        _ok(_forward(self._h, _ptr(x), _ptr(Y) if E else None, _ptr(s) if E else None,
                     _ptr(senders) if E else None, _ptr(row_ptr), N, _ptr(out),
                     _stream_handle(stream)), "e3conv_forward")
        return out

    def forward_rows(self, x, Y, s, senders, row_ptr, row_begin: int, row_end: int, out=None,
                     stream=None):
        """out[row_end-row_begin][nout][C] for the receiver rows [row_begin, row_end) of
        row_ptr; Y, s and senders hold those rows' edges only, and x is the table the
        senders index (any number of rows)."""
        import torch
        N = x.shape[0]
        E = senders.shape[0]
        dev = x.device
        self._check_inputs(x, Y, s, senders, row_ptr)
        if not 0 <= row_begin <= row_end < row_ptr.shape[0]:
            raise ValueError("rows must satisfy 0 <= row_begin <= row_end < len(row_ptr)")
        rows = row_end - row_begin
        if out is None:
            out = torch.empty((rows, self.nout, self.C), dtype=torch.float32, device=dev)
        else:
            _require("out", out, dev, torch.float32, rows * self.nout * self.C)
        _ok(_forward_rows(self._h, _ptr(x), N, _ptr(Y) if E else None, _ptr(s) if E else None,
                          _ptr(senders) if E else None, _ptr(row_ptr), row_begin, row_end,
                          _ptr(out), _stream_handle(stream)), "e3conv_forward_rows")
        return out

    def set_radial_mlp(self, r_max: float, weights):
        """Radial MLP from float32 weights [W_0 (num_basis x hidden), W_1 .. W_{L-1}
        (hidden x hidden), W_L (hidden x P*C)] (host arrays, input index first)."""
        ws = [np.ascontiguousarray(np.asarray(w, dtype=np.float32)) for w in weights]
        nb, hidden = ws[0].shape
        layers = len(ws) - 1
        hid = np.ascontiguousarray(np.stack(ws[1:-1])) if layers > 1 else None
        _ok(_set_radial(self._h, nb, float(r_max), hidden, layers, ws[0].ctypes.data_as(_vp),
                        hid.ctypes.data_as(_vp) if hid is not None else None,
                        ws[-1].ctypes.data_as(_vp)), "e3conv_set_radial_mlp")
        self._radial = (r_max, ws)

    def radial_scalars(self, edge_vectors, out=None, stream=None):
        """s [E][P][C] (plan dtype) from edge vectors float32 [E][4] on the device."""
        import torch
        _require("edge_vectors", edge_vectors, dtype=torch.float32)
        E = edge_vectors.shape[0]
        if tuple(edge_vectors.shape) != (E, 4):
            raise ValueError("edge_vectors must be [E][4]")
        want = torch.float16 if self.dtype == "f16" else torch.float32
        if out is None:
            out = torch.empty((E, self.num_paths, self.C), dtype=want, device=edge_vectors.device)
        else:
            _require("out", out, edge_vectors.device, want, E * self.num_paths * self.C)
        _ok(_radial_scalars(self._h, _ptr(edge_vectors) if E else None, E,
                            _ptr(out) if E else None, _stream_handle(stream)),
            "e3conv_radial_scalars")
        return out

    def backward(self, x, Y, s, senders, row_ptr, grad_out, receivers=None, sender_row_ptr=None,
                 sender_perm=None, need_x=True, need_edges=True, stream=None):
        """(grad_x, grad_sh, grad_scalars) of sum(grad_out * forward(...)); grad_x needs the
        edges' receivers and the sender CSR (e3conv_build_csr of `senders`)."""
        import torch
        N = x.shape[0]
        E = senders.shape[0]
        dev = x.device
        self._check_inputs(x, Y, s, senders, row_ptr)
        _require("grad_out", grad_out, dev, torch.float32, N * self.nout * self.C)
        gx = gY = gs = None
        if need_x:
            for name, tt in (("receivers", receivers), ("sender_row_ptr", sender_row_ptr),
                             ("sender_perm", sender_perm)):
                if tt is None:
                    raise ValueError(f"{name} is needed for grad_x")
                _require(name, tt, dev, torch.int32)
            gx = torch.empty((N, self.nx, self.C), dtype=torch.float32, device=dev)
        if need_edges:
            gY = torch.empty((E, self.ny), dtype=torch.float32, device=dev)
            gs = torch.empty((E, self.num_paths, self.C), dtype=torch.float32, device=dev)
        ne = E > 0
        _ok(_backward(self._h, _ptr(x), _ptr(Y) if ne else None, _ptr(s) if ne else None,
                      _ptr(senders) if ne else None, _ptr(receivers) if ne and need_x else None,
                      _ptr(row_ptr), _ptr(sender_row_ptr) if need_x else None,
                      _ptr(sender_perm) if ne and need_x else None, N, _ptr(grad_out),
                      _ptr(gx), _ptr(gY) if ne and need_edges else None,
                      _ptr(gs) if ne and need_edges else None, _stream_handle(stream)),
            "e3conv_backward")
        return gx, gY, gs

    def backward_source(self, which: int) -> str:
        n = ctypes.c_size_t()
        _ok(_backward_source(self._h, which, None, 0, ctypes.byref(n)), "e3conv_backward_source")
        buf = ctypes.create_string_buffer(n.value)
        _ok(_backward_source(self._h, which, buf, n.value, ctypes.byref(n)), "e3conv_backward_source")
        return buf.value.decode()

    def forward_raw(self, x_ptr, Y_ptr, s_ptr, senders_ptr, row_ptr_ptr, num_nodes, out_ptr,
                    stream_handle):
        """Pointer-level call of e3conv_forward (for timing loops)."""
        _ok(_forward(self._h, x_ptr, Y_ptr, s_ptr, senders_ptr, row_ptr_ptr, num_nodes, out_ptr,
                     stream_handle), "e3conv_forward")

    def forward_rows_raw(self, x_ptr, num_nodes, Y_ptr, s_ptr, senders_ptr, row_ptr_ptr,
                         row_begin, row_end, out_ptr, stream_handle):
        """Pointer-level call of e3conv_forward_rows (for timing loops)."""
        _ok(_forward_rows(self._h, x_ptr, num_nodes, Y_ptr, s_ptr, senders_ptr, row_ptr_ptr,
                          row_begin, row_end, out_ptr, stream_handle), "e3conv_forward_rows")

    def check(self, stream=None) -> bool:
        """True if no forward since the last check met a bad index."""
        rc = _check(self._h, _stream_handle(stream))
        if rc == ERR_BAD_INDEX:
            return False
        _ok(rc, "e3conv_check")
        return True


class IrrepsLinear:
    """Channel mixing within matching irreps on the tensor cores (e3conv_linear_*), on the
    convolution's feature layout."""

    def __init__(self, irreps_in: str, irreps_out: str, scale: float = 1.0):
        h = _vp()
        _ok(_lin_create(ctypes.byref(h), irreps_in.encode(), irreps_out.encode(), float(scale)),
            "e3conv_linear_create")
        self._h = h
        v = [ctypes.c_int() for _ in range(5)]
        _ok(_lin_query(h, *[ctypes.byref(q) for q in v]), "e3conv_linear_query")
        self.dim_in, self.dim_out, self.num_weight_blocks, self.mul_in, self.mul_out = \
            (q.value for q in v)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and _lin_destroy is not None:
            _lin_destroy(h)
            self._h = None

    @property
    def uses_tma(self) -> bool:
        """True when the forward runs the tensor-map kernel (else the row-per-thread one)."""
        t = ctypes.c_int()
        _ok(_lin_uses_tma(self._h, ctypes.byref(t)), "e3conv_linear_uses_tma")
        return bool(t.value)

    def set_tma(self, enable: bool):
        """False: always the row-per-thread kernel; True (default): the tensor-map kernel
        where the shape allows it."""
        _ok(_lin_set_tma(self._h, int(bool(enable))), "e3conv_linear_set_tma")

    def set_weights(self, weights):
        """weights: num_weight_blocks arrays [mul_in][mul_out] (host), matched irreps in
        output order."""
        w = np.ascontiguousarray(np.stack([np.asarray(q, dtype=np.float32) for q in weights])) \
            if len(weights) else np.zeros(1, np.float32)
        if len(weights) != self.num_weight_blocks:
            raise ValueError(f"{self.num_weight_blocks} weight blocks expected")
        _ok(_lin_set(self._h, w.ctypes.data_as(_vp)), "e3conv_linear_set_weights")

    def __call__(self, x, out=None, stream=None):
        import torch
        _require("x", x, dtype=torch.float32)
        N = x.shape[0]
        if x.numel() != N * self.dim_in:
            raise ValueError(f"x must hold {self.dim_in} floats per node")
        if out is None:
            out = torch.empty((N, self.dim_out), dtype=torch.float32, device=x.device)
        else:
            _require("out", out, x.device, torch.float32, N * self.dim_out)
        _ok(_lin_forward(self._h, _ptr(x), N, _ptr(out), _stream_handle(stream)),
            "e3conv_linear_forward")
        return out

    def check(self, stream=None) -> bool:
        _ok(_lin_check(self._h, _stream_handle(stream)), "e3conv_linear_check")
        return True


def partition_rows(row_ptr, parts: int) -> np.ndarray:
    """int64 [parts+1] boundaries of `parts` contiguous receiver-row ranges balanced on
    edges + rows (e3conv_partition_rows; row_ptr is a host array of num_nodes + 1)."""
    rp = np.ascontiguousarray(np.asarray(row_ptr), dtype=np.int32)
    bounds = np.zeros(parts + 1, dtype=np.int64)
    _ok(_partition(rp.ctypes.data_as(_vp), len(rp) - 1, parts, bounds.ctypes.data_as(_vp)),
        "e3conv_partition_rows")
    return bounds


def csr_workspace_size(num_edges: int, num_nodes: int) -> int:
    n = ctypes.c_size_t()
    _ok(_csr_ws(num_edges, num_nodes, ctypes.byref(n)), "e3conv_csr_workspace_size")
    return n.value


def build_csr(receivers, num_nodes: int, row_ptr=None, perm=None, workspace=None, stream=None):
    """(row_ptr int32 [N+1], perm int32 [E]) of int32 device `receivers`."""
    import torch
    E = receivers.shape[0]
    _require("receivers", receivers, dtype=torch.int32)
    dev = receivers.device
    if row_ptr is None:
        row_ptr = torch.empty(num_nodes + 1, dtype=torch.int32, device=dev)
    _require("row_ptr", row_ptr, dev, torch.int32, num_nodes + 1)
    if perm is None:
        perm = torch.empty(max(E, 1), dtype=torch.int32, device=dev)[:E]
    _require("perm", perm, dev, torch.int32, E)
    nbytes = csr_workspace_size(E, num_nodes)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _require("workspace", workspace, dev, torch.uint8)
    _ok(_build_csr(_ptr(receivers) if E else None, E, num_nodes, _ptr(row_ptr),
                   _ptr(perm) if E else None, _ptr(workspace), workspace.numel(),
                   _stream_handle(stream)), "e3conv_build_csr")
    return row_ptr, perm, workspace


def build_csr_noalloc(receivers, num_nodes: int, row_ptr=None, perm=None, stream=None):
    """e3conv_build_csr_noalloc: the CSR build with the library's fixed scratch
    (for callers that cannot allocate device memory; outputs may be passed in)."""
    import torch
    E = receivers.shape[0]
    _require("receivers", receivers, dtype=torch.int32)
    if row_ptr is None:
        row_ptr = torch.empty(num_nodes + 1, dtype=torch.int32, device=receivers.device)
    _require("row_ptr", row_ptr, receivers.device, torch.int32, num_nodes + 1)
    if perm is None:
        perm = torch.empty(max(E, 1), dtype=torch.int32, device=receivers.device)[:E]
    _require("perm", perm, receivers.device, torch.int32, E)
    _ok(_build_csr_noalloc(_ptr(receivers) if E else None, E, num_nodes, _ptr(row_ptr),
                           _ptr(perm) if E else None, _stream_handle(stream)),
        "e3conv_build_csr_noalloc")
    return row_ptr, perm


def csr_kernel_count(num_edges: int, num_nodes: int) -> int:
    n = ctypes.c_int()
    _ok(_csr_count(num_edges, num_nodes, ctypes.byref(n)), "e3conv_csr_kernel_count")
    return n.value


def csr_check(workspace, stream=None) -> bool:
    _require("workspace", workspace)
    rc = _csr_check(_ptr(workspace), _stream_handle(stream))
    if rc == ERR_BAD_INDEX:
        return False
    _ok(rc, "e3conv_csr_check")
    return True


def permute_rows(src, perm, dst=None, status=None, stream=None):
    """dst[t] = src[perm[t]] along the first axis (device)."""
    import torch
    rows = perm.shape[0]
    _require("src", src)
    _require("perm", perm, src.device, torch.int32)
    row_bytes = src[0].numel() * src.element_size() if src.shape[0] else 0
    if dst is None:
        dst = torch.empty((rows,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    _require("dst", dst, src.device, src.dtype, rows * (src[0].numel() if src.shape[0] else 0))
    if status is not None:
        _require("status", status, src.device, torch.int32, 1)
    _ok(_permute(_ptr(src), src.shape[0], _ptr(perm), rows, row_bytes, _ptr(dst), _ptr(status),
                 _stream_handle(stream)), "e3conv_permute_rows")
    return dst
