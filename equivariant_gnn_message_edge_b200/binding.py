"""Thin ctypes binding of libeqconv: same names as the C ABI (include/eqconv.h),
argument marshalling only.  Every computation runs in the library's CUDA
kernels; there is no fallback of any kind: if libeqconv.so is missing or fails
to load, every call raises.

Tensor arguments are CUDA torch tensors (contiguous, right dtype) or raw device
pointers (ints).  ``stream=None`` means torch's current stream on the current
device.
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np

LIB_PATH = os.environ.get("EQCONV_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                             "libeqconv.so")

EQCONV_OK = 0
EQCONV_ERR_INVALID_ARG = 1
EQCONV_ERR_UNSUPPORTED = 2
EQCONV_ERR_CUDA = 3
EQCONV_ERR_WORKSPACE = 4
EQCONV_ERR_DEVICE_CHECK = 5
EQCONV_DETERMINISTIC = 1
EQCONV_OUT_ALL_PARITY = 1
EQCONV_OUT_PER_PATH = 2

ABI_FUNCTIONS = (
    "eqconv_plan_create", "eqconv_plan_set_vec", "eqconv_plan_info", "eqconv_enumerate_paths", "eqconv_cg_table",
    "eqconv_graph_workspace_bytes", "eqconv_graph_build", "eqconv_forward",
    "eqconv_backward_workspace_bytes", "eqconv_backward", "eqconv_spherical_harmonics",
    "eqconv_get_device_error", "eqconv_plan_destroy", "eqconv_status_string", "eqconv_launch_count",
    "eqconv_last_error", "eqconv_graph_build_noalloc", "eqconv_plan_set_gather_budget",
    "eqconv_plan_create_ex", "eqconv_plan_path_rows", "eqconv_enumerate_paths_ex",
    "eqconv_double_backward_workspace_bytes", "eqconv_double_backward",
    "eqconv_node_product_plan_create", "eqconv_node_product", "eqconv_node_product_workspace_bytes",
    "eqconv_node_product_backward", "eqconv_radial_workspace_bytes", "eqconv_radial_weights",
    "eqconv_forward_radial_workspace_bytes", "eqconv_forward_radial",
    "eqconv_backward_radial_workspace_bytes", "eqconv_backward_radial",
    "eqconv_symmetric_contraction_plan_create", "eqconv_symmetric_contraction",
    "eqconv_symmetric_contraction_workspace_bytes", "eqconv_symmetric_contraction_backward",
)


class EqconvError(RuntimeError):
    def __init__(self, what: str, status: int):
        msg = f"{what}: {eqconv_status_string(status)} (status {status})"
        if status == EQCONV_ERR_CUDA:
            msg += f" [{eqconv_last_error()}]"
        super().__init__(msg)
        self.status = status


class eqconv_graph_t(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("E", ctypes.c_int32),
                ("senders", ctypes.c_void_p), ("receivers", ctypes.c_void_p),
                ("recv_ptr", ctypes.c_void_p), ("recv_perm", ctypes.c_void_p),
                ("send_ptr", ctypes.c_void_p), ("send_perm", ctypes.c_void_p)]


_lib = None
_lock = threading.Lock()
_vp, _ci, _cu, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t
_pi = ctypes.POINTER(ctypes.c_int)
_pd = ctypes.POINTER(ctypes.c_double)
_pg = ctypes.POINTER(eqconv_graph_t)

_SIGS = {
    "eqconv_plan_create": (_ci, [ctypes.POINTER(_vp), ctypes.c_char_p, _ci, ctypes.c_char_p, _ci]),
    "eqconv_plan_create_ex": (_ci, [ctypes.POINTER(_vp), ctypes.c_char_p, _ci, ctypes.c_char_p, _ci, _cu]),
    "eqconv_plan_path_rows": (_ci, [_vp, _pi]),
    "eqconv_enumerate_paths_ex": (_ci, [ctypes.c_char_p, _ci, ctypes.c_char_p, _cu, _pi, _pi, _pi, _pi, _ci]),
    "eqconv_plan_set_vec": (_ci, [_vp, _ci, _ci]),
    "eqconv_plan_set_gather_budget": (_ci, [_vp, _sz]),
    "eqconv_plan_info": (_ci, [_vp, _pi, _pi, _pi, _pi, _pi]),
    "eqconv_enumerate_paths": (_ci, [ctypes.c_char_p, _ci, ctypes.c_char_p, _pi, _pi, _ci]),
    "eqconv_cg_table": (_ci, [_ci, _ci, _ci, _pd, _ci]),
    "eqconv_graph_workspace_bytes": (_sz, [_ci, _ci]),
    "eqconv_graph_build": (_ci, [_vp, _pg, _vp, _sz, _vp]),
    "eqconv_graph_build_noalloc": (_ci, [_vp, _pg, _vp]),
    "eqconv_forward": (_ci, [_vp, _pg, _vp, _vp, _vp, _vp, _cu, _vp]),
    "eqconv_backward_workspace_bytes": (_sz, [_vp, _ci]),
    "eqconv_backward": (_ci, [_vp, _pg, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _cu, _vp]),
    "eqconv_double_backward_workspace_bytes": (_sz, [_vp, _ci]),
    "eqconv_double_backward": (_ci, [_vp, _pg] + [_vp] * 12 + [_sz, _vp]),
    "eqconv_node_product_plan_create": (_ci, [ctypes.POINTER(_vp), ctypes.c_char_p, _ci, ctypes.c_char_p, _ci,
                                                _cu]),
    "eqconv_node_product": (_ci, [_vp, _ci, _vp, _vp, _vp, _vp, _vp]),
    "eqconv_node_product_workspace_bytes": (_sz, [_vp, _ci]),
    "eqconv_node_product_backward": (_ci, [_vp, _ci] + [_vp] * 8 + [_sz, _vp]),
    "eqconv_spherical_harmonics": (_ci, [_vp, _ci, _vp, _vp, _vp]),
    "eqconv_radial_workspace_bytes": (_sz, [_vp, _ci]),
    "eqconv_forward_radial_workspace_bytes": (_sz, [_vp, _ci, _ci]),
    "eqconv_symmetric_contraction_plan_create": (_ci, [ctypes.POINTER(_vp), ctypes.c_char_p, ctypes.c_char_p, _ci,
                                                       _ci]),
    "eqconv_symmetric_contraction": (_ci, [_vp, _ci] + [_vp] * 5 + [_vp]),
    "eqconv_symmetric_contraction_workspace_bytes": (_sz, [_vp, _ci]),
    "eqconv_symmetric_contraction_backward": (_ci, [_vp, _ci] + [_vp] * 9 + [_sz, _vp]),
    "eqconv_backward_radial_workspace_bytes": (_sz, [_vp, _ci, _ci]),
    "eqconv_backward_radial": (_ci, [_vp, _pg] + [_vp] * 5 + [_ci, ctypes.c_float] + [_vp] * 7 + [_sz, _vp]),
    "eqconv_forward_radial": (_ci, [_vp, _pg] + [_vp] * 5 + [_ci, ctypes.c_float, _vp, _vp, _sz, _vp]),
    "eqconv_radial_weights": (_ci, [_vp, _ci] + [_vp] * 4 + [_ci, ctypes.c_float, _vp, _vp, _sz, _vp]),
    "eqconv_get_device_error": (_ci, [_vp, _vp, _pi]),
    "eqconv_plan_destroy": (None, [_vp]),
    "eqconv_status_string": (ctypes.c_char_p, [_ci]),
    "eqconv_launch_count": (ctypes.c_ulonglong, []),
    "eqconv_last_error": (ctypes.c_char_p, []),
}


def lib() -> ctypes.CDLL:
    """Load libeqconv.so (raises when it is absent: there is no fallback)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                                   "`python -m equivariant_gnn_message_edge_b200.build_lib`")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGS.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def _ptr(t, dtype=None) -> int:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"expected a CUDA tensor or a device pointer, got {type(t)}")
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"expected dtype {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, what: str):
    if rc != EQCONV_OK:
        raise EqconvError(what, rc)


def _f32():
    import torch
    return torch.float32


def _i32():
    import torch
    return torch.int32


# ------------------------------------------------------------------ ABI calls

def eqconv_status_string(status: int) -> str:
    return lib().eqconv_status_string(int(status)).decode()


def eqconv_last_error() -> str:
    return lib().eqconv_last_error().decode()


def eqconv_launch_count() -> int:
    return int(lib().eqconv_launch_count())


def eqconv_plan_create(irreps_in: str, L_sh: int, irreps_out: str, C: int) -> int:
    h = _vp()
    _check(lib().eqconv_plan_create(ctypes.byref(h), irreps_in.encode(), int(L_sh), irreps_out.encode(), int(C)),
           "eqconv_plan_create")
    return h.value


def eqconv_plan_create_ex(irreps_in: str, L_sh: int, irreps_out: str, C: int, out_mode: int) -> int:
    h = _vp()
    _check(lib().eqconv_plan_create_ex(ctypes.byref(h), irreps_in.encode(), int(L_sh), irreps_out.encode(), int(C),
                                       int(out_mode)), "eqconv_plan_create_ex")
    return h.value


def eqconv_plan_path_rows(plan: int) -> list:
    P = eqconv_plan_info(plan)["P"]
    buf = (ctypes.c_int * max(1, P))()
    _check(lib().eqconv_plan_path_rows(plan, buf), "eqconv_plan_path_rows")
    return list(buf[:P])


def eqconv_enumerate_paths_ex(irreps_in: str, L_sh: int, irreps_out: str, out_mode: int) -> dict:
    """{'paths': [(l1, l2, l3)], 'rows': [first output row], 'D_out': n}."""
    P, D = ctypes.c_int(), ctypes.c_int()
    args = (irreps_in.encode(), int(L_sh), irreps_out.encode(), int(out_mode))
    _check(lib().eqconv_enumerate_paths_ex(*args, ctypes.byref(P), None, None, ctypes.byref(D), 0),
           "eqconv_enumerate_paths_ex")
    paths = (ctypes.c_int * max(1, 3 * P.value))()
    rows = (ctypes.c_int * max(1, P.value))()
    _check(lib().eqconv_enumerate_paths_ex(*args, ctypes.byref(P), paths, rows, ctypes.byref(D), P.value),
           "eqconv_enumerate_paths_ex")
    return dict(paths=[tuple(paths[3 * i:3 * i + 3]) for i in range(P.value)], rows=list(rows[:P.value]),
                D_out=D.value)


def eqconv_plan_set_vec(plan: int, fwd_vec: int, bwd_vec: int) -> None:
    _check(lib().eqconv_plan_set_vec(plan, int(fwd_vec), int(bwd_vec)), "eqconv_plan_set_vec")


def eqconv_plan_set_gather_budget(plan: int, nbytes: int) -> None:
    _check(lib().eqconv_plan_set_gather_budget(plan, int(nbytes)), "eqconv_plan_set_gather_budget")


def eqconv_plan_info(plan: int) -> dict:
    P, Di, Ds, Do = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(lib().eqconv_plan_info(plan, ctypes.byref(P), ctypes.byref(Di), ctypes.byref(Ds), ctypes.byref(Do), None),
           "eqconv_plan_info")
    paths = (ctypes.c_int * (3 * P.value))()
    _check(lib().eqconv_plan_info(plan, None, None, None, None, paths), "eqconv_plan_info")
    return dict(P=P.value, D_in=Di.value, D_sh=Ds.value, D_out=Do.value,
                paths=[tuple(paths[3 * i:3 * i + 3]) for i in range(P.value)])


def eqconv_enumerate_paths(irreps_in: str, L_sh: int, irreps_out: str) -> list:
    P = ctypes.c_int()
    _check(lib().eqconv_enumerate_paths(irreps_in.encode(), int(L_sh), irreps_out.encode(), ctypes.byref(P),
                                        None, 0), "eqconv_enumerate_paths")
    buf = (ctypes.c_int * max(1, 3 * P.value))()
    _check(lib().eqconv_enumerate_paths(irreps_in.encode(), int(L_sh), irreps_out.encode(), ctypes.byref(P),
                                        buf, P.value), "eqconv_enumerate_paths")
    return [tuple(buf[3 * i:3 * i + 3]) for i in range(P.value)]


def eqconv_cg_table(l1: int, l2: int, l3: int) -> np.ndarray:
    out = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1), dtype=np.float64)
    _check(lib().eqconv_cg_table(int(l1), int(l2), int(l3), out.ctypes.data_as(_pd), out.size), "eqconv_cg_table")
    return out


def eqconv_graph_workspace_bytes(N: int, E: int) -> int:
    return int(lib().eqconv_graph_workspace_bytes(int(N), int(E)))


def eqconv_graph_build(plan: int, graph: eqconv_graph_t, workspace, workspace_bytes: int, stream=None) -> None:
    _check(lib().eqconv_graph_build(plan, ctypes.byref(graph), _ptr(workspace), int(workspace_bytes),
                                    _stream(stream)), "eqconv_graph_build")


def eqconv_graph_build_noalloc(plan: int, graph: eqconv_graph_t, stream=None) -> None:
    """eqconv_graph_build without workspace or allocation (scratch in the
    library's fixed 8 MiB device array; see include/eqconv.h)."""
    _check(lib().eqconv_graph_build_noalloc(plan, ctypes.byref(graph), _stream(stream)),
           "eqconv_graph_build_noalloc")


def eqconv_forward(plan: int, graph: eqconv_graph_t, x, r, w, y, flags: int = 0, stream=None) -> None:
    f = _f32()
    _check(lib().eqconv_forward(plan, ctypes.byref(graph), _ptr(x, f), _ptr(r, f), _ptr(w, f), _ptr(y, f),
                                int(flags), _stream(stream)), "eqconv_forward")


def eqconv_backward_workspace_bytes(plan: int, E: int) -> int:
    return int(lib().eqconv_backward_workspace_bytes(plan, int(E)))


def eqconv_backward(plan: int, graph: eqconv_graph_t, x, r, w, gy, dx, dw, dr, workspace=None,
                    workspace_bytes: int = 0, flags: int = 0, stream=None) -> None:
    f = _f32()
    _check(lib().eqconv_backward(plan, ctypes.byref(graph), _ptr(x, f), _ptr(r, f), _ptr(w, f), _ptr(gy, f),
                                 _ptr(dx, f), _ptr(dw, f), _ptr(dr, f), _ptr(workspace), int(workspace_bytes),
                                 int(flags), _stream(stream)), "eqconv_backward")


def eqconv_double_backward_workspace_bytes(plan: int, E: int) -> int:
    return int(lib().eqconv_double_backward_workspace_bytes(plan, int(E)))


def eqconv_double_backward(plan: int, graph: eqconv_graph_t, x, r, w, gy, ga, gb, gq, g_x, g_w, g_gy, g_r,
                           workspace=None, workspace_bytes: int = 0, stream=None) -> None:
    f = _f32()
    _check(lib().eqconv_double_backward(plan, ctypes.byref(graph), _ptr(x, f), _ptr(r, f), _ptr(w, f), _ptr(gy, f),
                                        _ptr(ga, f), _ptr(gb, f), _ptr(gq, f), _ptr(g_x, f), _ptr(g_w, f),
                                        _ptr(g_gy, f), _ptr(g_r, f), _ptr(workspace), int(workspace_bytes),
                                        _stream(stream)), "eqconv_double_backward")


def eqconv_node_product_plan_create(irreps_u: str, L_v: int, irreps_out: str, C: int, out_mode: int = 0) -> int:
    h = _vp()
    _check(lib().eqconv_node_product_plan_create(ctypes.byref(h), irreps_u.encode(), int(L_v), irreps_out.encode(),
                                                 int(C), int(out_mode)), "eqconv_node_product_plan_create")
    return h.value


def eqconv_node_product(plan: int, N: int, u, v, w, y, stream=None) -> None:
    f = _f32()
    _check(lib().eqconv_node_product(plan, int(N), _ptr(u, f), _ptr(v, f), _ptr(w, f), _ptr(y, f), _stream(stream)),
           "eqconv_node_product")


def eqconv_node_product_workspace_bytes(plan: int, N: int) -> int:
    return int(lib().eqconv_node_product_workspace_bytes(plan, int(N)))


def eqconv_node_product_backward(plan: int, N: int, u, v, w, gy, du, dv, dw, workspace=None,
                                 workspace_bytes: int = 0, stream=None) -> None:
    f = _f32()
    _check(lib().eqconv_node_product_backward(plan, int(N), _ptr(u, f), _ptr(v, f), _ptr(w, f), _ptr(gy, f),
                                              _ptr(du, f), _ptr(dv, f), _ptr(dw, f), _ptr(workspace),
                                              int(workspace_bytes), _stream(stream)), "eqconv_node_product_backward")


def eqconv_radial_workspace_bytes(plan: int, E: int) -> int:
    return int(lib().eqconv_radial_workspace_bytes(plan, int(E)))


def eqconv_radial_weights(plan: int, E: int, r, W1, W2, W3, n_basis: int, r_cut: float, w, workspace,
                          workspace_bytes: int, stream=None) -> None:
    f = _f32()
    _check(lib().eqconv_radial_weights(plan, int(E), _ptr(r, f), _ptr(W1, f), _ptr(W2, f), _ptr(W3, f),
                                       int(n_basis), float(r_cut), _ptr(w, f), _ptr(workspace),
                                       int(workspace_bytes), _stream(stream)), "eqconv_radial_weights")


def eqconv_forward_radial_workspace_bytes(plan: int, N: int, E: int) -> int:
    return int(lib().eqconv_forward_radial_workspace_bytes(plan, int(N), int(E)))


def eqconv_forward_radial(plan: int, graph: eqconv_graph_t, x, r, W1, W2, W3, n_basis: int, r_cut: float, y,
                          workspace, workspace_bytes: int, stream=None) -> None:
    f = _f32()
    _check(lib().eqconv_forward_radial(plan, ctypes.byref(graph), _ptr(x, f), _ptr(r, f), _ptr(W1, f), _ptr(W2, f),
                                       _ptr(W3, f), int(n_basis), float(r_cut), _ptr(y, f), _ptr(workspace),
                                       int(workspace_bytes), _stream(stream)), "eqconv_forward_radial")


def eqconv_backward_radial_workspace_bytes(plan: int, N: int, E: int) -> int:
    return int(lib().eqconv_backward_radial_workspace_bytes(plan, int(N), int(E)))


def eqconv_backward_radial(plan: int, graph: eqconv_graph_t, x, r, W1, W2, W3, n_basis: int, r_cut: float, gy,
                           dx, dr, gW1, gW2, gW3, workspace, workspace_bytes: int, stream=None) -> None:
    f = _f32()
    _check(lib().eqconv_backward_radial(plan, ctypes.byref(graph), _ptr(x, f), _ptr(r, f), _ptr(W1, f), _ptr(W2, f),
                                        _ptr(W3, f), int(n_basis), float(r_cut), _ptr(gy, f), _ptr(dx, f),
                                        _ptr(dr, f), _ptr(gW1, f), _ptr(gW2, f), _ptr(gW3, f), _ptr(workspace),
                                        int(workspace_bytes), _stream(stream)), "eqconv_backward_radial")


def eqconv_symmetric_contraction_plan_create(irreps_A: str, irreps_out: str, C: int, n_species: int) -> int:
    h = _vp()
    _check(lib().eqconv_symmetric_contraction_plan_create(ctypes.byref(h), irreps_A.encode(), irreps_out.encode(),
                                                          int(C), int(n_species)),
           "eqconv_symmetric_contraction_plan_create")
    return h.value


def eqconv_symmetric_contraction(plan: int, N: int, A, species, W1, W2, B_out, stream=None) -> None:
    f = _f32()
    _check(lib().eqconv_symmetric_contraction(plan, int(N), _ptr(A, f), _ptr(species, _i32()), _ptr(W1, f),
                                              _ptr(W2, f), _ptr(B_out, f), _stream(stream)),
           "eqconv_symmetric_contraction")


def eqconv_symmetric_contraction_workspace_bytes(plan: int, N: int) -> int:
    return int(lib().eqconv_symmetric_contraction_workspace_bytes(plan, int(N)))


def eqconv_symmetric_contraction_backward(plan: int, N: int, A, species, W1, W2, gB, dA, dW1, dW2, workspace,
                                          workspace_bytes: int, stream=None) -> None:
    f = _f32()
    _check(lib().eqconv_symmetric_contraction_backward(plan, int(N), _ptr(A, f), _ptr(species, _i32()), _ptr(W1, f),
                                                       _ptr(W2, f), _ptr(gB, f), _ptr(dA, f), _ptr(dW1, f),
                                                       _ptr(dW2, f), _ptr(workspace), int(workspace_bytes),
                                                       _stream(stream)),
           "eqconv_symmetric_contraction_backward")


def eqconv_spherical_harmonics(plan: int, E: int, r, Y, stream=None) -> None:
    f = _f32()
    _check(lib().eqconv_spherical_harmonics(plan, int(E), _ptr(r, f), _ptr(Y, f), _stream(stream)),
           "eqconv_spherical_harmonics")


def eqconv_get_device_error(plan: int, stream=None) -> int:
    st = ctypes.c_int()
    _check(lib().eqconv_get_device_error(plan, _stream(stream), ctypes.byref(st)), "eqconv_get_device_error")
    return st.value


def eqconv_plan_destroy(plan: int) -> None:
    if plan:
        lib().eqconv_plan_destroy(plan)
