"""User-level API over the C ABI: plans, edge layouts and the convolution as a
torch.autograd.Function.  Device memory and streams come from PyTorch; every
step of the convolution runs in libeqconv's kernels (see binding.py).

    conv = EqConv("0e+1o+2e", 2, "0e+1o+2e", C=128)
    g = conv.graph(senders, receivers, N)           # CSR + permutations, on device
    y = conv(g, x, r, w)                            # differentiable in x, r, w
"""
from __future__ import annotations

import torch

from . import binding as B


class Graph:
    """Edge layout on one device: the caller's senders/receivers (int32, kept
    alive here) plus the receiver/sender CSR built by eqconv_graph_build."""

    def __init__(self, plan: int, senders: torch.Tensor, receivers: torch.Tensor, N: int, stream=None):
        if senders.dtype != torch.int32 or receivers.dtype != torch.int32:
            raise ValueError("senders and receivers must be int32")
        if senders.shape != receivers.shape or senders.dim() != 1:
            raise ValueError("senders and receivers must be 1-D of equal length")
        dev = senders.device
        E = senders.numel()
        self.N, self.E = int(N), int(E)
        self.senders = senders.contiguous()
        self.receivers = receivers.contiguous()
        self.recv_ptr = torch.empty(N + 1, dtype=torch.int32, device=dev)
        self.send_ptr = torch.empty(N + 1, dtype=torch.int32, device=dev)
        self.recv_perm = torch.empty(max(E, 1), dtype=torch.int32, device=dev)
        self.send_perm = torch.empty(max(E, 1), dtype=torch.int32, device=dev)
        self.c = B.eqconv_graph_t(self.N, self.E, self.senders.data_ptr() if E else 0,
                                  self.receivers.data_ptr() if E else 0, self.recv_ptr.data_ptr(),
                                  self.recv_perm.data_ptr(), self.send_ptr.data_ptr(), self.send_perm.data_ptr())
        nbytes = B.eqconv_graph_workspace_bytes(self.N, self.E)
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
        B.eqconv_graph_build(plan, self.c, ws, nbytes, stream)
        self._ws = ws  # freed with the graph; the build is stream-ordered


class EqConv:
    """One convolution configuration (irreps, L_sh, C) on the current device.

    all_parity: outputs of both parities (irreps_out is then the both-parity
    prefix "0e+1o+1e+2e+2o..."); per_path: one output block per path, in path
    order, starting at row ``self.path_rows[p]`` (see include/eqconv.h)."""

    def __init__(self, irreps_in: str, L_sh: int, irreps_out: str, C: int, all_parity: bool = False,
                 per_path: bool = False):
        self.irreps_in, self.L_sh, self.irreps_out, self.C = irreps_in, L_sh, irreps_out, C
        mode = (B.EQCONV_OUT_ALL_PARITY if all_parity else 0) | (B.EQCONV_OUT_PER_PATH if per_path else 0)
        self.out_mode = mode
        self.plan = B.eqconv_plan_create_ex(irreps_in, L_sh, irreps_out, C, mode)
        info = B.eqconv_plan_info(self.plan)
        self.P, self.D_in, self.D_sh, self.D_out = info["P"], info["D_in"], info["D_sh"], info["D_out"]
        self.paths = info["paths"]
        self.path_rows = B.eqconv_plan_path_rows(self.plan)

    def __del__(self):
        try:
            B.eqconv_plan_destroy(self.plan)
        except Exception:
            pass

    def set_vec(self, fwd_vec: int, bwd_vec: int):
        B.eqconv_plan_set_vec(self.plan, fwd_vec, bwd_vec)

    def set_gather_budget(self, nbytes: int):
        """L2 budget of one gather band (0: no banding); see include/eqconv.h."""
        B.eqconv_plan_set_gather_budget(self.plan, nbytes)

    def graph(self, senders: torch.Tensor, receivers: torch.Tensor, N: int, stream=None) -> Graph:
        return Graph(self.plan, senders, receivers, N, stream)

    def forward_raw(self, g: Graph, x, r, w, y=None, stream=None):
        if y is None:
            y = torch.empty((g.N, self.D_out, self.C), dtype=torch.float32, device=x.device)
        B.eqconv_forward(self.plan, g.c, x, r, w, y, 0, stream)
        return y

    def backward_raw(self, g: Graph, x, r, w, gy, deterministic=True, out=None, workspace=None, stream=None):
        if out is None:
            dx = torch.empty_like(x)
            dw = torch.empty_like(w)
            dr = torch.empty_like(r)
        else:
            dx, dw, dr = out
        nbytes = B.eqconv_backward_workspace_bytes(self.plan, g.E)
        if nbytes and workspace is None:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
        B.eqconv_backward(self.plan, g.c, x, r, w, gy, dx, dw, dr, workspace, nbytes,
                          B.EQCONV_DETERMINISTIC if deterministic else 0, stream)
        return dx, dw, dr

    def double_backward_raw(self, g: Graph, x, r, w, gy, ga, gb, gq, out=None, workspace=None, stream=None):
        """Gradient of <ga, dx> + <gb, dw> + <gq, dr> w.r.t. (x, w, gy, r); see
        include/eqconv.h.  Returns (g_x, g_w, g_gy, g_r)."""
        if out is None:
            out = (torch.empty_like(x), torch.empty_like(w), torch.empty_like(gy), torch.empty_like(r))
        g_x, g_w, g_gy, g_r = out
        nbytes = B.eqconv_double_backward_workspace_bytes(self.plan, g.E)
        if nbytes and workspace is None:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
        B.eqconv_double_backward(self.plan, g.c, x, r, w, gy, ga, gb, gq, g_x, g_w, g_gy, g_r, workspace, nbytes,
                                 stream)
        return g_x, g_w, g_gy, g_r

    def __call__(self, g: Graph, x, r, w, deterministic=True):
        return _EqConvFn.apply(self, g, deterministic, x, r, w)


class _EqConvFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, conv: EqConv, g: Graph, deterministic: bool, x, r, w):
        x, r, w = x.contiguous(), r.contiguous(), w.contiguous()
        ctx.conv, ctx.g, ctx.det = conv, g, deterministic
        ctx.save_for_backward(x, r, w)
        return conv.forward_raw(g, x, r, w)

    @staticmethod
    def backward(ctx, gy):
        x, r, w = ctx.saved_tensors
        if torch.is_grad_enabled():
            # create_graph=True (force training): a differentiable backward
            dx, dw, dr = _EqConvBwdFn.apply(ctx.conv, ctx.g, ctx.det, x, r, w, gy.contiguous())
        else:
            dx, dw, dr = ctx.conv.backward_raw(ctx.g, x, r, w, gy.contiguous(), ctx.det)
        return None, None, None, dx, dr, dw


class _EqConvBwdFn(torch.autograd.Function):
    """The backward as a function of (x, r, w, gy), differentiated by the
    library's double backward."""

    @staticmethod
    def forward(ctx, conv: EqConv, g: Graph, deterministic: bool, x, r, w, gy):
        ctx.conv, ctx.g = conv, g
        ctx.save_for_backward(x, r, w, gy)
        return conv.backward_raw(g, x, r, w, gy, deterministic)

    @staticmethod
    def backward(ctx, ga, gb, gq):
        x, r, w, gy = ctx.saved_tensors
        z = lambda t, like: torch.zeros_like(like) if t is None else t.contiguous()
        g_x, g_w, g_gy, g_r = ctx.conv.double_backward_raw(ctx.g, x, r, w, gy, z(ga, x), z(gb, w), z(gq, r))
        return None, None, None, g_x, g_r, g_w, g_gy


class RadialEqConv:
    """The convolution with its weights produced on the chip from the edge
    lengths by the radial MLP (Bessel basis, C2 envelope, 2 SiLU layers of
    width 64; see include/eqconv.h, eqconv_forward_radial):

        conv = RadialEqConv("0e+1o+2e+3o", 3, "0e+1o+2e+3o", C=128, n_basis=8, r_cut=5.0)
        y = conv(g, x, r, W1, W2, W3)       # differentiable in x, r, W1, W2, W3

    The backward runs eqconv_backward_radial (deterministic; w and dw never
    in memory); it is not twice differentiable."""

    def __init__(self, irreps_in: str, L_sh: int, irreps_out: str, C: int, n_basis: int = 8, r_cut: float = 5.0,
                 per_path: bool = False):
        self.conv = EqConv(irreps_in, L_sh, irreps_out, C, per_path=per_path)
        self.plan, self.P, self.D_in, self.D_out, self.C = (self.conv.plan, self.conv.P, self.conv.D_in,
                                                            self.conv.D_out, C)
        self.n_basis, self.r_cut = int(n_basis), float(r_cut)
        if B.eqconv_forward_radial_workspace_bytes(self.plan, 1, 1) == 0:
            raise B.EqconvError("RadialEqConv: no fused radial path for this plan", B.EQCONV_ERR_UNSUPPORTED)

    def graph(self, senders, receivers, N, stream=None) -> Graph:
        return self.conv.graph(senders, receivers, N, stream)

    def forward_raw(self, g: Graph, x, r, W1, W2, W3, y=None, stream=None):
        if y is None:
            y = torch.empty((g.N, self.D_out, self.C), dtype=torch.float32, device=x.device)
        nbytes = B.eqconv_forward_radial_workspace_bytes(self.plan, g.N, g.E)
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
        B.eqconv_forward_radial(self.plan, g.c, x, r, W1, W2, W3, self.n_basis, self.r_cut, y, ws, nbytes, stream)
        return y

    def backward_raw(self, g: Graph, x, r, W1, W2, W3, gy, stream=None):
        dx, dr = torch.empty_like(x), torch.empty_like(r)
        gW1, gW2, gW3 = torch.empty_like(W1), torch.empty_like(W2), torch.empty_like(W3)
        nbytes = B.eqconv_backward_radial_workspace_bytes(self.plan, g.N, g.E)
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
        B.eqconv_backward_radial(self.plan, g.c, x, r, W1, W2, W3, self.n_basis, self.r_cut, gy, dx, dr, gW1, gW2,
                                 gW3, ws, nbytes, stream)
        return dx, dr, gW1, gW2, gW3

    def __call__(self, g: Graph, x, r, W1, W2, W3):
        return _RadialEqConvFn.apply(self, g, x, r, W1, W2, W3)


class _RadialEqConvFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, op: RadialEqConv, g: Graph, x, r, W1, W2, W3):
        args = [t.contiguous() for t in (x, r, W1, W2, W3)]
        ctx.op, ctx.g = op, g
        ctx.save_for_backward(*args)
        return op.forward_raw(g, *args)

    @staticmethod
    def backward(ctx, gy):
        x, r, W1, W2, W3 = ctx.saved_tensors
        dx, dr, gW1, gW2, gW3 = ctx.op.backward_raw(ctx.g, x, r, W1, W2, W3, gy.contiguous())
        return None, None, dx, dr, gW1, gW2, gW3


class NodeProduct:
    """Node-local channel-diagonal product of two node features (see
    include/eqconv.h): y = sum_p w_p C_p u_l1 v_l2, summed per output irrep or
    kept per path (per_path=True)."""

    def __init__(self, irreps_u: str, L_v: int, irreps_out: str, C: int, per_path: bool = False):
        self.irreps_u, self.L_v, self.irreps_out, self.C = irreps_u, L_v, irreps_out, C
        self.plan = B.eqconv_node_product_plan_create(irreps_u, L_v, irreps_out, C,
                                                      B.EQCONV_OUT_PER_PATH if per_path else 0)
        info = B.eqconv_plan_info(self.plan)
        self.P, self.D_u, self.D_v, self.D_out = info["P"], info["D_in"], info["D_sh"], info["D_out"]
        self.paths = info["paths"]
        self.path_rows = B.eqconv_plan_path_rows(self.plan)

    def __del__(self):
        try:
            B.eqconv_plan_destroy(self.plan)
        except Exception:
            pass

    def forward_raw(self, u, v, w=None, y=None, stream=None):
        if y is None:
            y = torch.empty((u.shape[0], self.D_out, self.C), dtype=torch.float32, device=u.device)
        B.eqconv_node_product(self.plan, u.shape[0], u, v, w, y, stream)
        return y

    def backward_raw(self, u, v, w, gy, need_dw=True, workspace=None, stream=None):
        N = u.shape[0]
        du, dv = torch.empty_like(u), torch.empty_like(v)
        if N == 0:      # no nodes: nothing to launch, dw is an empty sum
            return du, dv, (torch.zeros((self.P, self.C), dtype=torch.float32, device=u.device) if need_dw else None)
        dw = torch.empty((self.P, self.C), dtype=torch.float32, device=u.device) if need_dw else None
        nbytes = B.eqconv_node_product_workspace_bytes(self.plan, N) if need_dw else 0
        if nbytes and workspace is None:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=u.device)
        B.eqconv_node_product_backward(self.plan, N, u, v, w, gy, du, dv, dw, workspace, nbytes, stream)
        return du, dv, dw

    def __call__(self, u, v, w=None):
        return _NodeProductFn.apply(self, u, v, w)


class _NodeProductFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, op: NodeProduct, u, v, w):
        u, v = u.contiguous(), v.contiguous()
        w = None if w is None else w.contiguous()
        ctx.op, ctx.has_w = op, w is not None
        ctx.save_for_backward(u, v, w)
        return op.forward_raw(u, v, w)

    @staticmethod
    def backward(ctx, gy):
        u, v, w = ctx.saved_tensors
        need_dw = ctx.has_w and ctx.needs_input_grad[3]
        du, dv, dw = ctx.op.backward_raw(u, v, w, gy.contiguous(), need_dw=need_dw)
        return None, du, dv, dw


class SymmetricContraction:
    """Symmetric contraction of correlation order 2 with per-species weights
    (the MACE product basis; see include/eqconv.h):

        sc = SymmetricContraction("0e+1o+2e+3o", "0e+1o", C=128, n_species=2)
        B = sc(A, species, W1, W2)           # differentiable in A, W1, W2

    W1 [S][min(L_A, L_out)+1][C], W2 [S][P][C] with P = len(sc.paths)."""

    def __init__(self, irreps_A: str, irreps_out: str, C: int, n_species: int):
        self.C, self.S = C, n_species
        self.plan = B.eqconv_symmetric_contraction_plan_create(irreps_A, irreps_out, C, n_species)
        info = B.eqconv_plan_info(self.plan)
        self.P, self.D_A, self.D_out, self.paths = info["P"], info["D_in"], info["D_out"], info["paths"]
        L_A = int(round(self.D_A ** 0.5)) - 1
        L_out = int(round(self.D_out ** 0.5)) - 1
        self.L1N = min(L_A, L_out) + 1

    def __del__(self):
        try:
            B.eqconv_plan_destroy(self.plan)
        except Exception:
            pass

    def forward_raw(self, A, species, W1, W2, out=None, stream=None):
        N = A.shape[0]
        if out is None:
            out = torch.empty((N, self.D_out, self.C), dtype=torch.float32, device=A.device)
        B.eqconv_symmetric_contraction(self.plan, N, A, species, W1, W2, out, stream)
        return out

    def backward_raw(self, A, species, W1, W2, gB, stream=None):
        N = A.shape[0]
        dA, dW1, dW2 = torch.empty_like(A), torch.empty_like(W1), torch.empty_like(W2)
        nbytes = B.eqconv_symmetric_contraction_workspace_bytes(self.plan, N)
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=A.device)
        B.eqconv_symmetric_contraction_backward(self.plan, N, A, species, W1, W2, gB, dA, dW1, dW2, ws, nbytes,
                                                stream)
        return dA, dW1, dW2

    def __call__(self, A, species, W1, W2):
        return _SymContractionFn.apply(self, A, species, W1, W2)


class _SymContractionFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, op: SymmetricContraction, A, species, W1, W2):
        A, W1, W2 = A.contiguous(), W1.contiguous(), W2.contiguous()
        ctx.op = op
        ctx.save_for_backward(A, species, W1, W2)
        return op.forward_raw(A, species, W1, W2)

    @staticmethod
    def backward(ctx, gB):
        A, species, W1, W2 = ctx.saved_tensors
        dA, dW1, dW2 = ctx.op.backward_raw(A, species, W1, W2, gB.contiguous())
        return None, dA, None, dW1, dW2

