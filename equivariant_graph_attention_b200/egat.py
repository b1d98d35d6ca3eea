"""Python binding of libegat.so (argument marshalling only).

Every function here forwards torch tensors' device pointers to the C ABI in
``include/egat.h`` and raises :class:`EgatError` on a nonzero return code.
All arithmetic runs in the library's CUDA kernels; torch only allocates the
output and scratch buffers and supplies the current stream.  There is no CPU
fallback: importing the library fails loudly when ``libegat.so`` is missing
(build it with ``python -m equivariant_graph_attention_b200.build``).

Function names match the C entry points (``egat_build_graph`` ...).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libegat.so")

EGAT_OK = 0
EGAT_ERR_ARG = -1
EGAT_ERR_UNSUPPORTED = -2
EGAT_ERR_CUDA = -3
EGAT_ERR_WORKSPACE = -4
EGAT_ERR_SCRATCH_LIMIT = -5
EGAT_ERR_TIMEOUT = -6
#: size of the fixed scratch array behind egat_forward_noalloc
NOALLOC_SCRATCH_BYTES = 32 << 20
EGAT_F32 = 0
EGAT_BF16 = 1
EGAT_GRAPH_PADDED = 0
EGAT_GRAPH_CSR = 1

#: every symbol include/egat.h declares
EXPORTS = ["egat_version", "egat_strerror", "egat_num_paths", "egat_graph_workspace_bytes",
           "egat_build_graph", "egat_eaas_couple", "egat_otf_attention",
           "egat_otf_attention_coupled",
           "egat_forward_workspace_bytes", "egat_forward", "egat_forward_noalloc",
           "egat_attention_plan_bytes", "egat_build_attention_plan", "egat_otf_attention_tiled",
           "egat_eaas_couple_planned", "egat_take_device_status", "egat_selftest_wait_timeout",
           "egat_backward_workspace_bytes", "egat_backward", "egat_gather_rows",
           "egat_qk_projection", "egat_escn_num_weights", "egat_escn_conv"]


class EgatError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


class egat_shape(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int32), ("lmax", ctypes.c_int32), ("C", ctypes.c_int32),
                ("H", ctypes.c_int32), ("dk", ctypes.c_int32), ("K", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("graph_mode", ctypes.c_int32),
                ("n_edges", ctypes.c_int64)]


_lib = None


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libegat.so (once) and declare its signatures."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or _LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"libegat.so not found at {p}; build it with "
                          "`python -m equivariant_graph_attention_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sp = ctypes.POINTER(egat_shape)
    lib.egat_version.restype = ctypes.c_int
    lib.egat_version.argtypes = []
    lib.egat_strerror.restype = ctypes.c_char_p
    lib.egat_strerror.argtypes = [ctypes.c_int]
    lib.egat_num_paths.restype = ctypes.c_int
    lib.egat_num_paths.argtypes = [ctypes.c_int]
    lib.egat_graph_workspace_bytes.restype = ctypes.c_int
    lib.egat_graph_workspace_bytes.argtypes = [i32, ctypes.POINTER(sz)]
    lib.egat_build_graph.restype = ctypes.c_int
    lib.egat_build_graph.argtypes = [vp, i32, i32, i32, i32, vp, vp, i64, vp, vp, vp, sz, vp]
    lib.egat_eaas_couple.restype = ctypes.c_int
    lib.egat_eaas_couple.argtypes = [sp, vp, vp, vp, vp, vp]
    lib.egat_otf_attention.restype = ctypes.c_int
    lib.egat_otf_attention.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.egat_otf_attention_coupled.restype = ctypes.c_int
    lib.egat_otf_attention_coupled.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.egat_forward_workspace_bytes.restype = ctypes.c_int
    lib.egat_forward_workspace_bytes.argtypes = [sp, ctypes.POINTER(sz)]
    lib.egat_forward.restype = ctypes.c_int
    lib.egat_forward.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    lib.egat_attention_plan_bytes.restype = ctypes.c_int
    lib.egat_attention_plan_bytes.argtypes = [sp, ctypes.POINTER(sz)]
    lib.egat_build_attention_plan.restype = ctypes.c_int
    lib.egat_build_attention_plan.argtypes = [sp, vp, vp, vp, vp, vp, sz, vp]
    lib.egat_backward_workspace_bytes.restype = ctypes.c_int
    lib.egat_backward_workspace_bytes.argtypes = [sp, ctypes.POINTER(sz)]
    lib.egat_gather_rows.restype = ctypes.c_int
    lib.egat_gather_rows.argtypes = [vp, i64, i64, vp, i64, vp, vp]
    lib.egat_backward.restype = ctypes.c_int
    lib.egat_backward.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp, vp, vp, vp]
    lib.egat_escn_num_weights.restype = ctypes.c_int
    lib.egat_escn_num_weights.argtypes = [i32, i32]
    lib.egat_escn_conv.restype = ctypes.c_int
    lib.egat_escn_conv.argtypes = [sp, i32, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.egat_qk_projection.restype = ctypes.c_int
    lib.egat_qk_projection.argtypes = [sp, vp, vp, vp, vp, vp, vp]
    lib.egat_take_device_status.restype = ctypes.c_int
    lib.egat_take_device_status.argtypes = [vp]
    lib.egat_selftest_wait_timeout.restype = ctypes.c_int
    lib.egat_selftest_wait_timeout.argtypes = [i32, vp]
    lib.egat_eaas_couple_planned.restype = ctypes.c_int
    lib.egat_eaas_couple_planned.argtypes = [sp, vp, vp, vp, vp, vp]
    lib.egat_otf_attention_tiled.restype = ctypes.c_int
    lib.egat_otf_attention_tiled.argtypes = [sp, vp, vp, vp, vp, vp, vp, i32, vp]
    lib.egat_forward_noalloc.restype = ctypes.c_int
    lib.egat_forward_noalloc.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    if path is None:
        _lib = lib
    return lib


def _check(fn: str, code: int):
    if code != EGAT_OK:
        raise EgatError(fn, code, load_library().egat_strerror(code).decode())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("egat: tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("egat: tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


@dataclass(frozen=True)
class Shape:
    n: int
    lmax: int
    C: int
    H: int
    dk: int
    K: int
    dtype: str = "f32"          # "f32" or "bf16": storage of h, q, k and h'
    graph_mode: str = "padded"  # "padded" or "csr"
    n_edges: int = 0

    @property
    def D(self) -> int:
        return (self.lmax + 1) ** 2

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def c(self) -> egat_shape:
        return egat_shape(self.n, self.lmax, self.C, self.H, self.dk, self.K,
                          EGAT_BF16 if self.dtype == "bf16" else EGAT_F32,
                          EGAT_GRAPH_CSR if self.graph_mode == "csr" else EGAT_GRAPH_PADDED,
                          self.n_edges)


def tc_attention_shape(shape: Shape) -> bool:
    """Whether the shape is one the tensor-core attention path takes (bf16
    storage, padded graph, C = 128, H = 16, dk = 16, lmax 1-3); the library
    also requires n below its plan builder's limit (EGAT_ERR_UNSUPPORTED past
    it)."""
    return (shape.dtype == "bf16" and shape.graph_mode == "padded" and shape.C == 128
            and shape.H == 16 and shape.dk == 16 and 1 <= shape.lmax <= 3)


def egat_version() -> int:
    return load_library().egat_version()


def egat_num_paths(lmax: int) -> int:
    return load_library().egat_num_paths(lmax)


def egat_graph_workspace_bytes(n: int) -> int:
    out = ctypes.c_size_t(0)
    _check("egat_graph_workspace_bytes", load_library().egat_graph_workspace_bytes(n, ctypes.byref(out)))
    return out.value


def egat_forward_workspace_bytes(shape: Shape) -> int:
    out = ctypes.c_size_t(0)
    cs = shape.c()
    _check("egat_forward_workspace_bytes",
           load_library().egat_forward_workspace_bytes(ctypes.byref(cs), ctypes.byref(out)))
    return out.value


def egat_build_graph(pos_q: torch.Tensor, cutoff_q: int, K: int = 0, mode: str = "padded",
                     col_capacity: int = 0, want_order: bool = True,
                     workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """Radius graph of int32 grid positions [n, 3] on the device.

    padded: returns {"nbr": [n, K] int32, "cnt": [n] int32, "order", "overflow"};
    csr:    returns {"rowptr": [n+1], "col": [col_capacity], "order", "overflow"}.
    ``overflow`` is a one-element device tensor (dropped neighbours).
    """
    if pos_q.dtype != torch.int32 or pos_q.dim() != 2 or pos_q.shape[1] != 3:
        raise ValueError("pos_q must be int32 [n, 3]")
    n = pos_q.shape[0]
    dev = pos_q.device
    ws_bytes = egat_graph_workspace_bytes(n)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    order = torch.empty(n, dtype=torch.int32, device=dev) if want_order else None
    overflow = torch.zeros(1, dtype=torch.int32, device=dev)
    if mode == "padded":
        a = torch.empty((n, K), dtype=torch.int32, device=dev)
        b = torch.empty(n, dtype=torch.int32, device=dev)
        m = EGAT_GRAPH_PADDED
    elif mode == "csr":
        a = torch.empty(n + 1, dtype=torch.int32, device=dev)
        b = torch.empty(max(col_capacity, 1), dtype=torch.int32, device=dev)
        m = EGAT_GRAPH_CSR
    else:
        raise ValueError(mode)
    rc = load_library().egat_build_graph(
        _ptr(pos_q), n, int(cutoff_q), int(K), m, _ptr(a), _ptr(b), int(col_capacity),
        _ptr(order), _ptr(overflow), _ptr(workspace), workspace.numel(), _stream(stream))
    _check("egat_build_graph", rc)
    out = {"order": order, "overflow": overflow}
    if mode == "padded":
        out.update(nbr=a, cnt=b)
    else:
        out.update(rowptr=a, col=b[:col_capacity])
    return out


def egat_eaas_couple(shape: Shape, x: torch.Tensor, pos: torch.Tensor, w: torch.Tensor,
                     out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """EAAS coupling y = x (x) R(pos) with path weights w [P, C]; x, y [n, D, C]."""
    if out is None:
        out = torch.empty_like(x)
    cs = shape.c()
    rc = load_library().egat_eaas_couple(ctypes.byref(cs), _ptr(x), _ptr(pos), _ptr(w),
                                         _ptr(out), _stream(stream))
    _check("egat_eaas_couple", rc)
    return out


def egat_qk_projection(shape: Shape, h: torch.Tensor, wq: torch.Tensor, wk: torch.Tensor,
                       q: Optional[torch.Tensor] = None, k: Optional[torch.Tensor] = None,
                       stream=None):
    """Invariant queries and keys from the degree-0 channels of h:
    q[i, h, d] = sum_c h[i, 0, c] wq[c, h*dk + d] (k likewise); (q, k) [n, H, dk]
    in the storage type.  wq, wk float32 [C, H*dk]."""
    shp = (shape.n, shape.H, shape.dk)
    if q is None:
        q = torch.empty(shp, dtype=shape.torch_dtype, device=h.device)
    if k is None:
        k = torch.empty(shp, dtype=shape.torch_dtype, device=h.device)
    cs = shape.c()
    rc = load_library().egat_qk_projection(ctypes.byref(cs), _ptr(h), _ptr(wq), _ptr(wk), _ptr(q),
                                           _ptr(k), _stream(stream))
    _check("egat_qk_projection", rc)
    return q, k


def egat_escn_num_weights(lmax: int, mmax: int) -> int:
    return load_library().egat_escn_num_weights(lmax, mmax)


def egat_escn_conv(shape: Shape, mmax: int, h: torch.Tensor, pos: torch.Tensor, nbr: torch.Tensor,
                   cnt: Optional[torch.Tensor], w: torch.Tensor, order: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Edge-centric eSCN convolution out_i = sum_j D(Q_ij) SO2_w(D(Q_ij)^T h_j) over
    the padded graph; w float32 [egat_escn_num_weights(lmax, mmax), C]; out
    float32 [n, D, C]."""
    if out is None:
        out = torch.empty((shape.n, shape.D, shape.C), dtype=torch.float32, device=h.device)
    cs = shape.c()
    rc = load_library().egat_escn_conv(ctypes.byref(cs), mmax, _ptr(h), _ptr(pos), _ptr(nbr),
                                       _ptr(cnt), _ptr(order), _ptr(w), _ptr(out), _stream(stream))
    _check("egat_escn_conv", rc)
    return out


def egat_otf_attention(shape: Shape, q: torch.Tensor, k: torch.Tensor, hp: torch.Tensor,
                       nbr_or_rowptr: torch.Tensor, cnt_or_col: Optional[torch.Tensor],
                       order: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    """Streaming attention m_i = sum_j softmax(q_i.k_j/sqrt(dk)) h'_j; m float32 [n, D, C]."""
    if out is None:
        out = torch.empty((shape.n, shape.D, shape.C), dtype=torch.float32, device=hp.device)
    cs = shape.c()
    rc = load_library().egat_otf_attention(
        ctypes.byref(cs), _ptr(q), _ptr(k), _ptr(hp), _ptr(nbr_or_rowptr), _ptr(cnt_or_col),
        _ptr(order), _ptr(out), _stream(stream))
    _check("egat_otf_attention", rc)
    return out


def egat_otf_attention_coupled(shape: Shape, q: torch.Tensor, k: torch.Tensor, hp: torch.Tensor,
                               nbr_or_rowptr: torch.Tensor, cnt_or_col: Optional[torch.Tensor],
                               pos: torch.Tensor, w2: torch.Tensor,
                               order: Optional[torch.Tensor] = None,
                               out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Attention with the target coupling fused into its epilogue; ^h float32 [n, D, C]."""
    if out is None:
        out = torch.empty((shape.n, shape.D, shape.C), dtype=torch.float32, device=hp.device)
    cs = shape.c()
    rc = load_library().egat_otf_attention_coupled(
        ctypes.byref(cs), _ptr(q), _ptr(k), _ptr(hp), _ptr(nbr_or_rowptr), _ptr(cnt_or_col),
        _ptr(order), _ptr(pos), _ptr(w2), _ptr(out), _stream(stream))
    _check("egat_otf_attention_coupled", rc)
    return out


def egat_attention_plan_bytes(shape: Shape) -> int:
    out = ctypes.c_size_t(0)
    cs = shape.c()
    _check("egat_attention_plan_bytes",
           load_library().egat_attention_plan_bytes(ctypes.byref(cs), ctypes.byref(out)))
    return out.value


def egat_build_attention_plan(shape: Shape, nbr: torch.Tensor, cnt: Optional[torch.Tensor],
                              order: Optional[torch.Tensor] = None,
                              pos: Optional[torch.Tensor] = None,
                              plan: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Per-tile neighbour unions, membership masks and target records (atom ids,
    |r|^l, Wigner-D of the alignment rotations) for egat_otf_attention_tiled.
    `pos` (float32 [n, 3]) is required."""
    nb = egat_attention_plan_bytes(shape)
    if plan is None:
        plan = torch.empty(max(nb, 16), dtype=torch.uint8, device=nbr.device)
    cs = shape.c()
    rc = load_library().egat_build_attention_plan(ctypes.byref(cs), _ptr(nbr), _ptr(cnt),
                                                  _ptr(order), _ptr(pos), _ptr(plan),
                                                  plan.numel(), _stream(stream))
    _check("egat_build_attention_plan", rc)
    return plan


def egat_backward_workspace_bytes(shape: Shape) -> int:
    out = ctypes.c_size_t(0)
    cs = shape.c()
    _check("egat_backward_workspace_bytes",
           load_library().egat_backward_workspace_bytes(ctypes.byref(cs), ctypes.byref(out)))
    return out.value


def egat_backward(shape: Shape, h: torch.Tensor, pos: torch.Tensor, q: torch.Tensor,
                  k: torch.Tensor, nbr: torch.Tensor, cnt: Optional[torch.Tensor],
                  w1: torch.Tensor, w2: torch.Tensor, grad_out: torch.Tensor,
                  workspace: Optional[torch.Tensor] = None, positions: bool = True,
                  order: Optional[torch.Tensor] = None, stream=None):
    """(dL/dh, dL/dq, dL/dk, dL/dr) float32 for the upstream gradient grad_out = dL/d^h
    (dL/dr is None when positions=False, which also skips m and makes the call
    cheaper); order = the graph builder's traversal order (tiles of spatially
    adjacent atoms), optional: results do not depend on it up to rounding."""
    nb = egat_backward_workspace_bytes(shape)
    if workspace is None:
        workspace = torch.empty(max(nb, 16), dtype=torch.uint8, device=h.device)
    dev = h.device
    dh = torch.empty((shape.n, shape.D, shape.C), dtype=torch.float32, device=dev)
    dq = torch.empty((shape.n, shape.H, shape.dk), dtype=torch.float32, device=dev)
    dk = torch.empty((shape.n, shape.H, shape.dk), dtype=torch.float32, device=dev)
    dpos = torch.empty((shape.n, 3), dtype=torch.float32, device=dev) if positions else None
    cs = shape.c()
    rc = load_library().egat_backward(
        ctypes.byref(cs), _ptr(h), _ptr(pos), _ptr(q), _ptr(k), _ptr(nbr), _ptr(cnt), _ptr(order),
        _ptr(w1), _ptr(w2), _ptr(grad_out), _ptr(workspace), workspace.numel(), _ptr(dh), _ptr(dq),
        _ptr(dk), _ptr(dpos), _stream(stream))
    _check("egat_backward", rc)
    return dh, dq, dk, dpos


def egat_gather_rows(src: torch.Tensor, idx: torch.Tensor, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """out[r] = src[idx[r]] along the first dimension (an index outside
    [0, len(src)) gives a zero row); rows must be a multiple of 16 bytes."""
    n = src.shape[0]
    row_bytes = src[0].numel() * src.element_size() if n > 0 else (
        int(torch.tensor(src.shape[1:]).prod()) * src.element_size())
    if out is None:
        out = torch.empty((idx.numel(),) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    _check("egat_gather_rows", load_library().egat_gather_rows(
        _ptr(src) if n > 0 else None, n, row_bytes, _ptr(idx), idx.numel(), _ptr(out), _stream(stream)))
    return out


def egat_take_device_status(stream=None) -> int:
    """Synchronise the stream; EGAT_ERR_TIMEOUT if a bounded device wait gave up
    since the last call (the count is cleared), EGAT_OK otherwise."""
    return load_library().egat_take_device_status(_stream(stream))


def egat_selftest_wait_timeout(polls: int = 1000, stream=None) -> None:
    """Launch the wait that cannot succeed (see include/egat.h)."""
    _check("egat_selftest_wait_timeout",
           load_library().egat_selftest_wait_timeout(int(polls), _stream(stream)))


def egat_eaas_couple_planned(shape: Shape, h: torch.Tensor, plan: torch.Tensor, w: torch.Tensor,
                             out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Step 2 for the atoms of an attention plan, rotations from its tile records."""
    if out is None:
        out = torch.empty_like(h)
    cs = shape.c()
    rc = load_library().egat_eaas_couple_planned(ctypes.byref(cs), _ptr(h), _ptr(plan), _ptr(w),
                                                 _ptr(out), _stream(stream))
    _check("egat_eaas_couple_planned", rc)
    return out


def egat_otf_attention_tiled(shape: Shape, q: torch.Tensor, k: torch.Tensor, hp: torch.Tensor,
                             plan: torch.Tensor, w2: Optional[torch.Tensor] = None,
                             fused: bool = True, out: Optional[torch.Tensor] = None,
                             stream=None) -> torch.Tensor:
    """Tensor-core attention over a plan: ^h (fused, w2 required) or m, float32 [n, D, C]."""
    if out is None:
        out = torch.empty((shape.n, shape.D, shape.C), dtype=torch.float32, device=hp.device)
    cs = shape.c()
    rc = load_library().egat_otf_attention_tiled(
        ctypes.byref(cs), _ptr(q), _ptr(k), _ptr(hp), _ptr(plan), _ptr(w2), _ptr(out),
        1 if fused else 0, _stream(stream))
    _check("egat_otf_attention_tiled", rc)
    return out


def egat_forward(shape: Shape, h: torch.Tensor, pos: torch.Tensor, q: torch.Tensor,
                 k: torch.Tensor, nbr_or_rowptr: torch.Tensor, cnt_or_col: Optional[torch.Tensor],
                 w1: torch.Tensor, w2: torch.Tensor, order: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """Fused forward ^h = attention(EAAS(h, w1)) (x) R(r_i) with w2; float32 [n, D, C]."""
    if out is None:
        out = torch.empty((shape.n, shape.D, shape.C), dtype=torch.float32, device=h.device)
    ws = egat_forward_workspace_bytes(shape)
    if workspace is None:
        workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=h.device)
    cs = shape.c()
    rc = load_library().egat_forward(
        ctypes.byref(cs), _ptr(h), _ptr(pos), _ptr(q), _ptr(k), _ptr(nbr_or_rowptr),
        _ptr(cnt_or_col), _ptr(order), _ptr(w1), _ptr(w2), _ptr(workspace), workspace.numel(),
        _ptr(out), _stream(stream))
    _check("egat_forward", rc)
    return out


def egat_forward_noalloc(shape: Shape, h: torch.Tensor, pos: torch.Tensor, q: torch.Tensor,
                         k: torch.Tensor, nbr_or_rowptr: torch.Tensor,
                         cnt_or_col: Optional[torch.Tensor], w1: torch.Tensor, w2: torch.Tensor,
                         out: torch.Tensor, order: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """egat_forward without a workspace: the library's fixed scratch array holds h'.

    For callers that may not allocate device memory at call time; ``out`` must
    be provided by the caller.  Problems whose h' exceeds
    ``NOALLOC_SCRATCH_BYTES`` raise EgatError(EGAT_ERR_SCRATCH_LIMIT).  Calls
    that overlap on the GPU share the scratch and race; serialise them.
    """
    cs = shape.c()
    rc = load_library().egat_forward_noalloc(
        ctypes.byref(cs), _ptr(h), _ptr(pos), _ptr(q), _ptr(k), _ptr(nbr_or_rowptr),
        _ptr(cnt_or_col), _ptr(order), _ptr(w1), _ptr(w2), _ptr(out), _stream(stream))
    _check("egat_forward_noalloc", rc)
    return out
