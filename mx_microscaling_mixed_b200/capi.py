"""ctypes binding of libmxs (the C ABI in include/mxs.h), same entry-point names.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  torch supplies device memory (inputs, outputs, workspaces) and
streams.  The library must be built (``python -m mx_microscaling_mixed_b200.build``);
if it is missing this module raises on import -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmxs.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libmxs.so not built at {_LIB_PATH}; run python -m mx_microscaling_mixed_b200.build")
_lib = ctypes.CDLL(_LIB_PATH)

MXS_F32, MXS_BF16 = 0, 1
MXS_ALLOC_FRACTIONS, MXS_ALLOC_BUDGET, MXS_ALLOC_LAYER = 0, 1, 2
SEG_BITS = (8, 6, 4)

STATUS = {0: "MXS_OK", 1: "MXS_ERR_ARG", 2: "MXS_ERR_SHAPE", 3: "MXS_ERR_ALIGN", 4: "MXS_ERR_DTYPE",
          5: "MXS_ERR_BUDGET", 6: "MXS_ERR_CUDA", 7: "MXS_ERR_TIMEOUT", 8: "MXS_ERR_DEVICE",
          9: "MXS_ERR_WORKSPACE"}


class MxsError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.mxs_status_str(status).decode()}")


class Segment(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("k_real", ctypes.c_int64), ("k_pad", ctypes.c_int64),
                ("k_off", ctypes.c_int64)]


class LayoutC(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int64), ("K_pad", ctypes.c_int64), ("seg", Segment * 3),
                ("perm", ctypes.c_void_p)]


class MXTensorC(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("lay", LayoutC), ("codes", ctypes.c_void_p * 3),
                ("code_pitch", ctypes.c_int64 * 3), ("scales", ctypes.c_void_p * 3),
                ("scale_pitch", ctypes.c_int64 * 3)]


class StackC(ctypes.Structure):
    _fields_ = [("n_blocks", ctypes.c_int32), ("hidden", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("mlp", ctypes.c_int32), ("rms_eps", ctypes.c_float),
                ("rope_theta", ctypes.c_float), ("W", ctypes.c_void_p)]


class BudgetC(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("num", ctypes.c_int64), ("den", ctypes.c_int64),
                ("p8_num", ctypes.c_int64), ("p8_den", ctypes.c_int64), ("p6_num", ctypes.c_int64),
                ("p6_den", ctypes.c_int64), ("fixed8", ctypes.c_int64)]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_ST = ctypes.c_int


def _sig(name, args, res=_ST):
    f = getattr(_lib, name)
    f.argtypes = args
    f.restype = res
    return f


_sig("mxs_status_str", [_ST], ctypes.c_char_p)
_sig("mxs_launch_count", [], _I64)
_sig("mxs_sync", [_P])
_sig("mxs_set_wait_limit", [_I64])
_sig("mxs_layout_make", [_I64, _P, _P, ctypes.POINTER(LayoutC)])
_sig("mxs_mxtensor_bytes", [_I64, ctypes.POINTER(LayoutC), _P, _P, _P, _P])
_sig("mxs_sensitivity_workspace_bytes", [_I64, _I64, _I64, ctypes.POINTER(_SZ)])
_sig("mxs_sensitivity", [_P, _ST, _I64, _I64, _I64, _P, _ST, _I64, _I64, _P, _P, _P, _P, _SZ, _P])
_sig("mxs_sensitivity_noalloc", [_P, _ST, _I64, _I64, _I64, _P, _ST, _I64, _I64, _P, _P, _P, _P])
_sig("mxs_allocate_workspace_bytes", [ctypes.c_int32, _P, ctypes.POINTER(_SZ)])
_sig("mxs_allocate", [ctypes.c_int32, _P, _P, _P, _P, ctypes.POINTER(BudgetC), _P, _P, _P, _SZ, _P])
_sig("mxs_quantize_weight", [_P, _ST, _I64, _I64, ctypes.POINTER(MXTensorC), _P])
_sig("mxs_quantize_act", [_P, _ST, _I64, _I64, ctypes.POINTER(MXTensorC), _P])
_sig("mxs_dequantize", [ctypes.POINTER(MXTensorC), _P, _I64, _P])
_sig("mxs_gemm_workspace_bytes", [ctypes.POINTER(MXTensorC), ctypes.POINTER(MXTensorC), ctypes.POINTER(_SZ)])
_sig("mxs_gemm", [ctypes.POINTER(MXTensorC), ctypes.POINTER(MXTensorC), _P, _I64, _P, _SZ, _P])
_sig("mxs_layer_scores_workspace_bytes", [ctypes.POINTER(StackC), _I64, ctypes.POINTER(_SZ)])
_sig("mxs_layer_scores", [ctypes.POINTER(StackC), _P, _I64, _I64, _P, _P, _SZ, _P])
_sig("mxs_attn_decode_workspace_bytes", [_I64, _I64, _I64, _I64, ctypes.POINTER(_SZ)])
_sig("mxs_attn_decode", [_P, _I64, _I64, ctypes.POINTER(MXTensorC), ctypes.POINTER(MXTensorC), _I64, _I64,
                         ctypes.c_float, _P, _I64, _P, _SZ, _P])

EXPORTS = ["mxs_status_str", "mxs_launch_count", "mxs_sync", "mxs_set_wait_limit", "mxs_layout_make", "mxs_mxtensor_bytes",
           "mxs_sensitivity_workspace_bytes", "mxs_sensitivity", "mxs_sensitivity_noalloc",
           "mxs_allocate_workspace_bytes",
           "mxs_allocate", "mxs_quantize_weight", "mxs_quantize_act", "mxs_dequantize",
           "mxs_gemm_workspace_bytes", "mxs_gemm", "mxs_attn_decode_workspace_bytes", "mxs_attn_decode",
           "mxs_layer_scores_workspace_bytes", "mxs_layer_scores"]


def _check(st: int, where: str):
    if st != 0:
        raise MxsError(st, where)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MXS_F32
    if t.dtype == torch.bfloat16:
        return MXS_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _rowmajor(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit stride along K")
    return t.stride(0)


def _workspace(nbytes: int, device) -> torch.Tensor:
    # 1024 extra bytes so the base can be aligned to 1024 inside
    return torch.empty(int(nbytes) + 1024, dtype=torch.uint8, device=device)


def _aligned_ptr(buf: torch.Tensor, align: int = 1024) -> int:
    p = buf.data_ptr()
    return (p + align - 1) // align * align


# ------------------------------------------------------------------ layouts
@dataclass
class Layout:
    c: LayoutC
    counts: tuple
    perm: Optional[torch.Tensor] = None      # keeps the device permutation alive

    @property
    def K(self) -> int:
        return int(self.c.K)

    @property
    def K_pad(self) -> int:
        return int(self.c.K_pad)


def mxs_layout_make(K: int, counts: Sequence[int], perm: Optional[torch.Tensor] = None) -> Layout:
    arr = (ctypes.c_int64 * 3)(*[int(c) for c in counts])
    lay = LayoutC()
    if perm is not None:
        assert perm.dtype == torch.int32 and perm.is_cuda and perm.is_contiguous() and perm.numel() == K
    _check(_lib.mxs_layout_make(int(K), arr, None if perm is None else ctypes.c_void_p(perm.data_ptr()),
                                ctypes.byref(lay)), "mxs_layout_make")
    return Layout(lay, tuple(int(c) for c in counts), perm)


def mxs_mxtensor_bytes(rows: int, layout: Layout):
    cp, cb, sp, sb = [(ctypes.c_int64 * 3)() for _ in range(4)]
    _check(_lib.mxs_mxtensor_bytes(int(rows), ctypes.byref(layout.c), cp, cb, sp, sb), "mxs_mxtensor_bytes")
    return list(cp), list(cb), list(sp), list(sb)


@dataclass
class MXTensor:
    """A quantised matrix: per-segment code and scale buffers (torch uint8)."""
    rows: int
    layout: Layout
    codes: List[Optional[torch.Tensor]]
    scales: List[Optional[torch.Tensor]]
    c: MXTensorC = field(default_factory=MXTensorC)

    def code_rows(self, g: int) -> torch.Tensor:
        """Compact (rows x payload bytes) view of segment g's codes."""
        kp = self.layout.c.seg[g].k_pad
        return self.codes[g][:, :kp * SEG_BITS[g] // 8] if kp else torch.empty(self.rows, 0, dtype=torch.uint8)

    def scale_rows(self, g: int) -> torch.Tensor:
        kp = self.layout.c.seg[g].k_pad
        return self.scales[g][:, :kp // 32] if kp else torch.empty(self.rows, 0, dtype=torch.uint8)


def mxtensor_empty(rows: int, layout: Layout, device="cuda") -> MXTensor:
    cp, cb, sp, sb = mxs_mxtensor_bytes(rows, layout)
    codes, scales = [], []
    c = MXTensorC()
    c.rows = rows
    c.lay = layout.c
    for g in range(3):
        if cb[g] or (layout.c.seg[g].k_pad and rows):
            ct = torch.zeros((rows, cp[g]), dtype=torch.uint8, device=device)
            st = torch.zeros((rows, sp[g]), dtype=torch.uint8, device=device)
        else:
            ct = st = None
        codes.append(ct)
        scales.append(st)
        c.codes[g] = ct.data_ptr() if ct is not None else None
        c.scales[g] = st.data_ptr() if st is not None else None
        c.code_pitch[g] = cp[g]
        c.scale_pitch[g] = sp[g]
    return MXTensor(rows, layout, codes, scales, c)


# ------------------------------------------------------------- sensitivity
def mxs_sensitivity_workspace_bytes(T: int, N: int, K: int) -> int:
    need = _SZ(0)
    _check(_lib.mxs_sensitivity_workspace_bytes(T, N, K, ctypes.byref(need)), "mxs_sensitivity_workspace_bytes")
    return need.value


def mxs_sensitivity(X: torch.Tensor, W: torch.Tensor, stream=None, workspace: Optional[torch.Tensor] = None,
                    out=None):
    """(H, E, s) fp64 device tensors for calibration X (T x K) and weight W (N x K)."""
    T, K = X.shape
    N, K2 = W.shape
    assert K == K2
    need = _SZ(mxs_sensitivity_workspace_bytes(T, N, K))
    ws = workspace if workspace is not None else _workspace(need.value, X.device)
    if out is None:
        H = torch.empty(K, dtype=torch.float64, device=X.device)
        E = torch.empty_like(H)
        s = torch.empty_like(H)
    else:
        H, E, s = out
    _check(_lib.mxs_sensitivity(X.data_ptr(), _dt(X), T, K, _rowmajor(X), W.data_ptr(), _dt(W), N,
                                _rowmajor(W), H.data_ptr(), E.data_ptr(), s.data_ptr(),
                                _aligned_ptr(ws), need.value, _stream(stream)), "mxs_sensitivity")
    return H, E, s


NOALLOC_SCRATCH_BYTES = 16 << 20


def mxs_sensitivity_noalloc(X: torch.Tensor, W: torch.Tensor, out, stream=None):
    """mxs_sensitivity with the library's fixed device scratch instead of a
    workspace; `out` = (H, E, s) caller-allocated fp64 tensors of K."""
    T, K = X.shape
    N, K2 = W.shape
    assert K == K2
    H, E, s = out
    _check(_lib.mxs_sensitivity_noalloc(X.data_ptr(), _dt(X), T, K, _rowmajor(X), W.data_ptr(), _dt(W), N,
                                        _rowmajor(W), H.data_ptr(), E.data_ptr(), s.data_ptr(), _stream(stream)),
           "mxs_sensitivity_noalloc")
    return H, E, s


# --------------------------------------------------------------- allocation
def make_budget(mode: str, budget=(9, 2), p8=(5, 100), p6=(15, 100), fixed8: int = 32) -> BudgetC:
    b = BudgetC()
    b.mode = {"fractions": MXS_ALLOC_FRACTIONS, "budget": MXS_ALLOC_BUDGET, "layer": MXS_ALLOC_LAYER}[mode]
    b.num, b.den = int(budget[0]), int(budget[1])
    b.p8_num, b.p8_den = int(p8[0]), int(p8[1])
    b.p6_num, b.p6_den = int(p6[0]), int(p6[1])
    b.fixed8 = int(fixed8)
    return b


def mxs_allocate(s_list: Sequence[torch.Tensor], N_list: Sequence[int], *, mode: str, budget=(9, 2),
                 p8=(5, 100), p6=(15, 100), fixed8: int = 32, layer_w=None, stream=None,
                 perms: Optional[List[torch.Tensor]] = None, workspace: Optional[torch.Tensor] = None):
    """Returns (perms: list of device int32 tensors, counts: list of (n8, n6, n4)).
    mode: "fractions", "budget" or "layer" (layer_w = the layer scores).
    Synchronises the stream only in multi-layer budget mode."""
    L = len(s_list)
    dev = s_list[0].device
    K = (ctypes.c_int64 * L)(*[int(s.numel()) for s in s_list])
    N = (ctypes.c_int64 * L)(*[int(n) for n in N_list])
    sp = (ctypes.c_void_p * L)(*[s.data_ptr() for s in s_list])
    if perms is None:
        perms = [torch.empty(int(s.numel()), dtype=torch.int32, device=dev) for s in s_list]
    pp = (ctypes.c_void_p * L)(*[p.data_ptr() for p in perms])
    counts = (ctypes.c_int64 * (3 * L))()
    w = None if layer_w is None else (ctypes.c_double * L)(*[float(x) for x in layer_w])
    need = _SZ(0)
    _check(_lib.mxs_allocate_workspace_bytes(L, K, ctypes.byref(need)), "mxs_allocate_workspace_bytes")
    ws = workspace if workspace is not None else _workspace(need.value, dev)
    b = make_budget(mode, budget, p8, p6, fixed8)
    _check(_lib.mxs_allocate(L, K, N, sp, w, ctypes.byref(b), pp, counts, _aligned_ptr(ws), need.value,
                             _stream(stream)), "mxs_allocate")
    return perms, [tuple(counts[3 * l:3 * l + 3]) for l in range(L)]


# --------------------------------------------------------------- quantisers
def _quantize(fn, name, src: torch.Tensor, out: MXTensor, stream):
    _check(fn(src.data_ptr(), _dt(src), src.shape[0], _rowmajor(src), ctypes.byref(out.c), _stream(stream)), name)
    return out


def mxs_quantize_weight(W: torch.Tensor, out: MXTensor, stream=None) -> MXTensor:
    return _quantize(_lib.mxs_quantize_weight, "mxs_quantize_weight", W, out, stream)


def mxs_quantize_act(A: torch.Tensor, out: MXTensor, stream=None) -> MXTensor:
    return _quantize(_lib.mxs_quantize_act, "mxs_quantize_act", A, out, stream)


def mxs_dequantize(t: MXTensor, stream=None) -> torch.Tensor:
    dev = next(x.device for x in t.codes if x is not None)
    out = torch.empty((t.rows, t.layout.K_pad), dtype=torch.float32, device=dev)
    _check(_lib.mxs_dequantize(ctypes.byref(t.c), out.data_ptr(), out.stride(0), _stream(stream)), "mxs_dequantize")
    return out


# -------------------------------------------------------------------- GEMM
def mxs_gemm_workspace_bytes(A: MXTensor, W: MXTensor) -> int:
    need = _SZ(0)
    _check(_lib.mxs_gemm_workspace_bytes(ctypes.byref(A.c), ctypes.byref(W.c), ctypes.byref(need)),
           "mxs_gemm_workspace_bytes")
    return need.value


def mxs_gemm(A: MXTensor, W: MXTensor, Y: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
    dev = next(x.device for x in A.codes if x is not None)
    if Y is None:
        Y = torch.empty((A.rows, W.rows), dtype=torch.bfloat16, device=dev)
    need = mxs_gemm_workspace_bytes(A, W)
    ws = workspace if workspace is not None else _workspace(need, dev)
    _check(_lib.mxs_gemm(ctypes.byref(A.c), ctypes.byref(W.c), Y.data_ptr(), Y.stride(0), _aligned_ptr(ws), need,
                         _stream(stream)), "mxs_gemm")
    return Y


# -------------------------------------------------------- decode attention
def mxs_attn_decode_workspace_bytes(T: int, n_qh: int, n_kvh: int, d: int = 128) -> int:
    need = _SZ(0)
    _check(_lib.mxs_attn_decode_workspace_bytes(T, n_qh, n_kvh, d, ctypes.byref(need)),
           "mxs_attn_decode_workspace_bytes")
    return need.value


def mxs_attn_decode(q: torch.Tensor, K: MXTensor, V: MXTensor, T: int, n_kvh: int, sm_scale: float,
                    out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """fp32 (n_qh x 128) output of one decode step of grouped-query attention
    over the MXINT4 K/V caches K and V (T*n_kvh rows each, token-major)."""
    if q.dtype != torch.bfloat16:
        raise TypeError("q must be bf16")
    n_qh = q.shape[0]
    if out is None:
        out = torch.empty((n_qh, q.shape[1]), dtype=torch.float32, device=q.device)
    need = mxs_attn_decode_workspace_bytes(T, n_qh, n_kvh, q.shape[1])
    ws = workspace if workspace is not None else _workspace(need, q.device)
    _check(_lib.mxs_attn_decode(q.data_ptr(), n_qh, _rowmajor(q), ctypes.byref(K.c), ctypes.byref(V.c), T, n_kvh,
                                float(sm_scale), out.data_ptr(), _rowmajor(out), _aligned_ptr(ws, 256), need,
                                _stream(stream)), "mxs_attn_decode")
    return out


# ---------------------------------------------------------- layer scores
LINEARS = ("q", "k", "v", "o", "gate", "up", "down")


def _stack_c(blocks, hidden, n_heads, n_kv_heads, mlp, rms_eps, rope_theta):
    ptrs = (ctypes.c_void_p * (7 * len(blocks)))()
    for b, Ws in enumerate(blocks):
        for j, w in enumerate(Ws):
            if w.dtype != torch.bfloat16 or not w.is_contiguous():
                raise TypeError("stack weights must be contiguous bf16")
            ptrs[7 * b + j] = w.data_ptr()
    m = StackC(len(blocks), hidden, n_heads, n_kv_heads, mlp, rms_eps, rope_theta,
               ctypes.cast(ptrs, ctypes.c_void_p))
    return m, ptrs


def mxs_layer_scores_workspace_bytes(n_blocks: int, hidden: int, n_heads: int, n_kv_heads: int, mlp: int,
                                     T: int, rms_eps: float = 1e-5, rope_theta: float = 500000.0) -> int:
    m = StackC(n_blocks, hidden, n_heads, n_kv_heads, mlp, rms_eps, rope_theta, ctypes.c_void_p(1 << 20))
    need = _SZ(0)
    _check(_lib.mxs_layer_scores_workspace_bytes(ctypes.byref(m), T, ctypes.byref(need)),
           "mxs_layer_scores_workspace_bytes")
    return need.value


def mxs_layer_scores(x: torch.Tensor, blocks, *, n_heads: int, n_kv_heads: int, rms_eps: float = 1e-5,
                     rope_theta: float = 500000.0, workspace: Optional[torch.Tensor] = None, stream=None):
    """Layer-wise sensitivity scores (7 per block: q, k, v, o, gate, up, down)
    of the decoder stack `blocks` (a list of 7-tuples of bf16 weights) for the
    fp32 hidden states x (T x hidden).  Synchronises the stream."""
    import numpy as np
    T, hidden = x.shape
    mlp = blocks[0][4].shape[0]
    m, ptrs = _stack_c(blocks, hidden, n_heads, n_kv_heads, mlp, rms_eps, rope_theta)
    need = _SZ(0)
    _check(_lib.mxs_layer_scores_workspace_bytes(ctypes.byref(m), T, ctypes.byref(need)),
           "mxs_layer_scores_workspace_bytes")
    ws = workspace if workspace is not None else _workspace(need.value, x.device)
    out = np.zeros(7 * len(blocks))
    if x.dtype != torch.float32:
        raise TypeError("x must be fp32")
    _check(_lib.mxs_layer_scores(ctypes.byref(m), x.data_ptr(), T, _rowmajor(x),
                                 out.ctypes.data_as(ctypes.c_void_p), _aligned_ptr(ws, 256), need.value,
                                 _stream(stream)), "mxs_layer_scores")
    return out


def mxs_sync(stream=None) -> None:
    _check(_lib.mxs_sync(_stream(stream)), "mxs_sync")


def mxs_set_wait_limit(cycles: int) -> None:
    """Diagnostic: the spin limit (SM cycles) of the prefill GEMM kernels'
    pipeline waits on the current device; 0 restores the default."""
    _check(_lib.mxs_set_wait_limit(int(cycles)), "mxs_set_wait_limit")


def mxs_launch_count() -> int:
    return int(_lib.mxs_launch_count())


def mxs_status_str(st: int) -> str:
    return _lib.mxs_status_str(st).decode()
