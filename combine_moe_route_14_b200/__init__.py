"""B200-native MoE layer: route -> layout -> dispatch -> expert FFN -> combine.

A thin Python binding over the C ABI of ``libmoe.so`` (``include/moe.h``).
Functions carry the C names; they check tensor dtypes, shapes and devices,
allocate outputs with torch when none are given, and pass device pointers
and the current CUDA stream.  Every step of the layer runs in the library's
CUDA kernels: there is no CPU or PyTorch fallback, and a missing library is
an error.

Build the library first:  ``python -m combine_moe_route_14_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "MoeError", "LayerDesc", "load_library", "library_path",
    "moe_router_logits", "moe_route", "moe_route_ex", "moe_layout_workspace_size", "moe_layout",
    "moe_layout_static",
    "moe_dispatch", "moe_expert_gemm", "moe_expert_ffn", "moe_combine",
    "moe_workspace_size", "moe_layer_forward", "moe_device_status",
    "moe_kernel_launches_per_forward", "MoeLayer", "SCORES",
    "moe_quantize_experts_fp8", "moe_dispatch_fp8", "moe_expert_gemm_fp8",
    "moe_layer_forward_fp8", "moe_kernel_launches_per_forward_fp8",
    "moe_quantize_fp8", "moe_expert_gemm_gather", "moe_expert_gemm_gather_fp8",
    "moe_expert_ffn_fused_workspace_size", "moe_expert_ffn_fused", "moe_expert_ffn_fused_fp8",
    "moe_selftest_bounded_wait", "moe_dispatch_by_token", "moe_dispatch_fp8_by_token",
    "moe_ffn_pipeline_workspace_size", "moe_ffn_pipeline", "make_desc",
    "moe_host_workspace_size", "moe_layer_forward_host", "moe_route_layout",
    "LAYER_GATHER_ON_LOAD", "LAYER_FUSED_FFN", "LAYER_FUSED_COMBINE", "LAYER_FUSED_DISPATCH",
    "LAYER_PIPELINE",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmoe.so")
_lib = None
_lock = threading.Lock()

SCORES = {"softmax": 0, "sigmoid": 1}
LAYER_GATHER_ON_LOAD = 0x1  # moe_layer_desc.flags: dispatch fused into GEMM-1
LAYER_FUSED_FFN = 0x2       # moe_layer_desc.flags: both expert GEMMs in one persistent launch
LAYER_FUSED_COMBINE = 0x4   # moe_layer_desc.flags: combine in GEMM-2's epilogue (k <= 2)
LAYER_FUSED_DISPATCH = 0x8  # moe_layer_desc.flags: dispatch chunks inside the fused FFN launch
LAYER_PIPELINE = LAYER_FUSED_FFN | LAYER_FUSED_COMBINE | LAYER_FUSED_DISPATCH
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_CUDA",
          4: "MOE_ERR_DEVICE"}
DEV_BITS = {1: "MOE_DEV_BAD_EXPERT_ID", 2: "MOE_DEV_TIMEOUT", 4: "MOE_DEV_BAD_ROW"}


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class LayerDesc(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("f", ctypes.c_int32), ("score", ctypes.c_int32),
                ("renormalize", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("temperature", ctypes.c_float), ("min_prob", ctypes.c_float)]


def library_path() -> str:
    return _LIB_PATH


_P = ctypes.c_void_p
_I = ctypes.c_int32
_SIG = {
    "moe_router_logits": ([_P, _P, _I, _I, _I, _P, _P], ctypes.c_int),
    "moe_route": ([_P, _I, _I, _I, _I, _I, _P, _P, _P], ctypes.c_int),
    "moe_route_ex": ([_P, _I, _I, _I, _I, _I, ctypes.c_float, ctypes.c_float, _P, _P, _P],
                     ctypes.c_int),
    "moe_layout_workspace_size": ([_I, _I, _I], ctypes.c_size_t),
    "moe_layout": ([_P, _I, _I, _I, _P, _P, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "moe_layout_static": ([_P, _I, _I, _I, _P, _P, _P, _P, _P], ctypes.c_int),
    "moe_dispatch": ([_P, _P, _I, _I, _I, _P, _P], ctypes.c_int),
    "moe_dispatch_by_token": ([_P, _P, _I, _I, _I, _P, _P], ctypes.c_int),
    "moe_dispatch_fp8_by_token": ([_P, _P, _I, _I, _I, _P, _P, _P], ctypes.c_int),
    "moe_expert_gemm": ([_P, _P, _P, _I, _I, _I, _I, _I, _P, _P], ctypes.c_int),
    "moe_expert_ffn": ([_P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P], ctypes.c_int),
    "moe_combine": ([_P, _P, _P, _I, _I, _I, _P, _P], ctypes.c_int),
    "moe_workspace_size": ([ctypes.POINTER(LayerDesc)], ctypes.c_size_t),
    "moe_layer_forward": ([ctypes.POINTER(LayerDesc), _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                           ctypes.c_size_t, _P], ctypes.c_int),
    "moe_last_error_string": ([], ctypes.c_char_p),
    "moe_device_status": ([ctypes.POINTER(ctypes.c_uint32), _I], ctypes.c_int),
    "moe_kernel_launches_per_forward": ([ctypes.POINTER(LayerDesc), _I], ctypes.c_int32),
    "moe_quantize_experts_fp8": ([_P, _I, _I, _I, _P, _P, _P], ctypes.c_int),
    "moe_dispatch_fp8": ([_P, _P, _I, _I, _I, _P, _P, _P], ctypes.c_int),
    "moe_expert_gemm_fp8": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P], ctypes.c_int),
    "moe_layer_forward_fp8": ([ctypes.POINTER(LayerDesc), _P, _P, _P, _P, _P, _P, _P, _P, _P,
                               _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "moe_kernel_launches_per_forward_fp8": ([ctypes.POINTER(LayerDesc), _I], ctypes.c_int32),
    "moe_quantize_fp8": ([_P, _I, _I, _P, _P, _P], ctypes.c_int),
    "moe_selftest_bounded_wait": ([_I, ctypes.c_uint32, _P, _P], ctypes.c_int),
    "moe_expert_ffn_fused_workspace_size": ([_I, _I], ctypes.c_size_t),
    "moe_expert_ffn_fused": ([_P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, ctypes.c_size_t, _P],
                             ctypes.c_int),
    "moe_expert_ffn_fused_fp8": ([_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P,
                                  ctypes.c_size_t, _P], ctypes.c_int),
    "moe_route_layout_workspace_size": ([_I, _I], ctypes.c_size_t),
    "moe_route_layout": ([_P, _I, _I, _I, _I, _I, ctypes.c_float, ctypes.c_float, _P, _P, _P, _P,
                          _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "moe_host_workspace_size": ([ctypes.POINTER(LayerDesc), _I], ctypes.c_size_t),
    "moe_layer_forward_host": ([ctypes.POINTER(LayerDesc), _I, _P, _P, _P, _P, _P, _P, _P, _P,
                                ctypes.c_size_t, _P], ctypes.c_int),
    "moe_ffn_pipeline_workspace_size": ([_I, _I, _I, _I, _I], ctypes.c_size_t),
    "moe_ffn_pipeline": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P,
                          ctypes.c_size_t, _P], ctypes.c_int),
    "moe_expert_gemm_gather": ([_P, _P, _I, _I, _P, _P, _I, _I, _I, _I, _P, _P], ctypes.c_int),
    "moe_expert_gemm_gather_fp8": ([_P, _P, _P, _I, _I, _P, _P, _P, _I, _I, _I, _I, _P, _P],
                                   ctypes.c_int),
}


def load_library():
    """Load libmoe.so (raises if it has not been built: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise MoeError(3, f"{_LIB_PATH} is missing; build it with "
                                  "`python -m combine_moe_route_14_b200.build`")
            lib = ctypes.CDLL(_LIB_PATH)
            for name, (args, res) in _SIG.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = res
            _lib = lib
    return _lib


def _check(status: int):
    if status != 0:
        msg = load_library().moe_last_error_string().decode(errors="replace")
        raise MoeError(status, msg)


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t, name, dtype, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must live on a CUDA device")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def _need_host(t, name, dtype, shape):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype or t.device.type != "cpu" or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} CPU tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def _out(t, name, dtype, shape, device):
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    return _need(t, name, dtype, shape, device)


def _score(score) -> int:
    return SCORES[score] if isinstance(score, str) else int(score)


# ----------------------------------------------------------------------------
# stages
# ----------------------------------------------------------------------------
def moe_router_logits(X, Wr, logits=None, stream=None):
    lib = load_library()
    T, d = X.shape
    E = Wr.shape[0]
    dev = X.device
    _need(X, "X", torch.bfloat16, (T, d))
    _need(Wr, "Wr", torch.bfloat16, (E, d), dev)
    logits = _out(logits, "logits", torch.float32, (T, E), dev)
    _check(lib.moe_router_logits(_ptr(X), _ptr(Wr), T, d, E, _ptr(logits), _stream(stream, dev)))
    return logits


def moe_route(logits, k, score="softmax", renormalize=True, topk_idx=None, gates=None,
              stream=None):
    lib = load_library()
    T, E = logits.shape
    dev = logits.device
    _need(logits, "logits", torch.float32, (T, E))
    topk_idx = _out(topk_idx, "topk_idx", torch.int32, (T, k), dev)
    gates = _out(gates, "gates", torch.float32, (T, k), dev)
    _check(lib.moe_route(_ptr(logits), T, E, k, _score(score), int(bool(renormalize)),
                         _ptr(topk_idx), _ptr(gates), _stream(stream, dev)))
    return topk_idx, gates


def moe_route_ex(logits, k, score="softmax", renormalize=True, temperature=1.0, min_prob=0.0,
                 topk_idx=None, gates=None, stream=None):
    """moe_route with a router temperature and a minimum-probability threshold (-1 = dropped)."""
    lib = load_library()
    T, E = logits.shape
    dev = logits.device
    _need(logits, "logits", torch.float32, (T, E))
    topk_idx = _out(topk_idx, "topk_idx", torch.int32, (T, k), dev)
    gates = _out(gates, "gates", torch.float32, (T, k), dev)
    _check(lib.moe_route_ex(_ptr(logits), T, E, k, _score(score), int(bool(renormalize)),
                            float(temperature), float(min_prob), _ptr(topk_idx), _ptr(gates),
                            _stream(stream, dev)))
    return topk_idx, gates


def moe_layout_workspace_size(T, E, k) -> int:
    return int(load_library().moe_layout_workspace_size(T, E, k))


def moe_layout(topk_idx, E, counts=None, offsets=None, row_of=None, src_of=None, ws=None,
               stream=None):
    lib = load_library()
    T, k = topk_idx.shape
    dev = topk_idx.device
    _need(topk_idx, "topk_idx", torch.int32, (T, k))
    R = T * k
    counts = _out(counts, "counts", torch.int32, (E,), dev)
    offsets = _out(offsets, "offsets", torch.int32, (E + 1,), dev)
    row_of = _out(row_of, "row_of", torch.int32, (R,), dev)
    src_of = _out(src_of, "src_of", torch.int32, (R,), dev)
    need = moe_layout_workspace_size(T, E, k)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _need(ws, "ws", torch.uint8, None, dev)
    _check(lib.moe_layout(_ptr(topk_idx), T, E, k, _ptr(counts), _ptr(offsets), _ptr(row_of),
                          _ptr(src_of), _ptr(ws), ws.numel(), _stream(stream, dev)))
    return counts, offsets, row_of, src_of


def moe_layout_static(topk_idx, E, counts=None, offsets=None, row_of=None, src_of=None,
                      stream=None):
    """moe_layout with the scratch kept in the library's own static device array.

    For callers that cannot allocate device memory for a workspace; see
    include/moe.h.  Calls that may overlap on the GPU race on the shared array.
    """
    lib = load_library()
    T, k = topk_idx.shape
    dev = topk_idx.device
    _need(topk_idx, "topk_idx", torch.int32, (T, k))
    R = T * k
    counts = _out(counts, "counts", torch.int32, (E,), dev)
    offsets = _out(offsets, "offsets", torch.int32, (E + 1,), dev)
    row_of = _out(row_of, "row_of", torch.int32, (R,), dev)
    src_of = _out(src_of, "src_of", torch.int32, (R,), dev)
    _check(lib.moe_layout_static(_ptr(topk_idx), T, E, k, _ptr(counts), _ptr(offsets),
                                 _ptr(row_of), _ptr(src_of), _stream(stream, dev)))
    return counts, offsets, row_of, src_of


def moe_dispatch(X, src_of, k, Xe=None, stream=None):
    lib = load_library()
    T, d = X.shape
    dev = X.device
    _need(X, "X", torch.bfloat16, (T, d))
    _need(src_of, "src_of", torch.int32, (T * k,), dev)
    Xe = _out(Xe, "Xe", torch.bfloat16, (T * k, d), dev)
    _check(lib.moe_dispatch(_ptr(X), _ptr(src_of), T, d, k, _ptr(Xe), _stream(stream, dev)))
    return Xe


def moe_dispatch_by_token(X, row_of, k, Xe=None, stream=None):
    """moe_dispatch walked by token: Xe[row_of[t*k+j]] = X[t] (each token read once)."""
    lib = load_library()
    T, d = X.shape
    dev = X.device
    _need(X, "X", torch.bfloat16, (T, d))
    _need(row_of, "row_of", torch.int32, (T * k,), dev)
    Xe = _out(Xe, "Xe", torch.bfloat16, (T * k, d), dev)
    _check(lib.moe_dispatch_by_token(_ptr(X), _ptr(row_of), T, d, k, _ptr(Xe),
                                     _stream(stream, dev)))
    return Xe


def moe_dispatch_fp8_by_token(X, row_of, k, Xeq=None, x_scale=None, stream=None):
    lib = load_library()
    T, d = X.shape
    dev = X.device
    _need(X, "X", torch.bfloat16, (T, d))
    _need(row_of, "row_of", torch.int32, (T * k,), dev)
    Xeq = _out(Xeq, "Xeq", torch.uint8, (T * k, d), dev)
    x_scale = _out(x_scale, "x_scale", torch.float32, (2,), dev)
    _check(lib.moe_dispatch_fp8_by_token(_ptr(X), _ptr(row_of), T, d, k, _ptr(Xeq),
                                         _ptr(x_scale), _stream(stream, dev)))
    return Xeq, x_scale


def moe_expert_gemm(A, offsets, W, gelu, out=None, stream=None):
    lib = load_library()
    R, K = A.shape
    E, N, K2 = W.shape
    dev = A.device
    if K2 != K:
        raise ValueError("W's last dim must equal A's")
    _need(A, "A", torch.bfloat16, (R, K))
    _need(offsets, "offsets", torch.int32, (E + 1,), dev)
    _need(W, "W", torch.bfloat16, (E, N, K), dev)
    out = _out(out, "out", torch.bfloat16, (R, N), dev)
    _check(lib.moe_expert_gemm(_ptr(A), _ptr(offsets), _ptr(W), E, R, N, K, int(bool(gelu)),
                               _ptr(out), _stream(stream, dev)))
    return out


def moe_expert_ffn(Xe, offsets, W1, W2, H=None, Ye=None, stream=None):
    lib = load_library()
    R, d = Xe.shape
    E, f, _ = W1.shape
    dev = Xe.device
    _need(Xe, "Xe", torch.bfloat16, (R, d))
    _need(offsets, "offsets", torch.int32, (E + 1,), dev)
    _need(W1, "W1", torch.bfloat16, (E, f, d), dev)
    _need(W2, "W2", torch.bfloat16, (E, d, f), dev)
    H = _out(H, "H", torch.bfloat16, (R, f), dev)
    Ye = _out(Ye, "Ye", torch.bfloat16, (R, d), dev)
    _check(lib.moe_expert_ffn(_ptr(Xe), _ptr(offsets), _ptr(W1), _ptr(W2), E, R, d, f, _ptr(H),
                              _ptr(Ye), _stream(stream, dev)))
    return H, Ye


def moe_expert_ffn_fused_workspace_size(E, R) -> int:
    return int(load_library().moe_expert_ffn_fused_workspace_size(E, R))


def moe_expert_ffn_fused(Xe, offsets, W1, W2, H=None, Ye=None, ws=None, stream=None):
    """moe_expert_ffn as one persistent kernel (GEMM-2 starts per token block)."""
    lib = load_library()
    R, d = Xe.shape
    E, f, _ = W1.shape
    dev = Xe.device
    _need(Xe, "Xe", torch.bfloat16, (R, d))
    _need(offsets, "offsets", torch.int32, (E + 1,), dev)
    _need(W1, "W1", torch.bfloat16, (E, f, d), dev)
    _need(W2, "W2", torch.bfloat16, (E, d, f), dev)
    H = _out(H, "H", torch.bfloat16, (R, f), dev)
    Ye = _out(Ye, "Ye", torch.bfloat16, (R, d), dev)
    if ws is None:
        ws = torch.empty(max(moe_expert_ffn_fused_workspace_size(E, R), 16), dtype=torch.uint8,
                         device=dev)
    _need(ws, "ws", torch.uint8, None, dev)
    _check(lib.moe_expert_ffn_fused(_ptr(Xe), _ptr(offsets), _ptr(W1), _ptr(W2), E, R, d, f,
                                    _ptr(H), _ptr(Ye), _ptr(ws), ws.numel(), _stream(stream, dev)))
    return H, Ye


def moe_expert_ffn_fused_fp8(Xeq, x_scale, offsets, W1q, w1_scale, W2, H=None, Ye=None, ws=None,
                             stream=None):
    lib = load_library()
    R, d = Xeq.shape
    E, f, _ = W1q.shape
    dev = Xeq.device
    _need(Xeq, "Xeq", torch.uint8, (R, d))
    if x_scale.dtype != torch.float32 or x_scale.device != dev or x_scale.numel() < 1:
        raise ValueError("x_scale must be a float32 device tensor")
    _need(offsets, "offsets", torch.int32, (E + 1,), dev)
    _need(W1q, "W1q", torch.uint8, (E, f, d), dev)
    _need(w1_scale, "w1_scale", torch.float32, (E,), dev)
    _need(W2, "W2", torch.bfloat16, (E, d, f), dev)
    H = _out(H, "H", torch.bfloat16, (R, f), dev)
    Ye = _out(Ye, "Ye", torch.bfloat16, (R, d), dev)
    if ws is None:
        ws = torch.empty(max(moe_expert_ffn_fused_workspace_size(E, R), 16), dtype=torch.uint8,
                         device=dev)
    _need(ws, "ws", torch.uint8, None, dev)
    _check(lib.moe_expert_ffn_fused_fp8(_ptr(Xeq), _ptr(x_scale), _ptr(offsets), _ptr(W1q),
                                        _ptr(w1_scale), _ptr(W2), E, R, d, f, _ptr(H), _ptr(Ye),
                                        _ptr(ws), ws.numel(), _stream(stream, dev)))
    return H, Ye


def moe_combine(Ye, row_of, gates, Y=None, stream=None):
    lib = load_library()
    T, k = gates.shape
    R, d = Ye.shape
    dev = Ye.device
    if R != T * k:
        raise ValueError("Ye must have T*k rows")
    _need(Ye, "Ye", torch.bfloat16, (R, d))
    _need(row_of, "row_of", torch.int32, (R,), dev)
    _need(gates, "gates", torch.float32, (T, k), dev)
    Y = _out(Y, "Y", torch.bfloat16, (T, d), dev)
    _check(lib.moe_combine(_ptr(Ye), _ptr(row_of), _ptr(gates), T, d, k, _ptr(Y),
                           _stream(stream, dev)))
    return Y


def moe_ffn_pipeline_workspace_size(T, d, E, k, f) -> int:
    return int(load_library().moe_ffn_pipeline_workspace_size(T, d, E, k, f))


def moe_ffn_pipeline(X, src_of, row_of, gates, offsets, W1, W2, Y=None, ws=None, stream=None):
    """Dispatch, GEMM-1 + GELU, GEMM-2 and (k <= 2) the combine in one persistent launch."""
    lib = load_library()
    T, d = X.shape
    E, f, _ = W1.shape
    k = gates.shape[1]
    dev = X.device
    _need(X, "X", torch.bfloat16, (T, d))
    _need(src_of, "src_of", torch.int32, (T * k,), dev)
    _need(row_of, "row_of", torch.int32, (T * k,), dev)
    _need(gates, "gates", torch.float32, (T, k), dev)
    _need(offsets, "offsets", torch.int32, (E + 1,), dev)
    _need(W1, "W1", torch.bfloat16, (E, f, d), dev)
    _need(W2, "W2", torch.bfloat16, (E, d, f), dev)
    Y = _out(Y, "Y", torch.bfloat16, (T, d), dev)
    if ws is None:
        ws = torch.empty(max(moe_ffn_pipeline_workspace_size(T, d, E, k, f), 16),
                         dtype=torch.uint8, device=dev)
    _need(ws, "ws", torch.uint8, None, dev)
    _check(lib.moe_ffn_pipeline(_ptr(X), _ptr(src_of), _ptr(row_of), _ptr(gates), _ptr(offsets),
                                _ptr(W1), _ptr(W2), T, d, E, k, f, _ptr(Y), _ptr(ws), ws.numel(),
                                _stream(stream, dev)))
    return Y


# ----------------------------------------------------------------------------
# whole layer
# ----------------------------------------------------------------------------
def make_desc(T, d, E, k, f, score="softmax", renormalize=True, temperature=1.0,
              min_prob=0.0, gather_on_load=False, fused_ffn=False, fused_combine=False,
              fused_dispatch=False, pipeline=False) -> LayerDesc:
    """pipeline=True sets fused_ffn, fused_combine and fused_dispatch together."""
    flags = ((LAYER_GATHER_ON_LOAD if gather_on_load else 0) |
             (LAYER_FUSED_FFN if fused_ffn else 0) |
             (LAYER_FUSED_COMBINE if fused_combine else 0) |
             (LAYER_FUSED_DISPATCH if fused_dispatch else 0) |
             (LAYER_PIPELINE if pipeline else 0))
    return LayerDesc(T, d, E, k, f, _score(score), int(bool(renormalize)), flags,
                     float(temperature), float(min_prob))


def moe_workspace_size(desc: LayerDesc) -> int:
    return int(load_library().moe_workspace_size(ctypes.byref(desc)))


def moe_kernel_launches_per_forward(desc: LayerDesc, with_router: bool) -> int:
    return int(load_library().moe_kernel_launches_per_forward(ctypes.byref(desc),
                                                              int(bool(with_router))))


def moe_layer_forward(X, W1, W2, k, score="softmax", renormalize=True, logits=None, Wr=None,
                      Y=None, topk_idx_out=None, gates_out=None, counts_out=None, ws=None,
                      stream=None, temperature=1.0, min_prob=0.0, gather_on_load=False,
                      fused_ffn=False, fused_combine=False, fused_dispatch=False,
                      pipeline=False):
    lib = load_library()
    T, d = X.shape
    E, f, _ = W1.shape
    dev = X.device
    _need(X, "X", torch.bfloat16, (T, d))
    _need(W1, "W1", torch.bfloat16, (E, f, d), dev)
    _need(W2, "W2", torch.bfloat16, (E, d, f), dev)
    if logits is not None:
        _need(logits, "logits", torch.float32, (T, E), dev)
    if Wr is not None:
        _need(Wr, "Wr", torch.bfloat16, (E, d), dev)
    Y = _out(Y, "Y", torch.bfloat16, (T, d), dev)
    if topk_idx_out is not None:
        _need(topk_idx_out, "topk_idx_out", torch.int32, (T, k), dev)
    if gates_out is not None:
        _need(gates_out, "gates_out", torch.float32, (T, k), dev)
    if counts_out is not None:
        _need(counts_out, "counts_out", torch.int32, (E,), dev)
    desc = make_desc(T, d, E, k, f, score, renormalize, temperature, min_prob, gather_on_load,
                     fused_ffn, fused_combine, fused_dispatch, pipeline)
    if ws is None:
        ws = torch.empty(max(moe_workspace_size(desc), 16), dtype=torch.uint8, device=dev)
    _need(ws, "ws", torch.uint8, None, dev)
    _check(lib.moe_layer_forward(ctypes.byref(desc), _ptr(X), _ptr(logits), _ptr(Wr), _ptr(W1),
                                 _ptr(W2), _ptr(Y), _ptr(topk_idx_out), _ptr(gates_out),
                                 _ptr(counts_out), _ptr(ws), ws.numel(), _stream(stream, dev)))
    return Y


# ----------------------------------------------------------------------------
# FP8 (E4M3) mode: codes are torch.uint8 tensors, scales fp32
# ----------------------------------------------------------------------------
def moe_quantize_experts_fp8(W, Wq=None, scales=None, stream=None):
    """Per-expert E4M3 quantisation of bf16 expert weights [E, rows, cols]."""
    lib = load_library()
    E, rows, cols = W.shape
    dev = W.device
    _need(W, "W", torch.bfloat16, (E, rows, cols))
    Wq = _out(Wq, "Wq", torch.uint8, (E, rows, cols), dev)
    scales = _out(scales, "scales", torch.float32, (E,), dev)
    _check(lib.moe_quantize_experts_fp8(_ptr(W), E, rows, cols, _ptr(Wq), _ptr(scales),
                                        _stream(stream, dev)))
    return Wq, scales


def moe_dispatch_fp8(X, src_of, k, Xeq=None, x_scale=None, stream=None):
    """Quantising dispatch; returns (Xeq uint8 [T*k, d], x_scale fp32 [2] = [scale, amax])."""
    lib = load_library()
    T, d = X.shape
    dev = X.device
    _need(X, "X", torch.bfloat16, (T, d))
    _need(src_of, "src_of", torch.int32, (T * k,), dev)
    Xeq = _out(Xeq, "Xeq", torch.uint8, (T * k, d), dev)
    x_scale = _out(x_scale, "x_scale", torch.float32, (2,), dev)
    _check(lib.moe_dispatch_fp8(_ptr(X), _ptr(src_of), T, d, k, _ptr(Xeq), _ptr(x_scale),
                                _stream(stream, dev)))
    return Xeq, x_scale


def moe_expert_gemm_fp8(Aq, a_scale, offsets, Wq, w_scale, gelu, out=None, stream=None):
    lib = load_library()
    R, K = Aq.shape
    E, N, K2 = Wq.shape
    dev = Aq.device
    if K2 != K:
        raise ValueError("Wq's last dim must equal Aq's")
    _need(Aq, "Aq", torch.uint8, (R, K))
    if a_scale.dtype != torch.float32 or a_scale.device != dev or a_scale.numel() < 1:
        raise ValueError("a_scale must be a float32 device tensor")
    _need(offsets, "offsets", torch.int32, (E + 1,), dev)
    _need(Wq, "Wq", torch.uint8, (E, N, K), dev)
    _need(w_scale, "w_scale", torch.float32, (E,), dev)
    out = _out(out, "out", torch.bfloat16, (R, N), dev)
    _check(lib.moe_expert_gemm_fp8(_ptr(Aq), _ptr(a_scale), _ptr(offsets), _ptr(Wq),
                                   _ptr(w_scale), E, R, N, K, int(bool(gelu)), _ptr(out),
                                   _stream(stream, dev)))
    return out


def moe_quantize_fp8(X, Xq=None, x_scale=None, stream=None):
    """Per-tensor E4M3 quantisation of a bf16 matrix; returns (Xq uint8, x_scale [scale, amax])."""
    lib = load_library()
    rows, cols = X.shape
    dev = X.device
    _need(X, "X", torch.bfloat16, (rows, cols))
    Xq = _out(Xq, "Xq", torch.uint8, (rows, cols), dev)
    x_scale = _out(x_scale, "x_scale", torch.float32, (2,), dev)
    _check(lib.moe_quantize_fp8(_ptr(X), rows, cols, _ptr(Xq), _ptr(x_scale),
                                _stream(stream, dev)))
    return Xq, x_scale


def moe_expert_gemm_gather(X, src_of, k, offsets, W, gelu, out=None, stream=None):
    """Grouped GEMM whose row r reads token src_of[r] // k of X directly (no dispatched copy)."""
    lib = load_library()
    T, K = X.shape
    E, N, K2 = W.shape
    dev = X.device
    if K2 != K:
        raise ValueError("W's last dim must equal X's")
    _need(X, "X", torch.bfloat16, (T, K))
    _need(src_of, "src_of", torch.int32, (T * k,), dev)
    _need(offsets, "offsets", torch.int32, (E + 1,), dev)
    _need(W, "W", torch.bfloat16, (E, N, K), dev)
    out = _out(out, "out", torch.bfloat16, (T * k, N), dev)
    _check(lib.moe_expert_gemm_gather(_ptr(X), _ptr(src_of), T, k, _ptr(offsets), _ptr(W), E, N,
                                      K, int(bool(gelu)), _ptr(out), _stream(stream, dev)))
    return out


def moe_expert_gemm_gather_fp8(Xq, x_scale, src_of, k, offsets, Wq, w_scale, gelu, out=None,
                               stream=None):
    lib = load_library()
    T, K = Xq.shape
    E, N, K2 = Wq.shape
    dev = Xq.device
    if K2 != K:
        raise ValueError("Wq's last dim must equal Xq's")
    _need(Xq, "Xq", torch.uint8, (T, K))
    if x_scale.dtype != torch.float32 or x_scale.device != dev or x_scale.numel() < 1:
        raise ValueError("x_scale must be a float32 device tensor")
    _need(src_of, "src_of", torch.int32, (T * k,), dev)
    _need(offsets, "offsets", torch.int32, (E + 1,), dev)
    _need(Wq, "Wq", torch.uint8, (E, N, K), dev)
    _need(w_scale, "w_scale", torch.float32, (E,), dev)
    out = _out(out, "out", torch.bfloat16, (T * k, N), dev)
    _check(lib.moe_expert_gemm_gather_fp8(_ptr(Xq), _ptr(x_scale), _ptr(src_of), T, k,
                                          _ptr(offsets), _ptr(Wq), _ptr(w_scale), E, N, K,
                                          int(bool(gelu)), _ptr(out), _stream(stream, dev)))
    return out


def moe_kernel_launches_per_forward_fp8(desc: LayerDesc, with_router: bool) -> int:
    return int(load_library().moe_kernel_launches_per_forward_fp8(ctypes.byref(desc),
                                                                  int(bool(with_router))))


def moe_layer_forward_fp8(X, W1q, w1_scale, W2, k, score="softmax", renormalize=True,
                          logits=None, Wr=None, Y=None, topk_idx_out=None, gates_out=None,
                          counts_out=None, ws=None, stream=None, temperature=1.0, min_prob=0.0,
                          gather_on_load=False, fused_ffn=False, fused_combine=False,
                          fused_dispatch=False, pipeline=False):
    """The layer with FP8 dispatch and FP8 GEMM-1 (W1q, w1_scale from moe_quantize_experts_fp8)."""
    lib = load_library()
    T, d = X.shape
    E, f, _ = W1q.shape
    dev = X.device
    _need(X, "X", torch.bfloat16, (T, d))
    _need(W1q, "W1q", torch.uint8, (E, f, d), dev)
    _need(w1_scale, "w1_scale", torch.float32, (E,), dev)
    _need(W2, "W2", torch.bfloat16, (E, d, f), dev)
    if logits is not None:
        _need(logits, "logits", torch.float32, (T, E), dev)
    if Wr is not None:
        _need(Wr, "Wr", torch.bfloat16, (E, d), dev)
    Y = _out(Y, "Y", torch.bfloat16, (T, d), dev)
    if topk_idx_out is not None:
        _need(topk_idx_out, "topk_idx_out", torch.int32, (T, k), dev)
    if gates_out is not None:
        _need(gates_out, "gates_out", torch.float32, (T, k), dev)
    if counts_out is not None:
        _need(counts_out, "counts_out", torch.int32, (E,), dev)
    desc = make_desc(T, d, E, k, f, score, renormalize, temperature, min_prob, gather_on_load,
                     fused_ffn, fused_combine, fused_dispatch, pipeline)
    if ws is None:
        ws = torch.empty(max(moe_workspace_size(desc), 16), dtype=torch.uint8, device=dev)
    _need(ws, "ws", torch.uint8, None, dev)
    _check(lib.moe_layer_forward_fp8(ctypes.byref(desc), _ptr(X), _ptr(logits), _ptr(Wr),
                                     _ptr(W1q), _ptr(w1_scale), _ptr(W2), _ptr(Y),
                                     _ptr(topk_idx_out), _ptr(gates_out), _ptr(counts_out),
                                     _ptr(ws), ws.numel(), _stream(stream, dev)))
    return Y


def moe_route_layout(logits, k, score="softmax", renormalize=True, temperature=1.0,
                     min_prob=0.0, out=None, ws=None, stream=None):
    """Routing and layout in one pass (C ABI moe_route_layout).

    out: optional (topk_idx, gates, counts, offsets, row_of, src_of) tensors to
    fill.  Returns that tuple."""
    lib = load_library()
    T, E = logits.shape
    dev = logits.device
    _need(logits, "logits", torch.float32, (T, E))
    i32 = dict(dtype=torch.int32, device=dev)
    if out is None:
        out = (torch.empty((T, k), **i32), torch.empty((T, k), dtype=torch.float32, device=dev),
               torch.empty((E,), **i32), torch.empty((E + 1,), **i32),
               torch.empty((T * k,), **i32), torch.empty((T * k,), **i32))
    idx, gates, counts, offsets, row_of, src_of = out
    for t, n, dt, shp in ((idx, "topk_idx", torch.int32, (T, k)),
                          (gates, "gates", torch.float32, (T, k)),
                          (counts, "counts", torch.int32, (E,)),
                          (offsets, "offsets", torch.int32, (E + 1,)),
                          (row_of, "row_of", torch.int32, (T * k,)),
                          (src_of, "src_of", torch.int32, (T * k,))):
        _need(t, n, dt, shp, dev)
    if ws is None:
        ws = torch.empty(max(16, int(lib.moe_route_layout_workspace_size(T, E))),
                         dtype=torch.uint8, device=dev)
    _need(ws, "ws", torch.uint8, None, dev)
    _check(lib.moe_route_layout(_ptr(logits), T, E, k, _score(score), int(bool(renormalize)),
                                float(temperature), float(min_prob), _ptr(idx), _ptr(gates),
                                _ptr(counts), _ptr(offsets), _ptr(row_of), _ptr(src_of), _ptr(ws),
                                ws.numel(), _stream(stream, dev)))
    return idx, gates, counts, offsets, row_of, src_of


def moe_host_workspace_size(desc: LayerDesc, with_logits: bool) -> int:
    return int(load_library().moe_host_workspace_size(ctypes.byref(desc), int(bool(with_logits))))


def moe_layer_forward_host(X_host, W1, W2, k, Y_host, score="softmax", renormalize=True,
                           logits_host=None, Wr=None, w1_scale=None, ws=None, stream=None,
                           temperature=1.0, min_prob=0.0, **flags):
    """The layer over len(X_host) batches in host memory (C ABI moe_layer_forward_host).

    X_host / Y_host: lists of [T, d] bf16 CPU tensors (pinned for overlap);
    logits_host: a list of [T, E] fp32 CPU tensors, or None with Wr given.
    W1 holds E4M3 codes when w1_scale is given (FP8 mode).  Returns once the
    work is enqueued; `stream` (default: the current one) waits for the last
    copy out."""
    lib = load_library()
    n = len(X_host)
    if len(Y_host) != n or (logits_host is not None and len(logits_host) != n):
        raise ValueError("one output (and logits) tensor per batch")
    T, d = X_host[0].shape
    E, f, _ = W1.shape
    dev = W1.device
    for i in range(n):
        _need_host(X_host[i], f"X_host[{i}]", torch.bfloat16, (T, d))
        _need_host(Y_host[i], f"Y_host[{i}]", torch.bfloat16, (T, d))
        if logits_host is not None:
            _need_host(logits_host[i], f"logits_host[{i}]", torch.float32, (T, E))
    _need(W1, "W1", torch.uint8 if w1_scale is not None else torch.bfloat16, (E, f, d))
    _need(W2, "W2", torch.bfloat16, (E, d, f), dev)
    if Wr is not None:
        _need(Wr, "Wr", torch.bfloat16, (E, d), dev)
    if w1_scale is not None:
        _need(w1_scale, "w1_scale", torch.float32, (E,), dev)
    desc = make_desc(T, d, E, k, f, score, renormalize, temperature, min_prob, **flags)
    if ws is None:
        ws = torch.empty(max(moe_host_workspace_size(desc, logits_host is not None), 16),
                         dtype=torch.uint8, device=dev)
    _need(ws, "ws", torch.uint8, None, dev)
    arr = lambda ts: (ctypes.c_void_p * n)(*[t.data_ptr() for t in ts])  # noqa: E731
    _check(lib.moe_layer_forward_host(ctypes.byref(desc), n, arr(X_host),
                                      None if logits_host is None else arr(logits_host),
                                      _ptr(Wr), _ptr(W1), _ptr(w1_scale), _ptr(W2), arr(Y_host),
                                      _ptr(ws), ws.numel(), _stream(stream, dev)))


def moe_selftest_bounded_wait(which: int, limit_us: int, counter=None, stream=None):
    """Run one bounded device wait that times out (0: readiness counts, 1: ring mbarrier,
    2: combine flag bit, 3: work-item queue mbarrier, cluster scope)."""
    lib = load_library()
    dev = counter.device if counter is not None else torch.device("cuda", torch.cuda.current_device())
    if counter is not None:
        _need(counter, "counter", torch.int32, (1,), dev)
    _check(lib.moe_selftest_bounded_wait(int(which), int(limit_us), _ptr(counter),
                                         _stream(stream, dev)))


def moe_device_status(clear: bool = True) -> int:
    """Synchronise the current device and return its sticky MOE_DEV_* bits."""
    lib = load_library()
    bits = ctypes.c_uint32(0)
    st = lib.moe_device_status(ctypes.byref(bits), int(bool(clear)))
    if st not in (0, 4):
        _check(st)
    return int(bits.value)


class MoeLayer:
    """A layer's weights plus a reusable workspace (allocation stays outside the call)."""

    def __init__(self, W1, W2, k, score="softmax", renormalize=True, Wr=None, temperature=1.0,
                 min_prob=0.0, fp8=False, gather_on_load=False, fused_ffn=False,
                 fused_combine=False, fused_dispatch=False, pipeline=False):
        self.W1, self.W2, self.Wr = W1, W2, Wr
        self.fp8 = bool(fp8)
        self.flags = dict(gather_on_load=bool(gather_on_load), fused_ffn=bool(fused_ffn),
                          fused_combine=bool(fused_combine), fused_dispatch=bool(fused_dispatch),
                          pipeline=bool(pipeline))
        # FP8 mode keeps W1 as E4M3 codes with per-expert scales (quantised once here)
        self.W1q, self.w1_scale = moe_quantize_experts_fp8(W1) if self.fp8 else (None, None)
        self.k, self.score, self.renormalize = k, score, renormalize
        self.temperature, self.min_prob = temperature, min_prob
        self.E, self.f, self.d = W1.shape
        self._ws = None

    def workspace(self, T):
        desc = make_desc(T, self.d, self.E, self.k, self.f, self.score, self.renormalize)
        need = max(moe_workspace_size(desc), 16)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.W1.device)
        return self._ws

    def __call__(self, X, logits=None, Y=None, topk_idx_out=None, gates_out=None,
                 counts_out=None, stream=None):
        kw = dict(logits=logits, Wr=None if logits is not None else self.Wr, Y=Y,
                  topk_idx_out=topk_idx_out, gates_out=gates_out, counts_out=counts_out,
                  ws=self.workspace(X.shape[0]), stream=stream, temperature=self.temperature,
                  min_prob=self.min_prob, **self.flags)
        if self.fp8:
            return moe_layer_forward_fp8(X, self.W1q, self.w1_scale, self.W2, self.k, self.score,
                                         self.renormalize, **kw)
        return moe_layer_forward(X, self.W1, self.W2, self.k, self.score, self.renormalize, **kw)


from .pipeline import HostPipeline  # noqa: E402  (stream plumbing for host-buffer batches)

__all__.append("HostPipeline")
