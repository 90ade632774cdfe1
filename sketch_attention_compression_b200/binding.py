"""ctypes binding of libsa.so (argument marshalling only).

Every step of the SA layer runs in the CUDA library; this module turns torch
tensors and streams into the plain pointers and sizes of the C ABI declared
in include/sa.h.  PyTorch provides device memory and streams.  There is no
fallback: if libsa.so is missing or a call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libsa.so")

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_WORKSPACE, SA_ERR_CUDA, \
    SA_ERR_DEVICE_FLAG = range(6)
SA_BF16, SA_FP32 = 0, 1
DEVFLAG_OFFSET0_NONZERO, DEVFLAG_OFFSETS_DECREASE, DEVFLAG_OFFSET_LAST, DEVFLAG_TIMEOUT, \
    DEVFLAG_SMEM_ALIGN, DEVFLAG_ACTION_TYPE = 1, 2, 4, 8, 16, 32

# name -> (restype, argtypes); mirrors include/sa.h
_vp, _i32, _i64, _sz, _f32, _f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, \
    ctypes.c_size_t, ctypes.c_float, ctypes.c_double
_FWD_ARGS = [_vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _sz, _vp]
SIGNATURES = {
    "sa_prepare_query": (_i32, [_vp, _vp, _vp, _i32, _i32, _f32, _i32, _vp,
                                ctypes.POINTER(_vp)]),
    "sa_sketch_free": (None, [_vp]),
    "sa_workspace_bytes": (_sz, [_vp, _i64, _i64]),
    "sa_sketch_forward": (_i32, _FWD_ARGS),
    "sa_sketch_partials": (_i32, _FWD_ARGS),
    "sa_sketch_finalize": (_i32, _FWD_ARGS),
    "sa_workspace_bytes_user_queries": (_sz, [_vp, _i64, _i64]),
    "sa_sketch_forward_user_queries": (_i32, [_vp, _vp] + _FWD_ARGS[1:]),
    "sa_sketch_partials_user_queries": (_i32, [_vp, _vp] + _FWD_ARGS[1:]),
    "sa_host_path_device_bytes": (_sz, [_vp, _i64, _i64]),
    "sa_sketch_forward_host": (_i32, _FWD_ARGS),
    "sa_sketch_forward_noalloc": (_i32, [_vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp]),
    "sa_read_device_status": (_i32, [_vp, _sz, _vp, ctypes.POINTER(ctypes.c_uint32)]),
    "sa_mass_normalise": (_i32, [_vp, _vp, _i64, _i32, _i32, _vp, _vp]),
    "sa_status_string": (ctypes.c_char_p, [_i32]),
    "sa_query_info": (_i32, [_vp, ctypes.POINTER(_i32), ctypes.POINTER(_i32),
                             ctypes.POINTER(_i32), ctypes.POINTER(_i32)]),
    "sa_workspace_bytes_backward": (_sz, [_vp, _i64, _i64]),
    "sa_sketch_backward": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp,
                                  _vp, _vp, _vp, _vp, _sz, _vp]),
    "sa_prepare_refine": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp,
                                 ctypes.POINTER(_vp)]),
    "sa_refine_free": (None, [_vp]),
    "sa_refine_update": (_i32, [_vp, _vp, _i32, _vp, _vp, _i64, _i32, _vp, _vp, _vp]),
    "sa_workspace_bytes_refine_layer": (_sz, [_vp, _i64, _i64]),
    "sa_refine_layer_forward": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _vp, _vp, _sz,
                                       _vp]),
    "sa_workspace_bytes_refine_stack": (_sz, [_vp, _i64, _i64]),
    "sa_refine_stack_forward": (_i32, [_i32, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _vp, _vp, _sz,
                                       _vp]),
    "sa_cache_create": (_i32, [_i32, _i32, _i64, _f64, ctypes.POINTER(_vp)]),
    "sa_cache_free": (None, [_vp]),
    "sa_cache_lookup": (_i32, [_vp, _vp, _i64, _f64, _vp, _vp, _vp, _vp]),
    "sa_cache_insert": (_i32, [_vp, _vp, _i64, _f64, _vp, _vp, _vp]),
    "sa_cache_stats": (_i32, [_vp, _vp, _vp, _vp, _vp]),
    "sa_cache_forward_workspace_bytes": (_sz, [_vp, _i64, _i64]),
    "sa_cache_forward": (_i32, [_vp, _vp, _vp, _f64, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _sz,
                                _vp]),
    "sa_prepare_adapter": (_i32, [_vp, _i32, _i32, _vp, ctypes.POINTER(_vp)]),
    "sa_adapter_free": (None, [_vp]),
    "sa_adapter_forward": (_i32, [_vp, _vp, _i64, _vp, _vp, _vp]),
    "sa_prepare_action": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp,
                                 ctypes.POINTER(_vp)]),
    "sa_action_free": (None, [_vp]),
    "sa_action_fuse": (_i32, [_vp, _vp, _vp, _i64, _vp, _vp, _vp]),
    "sa_workspace_bytes_action_sketch": (_sz, [_vp, _i64, _i64]),
    "sa_action_sketch_forward": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _sz,
                                        _vp]),
}


class CacheKey(ctypes.Structure):
    """sa_cache_key: the cache key of section 2.4 (user, model version,
    history timestamp, sketch configuration)."""
    _fields_ = [("user", ctypes.c_int64), ("model_version", ctypes.c_int64),
                ("history_ts", ctypes.c_int64), ("config", ctypes.c_int64)]


def _keys_array(keys):
    """The keys as a C-contiguous (n, 4) int64 array: the memory layout of n
    sa_cache_key structs (user, model_version, history_ts, config).  Accepts
    such an array as is, or any sequence of 4-tuples."""
    arr = np.ascontiguousarray(keys, dtype=np.int64).reshape(-1, 4)
    if arr.shape[0] == 0:
        arr = np.zeros((1, 4), dtype=np.int64)
    return arr

_lib: Optional[ctypes.CDLL] = None


class SAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libsa.so (built in-tree) and declares its signatures."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m sketch_attention_compression_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    try:
        return load_library().sa_status_string(status).decode()
    except Exception:  # pragma: no cover - only for messages
        return "unknown"


def _check(status: int, what: str) -> None:
    if status != SA_OK:
        raise SAError(status, what)


def _torch():
    import torch  # deferred: the binding is importable without torch for the ABI checks
    return torch


def _stream_handle(stream) -> int:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t) -> int:
    torch = _torch()
    if t == torch.bfloat16:
        return SA_BF16
    if t == torch.float32:
        return SA_FP32
    raise TypeError(f"unsupported dtype {t}; use torch.bfloat16 or torch.float32")


def _dev_ptr(t, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


class SketchQuery:
    """A prepared SA query: Q' = P W_Q W_K^T * scale for one weight set.

    P (k, d), W_Q and W_K (d, d) are CUDA tensors of one dtype (bf16 or fp32).
    """

    def __init__(self, P, W_Q, W_K, scale: float, stream=None):
        lib = load_library()
        if P.dtype != W_Q.dtype or P.dtype != W_K.dtype:
            raise TypeError("P, W_Q and W_K must share a dtype")
        self.k, self.d = int(P.shape[0]), int(P.shape[1])
        if tuple(W_Q.shape) != (self.d, self.d) or tuple(W_K.shape) != (self.d, self.d):
            raise ValueError("W_Q and W_K must be d x d")
        self.dtype = P.dtype
        self.device = P.device
        handle = ctypes.c_void_p()
        st = lib.sa_prepare_query(_dev_ptr(P, "P"), _dev_ptr(W_Q, "W_Q"), _dev_ptr(W_K, "W_K"),
                                  self.k, self.d, float(scale), _dtype_code(P.dtype),
                                  ctypes.c_void_p(_stream_handle(stream)), ctypes.byref(handle))
        _check(st, "sa_prepare_query")
        self._h = handle
        self._lib = lib
        k, d, dt, kp = (ctypes.c_int() for _ in range(4))
        _check(lib.sa_query_info(self._h, ctypes.byref(k), ctypes.byref(d), ctypes.byref(dt),
                                 ctypes.byref(kp)), "sa_query_info")
        self.k_pad = kp.value

    # -- sizes -------------------------------------------------------------
    def workspace_bytes(self, batch: int, total_rows: int) -> int:
        return int(self._lib.sa_workspace_bytes(self._h, batch, total_rows))

    def host_path_device_bytes(self, batch: int, total_rows: int) -> int:
        return int(self._lib.sa_host_path_device_bytes(self._h, batch, total_rows))

    def new_workspace(self, batch: int, total_rows: int):
        torch = _torch()
        return torch.empty(self.workspace_bytes(batch, total_rows), dtype=torch.uint8,
                           device=self.device)

    # -- device path -------------------------------------------------------
    def _args(self, X, offsets, X_tilde, mass, workspace):
        torch = _torch()
        if X.dtype != self.dtype:
            raise TypeError(f"X dtype {X.dtype} != query dtype {self.dtype}")
        if X.dim() != 2 or X.shape[1] != self.d:
            raise ValueError("X must be (N, d)")
        if offsets.dtype != torch.int64 or offsets.dim() != 1:
            raise TypeError("offsets must be a 1-D int64 tensor")
        B = int(offsets.shape[0]) - 1
        N = int(X.shape[0])
        if X_tilde is None:
            X_tilde = torch.empty((B, self.k, self.d), dtype=torch.float32, device=X.device)
        if mass is None:
            mass = torch.empty((B, self.k), dtype=torch.float32, device=X.device)
        if workspace is None:
            workspace = self.new_workspace(B, N)
        xp = ctypes.c_void_p(X.data_ptr()) if N > 0 else ctypes.c_void_p(0)
        if N > 0:
            _dev_ptr(X, "X")
        args = (xp, _dev_ptr(offsets, "offsets"), B, N, _dev_ptr(X_tilde, "X_tilde"),
                _dev_ptr(mass, "mass"), _dev_ptr(workspace, "workspace"),
                int(workspace.numel() * workspace.element_size()))
        return args, X_tilde, mass, workspace

    def forward(self, X, offsets, X_tilde=None, mass=None, workspace=None, stream=None,
                check: bool = False) -> Tuple[object, object]:
        """X~ (B, k, d) and m (B, k) for the ragged batch (X (N, d), offsets (B+1,))."""
        args, X_tilde, mass, workspace = self._args(X, offsets, X_tilde, mass, workspace)
        sh = ctypes.c_void_p(_stream_handle(stream))
        _check(self._lib.sa_sketch_forward(self._h, *args, sh), "sa_sketch_forward")
        if check:
            read_device_status(workspace, stream)
        return X_tilde, mass

    def workspace_bytes_user_queries(self, batch: int, total_rows: int) -> int:
        return int(self._lib.sa_workspace_bytes_user_queries(self._h, batch, total_rows))

    def forward_user_queries(self, queries, X, offsets, X_tilde=None, mass=None, workspace=None,
                             stream=None, check: bool = False) -> Tuple[object, object]:
        """The SA step of a refinement layer: user b's rows queried by
        ``queries[b]`` ((B, k, d) fp32 CUDA tensor) with this query's W_Q,
        W_K and scale.  Returns X~ (B, k, d) and m (B, k)."""
        torch = _torch()
        B = int(offsets.shape[0]) - 1
        if queries.dtype != torch.float32 or tuple(queries.shape) != (B, self.k, self.d):
            raise ValueError(f"queries must be float32 of shape ({B}, {self.k}, {self.d})")
        if workspace is None:
            workspace = torch.empty(self.workspace_bytes_user_queries(B, int(X.shape[0])),
                                    dtype=torch.uint8, device=X.device)
        args, X_tilde, mass, workspace = self._args(X, offsets, X_tilde, mass, workspace)
        qp = _dev_ptr(queries, "queries") if B > 0 else ctypes.c_void_p(0)
        sh = ctypes.c_void_p(_stream_handle(stream))
        _check(self._lib.sa_sketch_forward_user_queries(self._h, qp, *args, sh),
               "sa_sketch_forward_user_queries")
        if check:
            read_device_status(workspace, stream)
        return X_tilde, mass

    def partials_user_queries(self, queries, X, offsets, X_tilde, mass, workspace,
                              stream=None) -> None:
        """Q'_b and the fused pass of forward_user_queries (finalize() completes it)."""
        args, *_ = self._args(X, offsets, X_tilde, mass, workspace)
        _check(self._lib.sa_sketch_partials_user_queries(
            self._h, _dev_ptr(queries, "queries"), *args, ctypes.c_void_p(_stream_handle(stream))),
            "sa_sketch_partials_user_queries")

    def partials(self, X, offsets, X_tilde, mass, workspace, stream=None) -> None:
        args, *_ = self._args(X, offsets, X_tilde, mass, workspace)
        _check(self._lib.sa_sketch_partials(self._h, *args, ctypes.c_void_p(_stream_handle(stream))),
               "sa_sketch_partials")

    def finalize(self, X, offsets, X_tilde, mass, workspace, stream=None) -> None:
        args, *_ = self._args(X, offsets, X_tilde, mass, workspace)
        _check(self._lib.sa_sketch_finalize(self._h, *args, ctypes.c_void_p(_stream_handle(stream))),
               "sa_sketch_finalize")

    def forward_noalloc(self, X, offsets, X_tilde=None, mass=None, device_flags=None,
                        stream=None) -> Tuple[object, object]:
        """Same layer through sa_sketch_forward_noalloc: no workspace, the
        library's fixed scratch array instead (see include/sa.h).  Outputs
        are allocated here when not given; the C call allocates nothing.
        ``device_flags`` (int32 CUDA tensor of 2 words) receives the call's
        device flags."""
        torch = _torch()
        if X.dtype != self.dtype:
            raise TypeError(f"X dtype {X.dtype} != query dtype {self.dtype}")
        if X.dim() != 2 or X.shape[1] != self.d:
            raise ValueError("X must be (N, d)")
        if offsets.dtype != torch.int64 or offsets.dim() != 1:
            raise TypeError("offsets must be a 1-D int64 tensor")
        B = int(offsets.shape[0]) - 1
        N = int(X.shape[0])
        if X_tilde is None:
            X_tilde = torch.empty((B, self.k, self.d), dtype=torch.float32, device=X.device)
        if mass is None:
            mass = torch.empty((B, self.k), dtype=torch.float32, device=X.device)
        xp = _dev_ptr(X, "X") if N > 0 else ctypes.c_void_p(0)
        fp = ctypes.c_void_p(0)
        if device_flags is not None:
            if device_flags.numel() * device_flags.element_size() < 8:
                raise ValueError("device_flags must hold 2 uint32 words")
            fp = _dev_ptr(device_flags, "device_flags")
        st = self._lib.sa_sketch_forward_noalloc(
            self._h, xp, _dev_ptr(offsets, "offsets"), B, N, _dev_ptr(X_tilde, "X_tilde"),
            _dev_ptr(mass, "mass"), fp, ctypes.c_void_p(_stream_handle(stream)))
        _check(st, "sa_sketch_forward_noalloc")
        return X_tilde, mass

    # -- host path ---------------------------------------------------------
    def forward_host(self, X_host, offsets_host: np.ndarray, device_buffer=None, stream=None,
                     out_x: Optional[np.ndarray] = None, out_m: Optional[np.ndarray] = None):
        """Same layer on host arrays.  X_host: a CPU torch tensor (bf16/fp32,
        ideally pinned) or a float32 numpy array for fp32 queries; offsets a
        numpy int64 array.  Returns numpy X~ (B, k, d) and m (B, k)."""
        torch = _torch()
        offsets_host = np.ascontiguousarray(offsets_host, dtype=np.int64)
        B = len(offsets_host) - 1
        if isinstance(X_host, np.ndarray):
            if self.dtype != torch.float32:
                raise TypeError("numpy X is only accepted for fp32 queries")
            X_host = torch.from_numpy(np.ascontiguousarray(X_host, dtype=np.float32))
        if X_host.is_cuda or X_host.dtype != self.dtype or not X_host.is_contiguous():
            raise ValueError("X_host must be a contiguous CPU tensor of the query dtype")
        N = int(X_host.shape[0])
        if device_buffer is None:
            device_buffer = torch.empty(self.host_path_device_bytes(B, N), dtype=torch.uint8,
                                        device=self.device)
        if out_x is None:
            out_x = np.empty((B, self.k, self.d), dtype=np.float32)
        if out_m is None:
            out_m = np.empty((B, self.k), dtype=np.float32)
        st = self._lib.sa_sketch_forward_host(
            self._h, ctypes.c_void_p(X_host.data_ptr() if N > 0 else 0),
            offsets_host.ctypes.data_as(ctypes.c_void_p), B, N,
            out_x.ctypes.data_as(ctypes.c_void_p), out_m.ctypes.data_as(ctypes.c_void_p),
            _dev_ptr(device_buffer, "device_buffer"),
            int(device_buffer.numel()), ctypes.c_void_p(_stream_handle(stream)))
        _check(st, "sa_sketch_forward_host")
        return out_x, out_m

    def backward(self, X, offsets, G, g=None, P_f32=None, W_Q_f32=None, W_K_f32=None,
                 queries=None, workspace=None, stream=None):
        """Gradients of the layer (sa_sketch_backward) for upstream G = dL/dX~
        (B, k, d) and g = dL/dm (B, k) or None.  P_f32 (shared queries) or
        queries (B, k, d), and W_Q_f32, W_K_f32 are the fp32 values the query
        was prepared with.  Returns dict(dX (N, d) bf16, dP (k, d) or
        dQueries (B, k, d), dW_Q, dW_K (d, d)) and the workspace."""
        torch = _torch()
        B, N = int(offsets.shape[0]) - 1, int(X.shape[0])
        dX = torch.empty((N, self.d), dtype=torch.bfloat16, device=X.device)
        dP = torch.empty((self.k, self.d) if queries is None else (B, self.k, self.d),
                         dtype=torch.float32, device=X.device)
        dWQ = torch.empty((self.d, self.d), dtype=torch.float32, device=X.device)
        dWK = torch.empty_like(dWQ)
        if workspace is None:
            workspace = torch.empty(int(self._lib.sa_workspace_bytes_backward(self._h, B, N)),
                                    dtype=torch.uint8, device=X.device)
        opt = lambda t, n: _dev_ptr(t, n) if t is not None else ctypes.c_void_p(0)  # noqa: E731
        _check(self._lib.sa_sketch_backward(
            self._h, opt(queries, "queries"), opt(P_f32, "P_f32"), _dev_ptr(W_Q_f32, "W_Q_f32"),
            _dev_ptr(W_K_f32, "W_K_f32"), ctypes.c_void_p(X.data_ptr() if N > 0 else 0),
            _dev_ptr(offsets, "offsets"), B, N, _dev_ptr(G, "G"), opt(g, "g"),
            ctypes.c_void_p(dX.data_ptr() if N > 0 else 0), _dev_ptr(dP, "dP"),
            _dev_ptr(dWQ, "dW_Q"), _dev_ptr(dWK, "dW_K"), _dev_ptr(workspace, "workspace"),
            int(workspace.numel() * workspace.element_size()),
            ctypes.c_void_p(_stream_handle(stream))), "sa_sketch_backward")
        out = dict(dX=dX, dW_Q=dWQ, dW_K=dWK)
        out["dP" if queries is None else "dQueries"] = dP
        return out, workspace

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._lib.sa_sketch_free(self._h)
            self._h = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass


class RefineParams:
    """The LN and FFN parameters of one refinement layer (sa_prepare_refine):
    W1, W3 (d, h), W2 (h, d), gamma1, beta1, gamma2, beta2 (d,), fp32 CUDA
    tensors."""

    def __init__(self, W1, W3, W2, gamma1, beta1, gamma2, beta2, stream=None):
        torch = _torch()
        lib = load_library()
        for name, t in (("W1", W1), ("W3", W3), ("W2", W2), ("gamma1", gamma1), ("beta1", beta1),
                        ("gamma2", gamma2), ("beta2", beta2)):
            if t.dtype != torch.float32:
                raise TypeError(f"{name} must be float32")
        self.d, self.h = int(W1.shape[0]), int(W1.shape[1])
        if tuple(W3.shape) != (self.d, self.h) or tuple(W2.shape) != (self.h, self.d):
            raise ValueError("W1, W3 must be (d, h) and W2 (h, d)")
        handle = ctypes.c_void_p()
        st = lib.sa_prepare_refine(*(_dev_ptr(t, n) for n, t in (
            ("W1", W1), ("W3", W3), ("W2", W2), ("gamma1", gamma1), ("beta1", beta1),
            ("gamma2", gamma2), ("beta2", beta2))), self.d, self.h,
            ctypes.c_void_p(_stream_handle(stream)), ctypes.byref(handle))
        _check(st, "sa_prepare_refine")
        self._h = handle
        self._lib = lib

    def update(self, prev, X_tilde, mass, out=None, prev_shared: bool = False,
               device_flags=None, stream=None):
        """out = LN2(z + FFN(z)), z = LN1(prev + X~ / m) for (B, k, d) fp32
        tensors; prev is (k, d) and shared by every user with prev_shared."""
        torch = _torch()
        B, k, d = (int(x) for x in X_tilde.shape)
        if out is None:
            out = torch.empty_like(X_tilde)
        fp = _dev_ptr(device_flags, "device_flags") if device_flags is not None else ctypes.c_void_p(0)
        _check(self._lib.sa_refine_update(self._h, _dev_ptr(prev, "prev"), int(prev_shared),
                                          _dev_ptr(X_tilde, "X_tilde"), _dev_ptr(mass, "mass"), B, k,
                                          _dev_ptr(out, "out"), fp,
                                          ctypes.c_void_p(_stream_handle(stream))),
               "sa_refine_update")
        return out

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._lib.sa_refine_free(self._h)
            self._h = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass


def refine_layer_forward(query: "SketchQuery", params: RefineParams, X, offsets, prev=None,
                         P_f32=None, out=None, workspace=None, stream=None):
    """One refinement layer (sa_refine_layer_forward): prev None means layer 1
    (queried by, and residual on, the prototypes P_f32 (k, d) fp32)."""
    torch = _torch()
    lib = load_library()
    B, N = int(offsets.shape[0]) - 1, int(X.shape[0])
    if out is None:
        out = torch.empty((B, query.k, query.d), dtype=torch.float32, device=X.device)
    if workspace is None:
        workspace = torch.empty(int(lib.sa_workspace_bytes_refine_layer(query._h, B, N)),
                                dtype=torch.uint8, device=X.device)
    _check(lib.sa_refine_layer_forward(
        query._h, params._h, _dev_ptr(prev, "prev") if prev is not None else ctypes.c_void_p(0),
        _dev_ptr(P_f32, "P_f32") if P_f32 is not None else ctypes.c_void_p(0),
        ctypes.c_void_p(X.data_ptr() if N > 0 else 0), _dev_ptr(offsets, "offsets"), B, N,
        _dev_ptr(out, "out"), _dev_ptr(workspace, "workspace"),
        int(workspace.numel() * workspace.element_size()),
        ctypes.c_void_p(_stream_handle(stream))), "sa_refine_layer_forward")
    return out, workspace


def refine_stack_forward(queries, params, P_f32, X, offsets, out=None, workspace=None,
                         stream=None):
    """len(queries) refinement layers (sa_refine_stack_forward); queries[l]
    and params[l] are layer l's handles.  Returns (out, workspace)."""
    torch = _torch()
    lib = load_library()
    L = len(queries)
    if L != len(params) or L < 1:
        raise ValueError("one query and one parameter set per layer")
    B, N = int(offsets.shape[0]) - 1, int(X.shape[0])
    q0 = queries[0]
    if out is None:
        out = torch.empty((B, q0.k, q0.d), dtype=torch.float32, device=X.device)
    if workspace is None:
        workspace = torch.empty(int(lib.sa_workspace_bytes_refine_stack(q0._h, B, N)),
                                dtype=torch.uint8, device=X.device)
    qs = (ctypes.c_void_p * L)(*[q._h.value for q in queries])
    rs = (ctypes.c_void_p * L)(*[r._h.value for r in params])
    _check(lib.sa_refine_stack_forward(
        L, ctypes.cast(qs, ctypes.c_void_p), ctypes.cast(rs, ctypes.c_void_p),
        _dev_ptr(P_f32, "P_f32"), ctypes.c_void_p(X.data_ptr() if N > 0 else 0),
        _dev_ptr(offsets, "offsets"), B, N, _dev_ptr(out, "out"),
        _dev_ptr(workspace, "workspace"), int(workspace.numel() * workspace.element_size()),
        ctypes.c_void_p(_stream_handle(stream))), "sa_refine_stack_forward")
    return out, workspace


def mass_normalise(X_tilde, mass, out=None, stream=None):
    """X~_bj / m_bj (0 where m_bj == 0) for fp32 CUDA tensors X~ (B, k, d)
    and m (B, k); ``out`` may be X_tilde (in place)."""
    torch = _torch()
    lib = load_library()
    if X_tilde.dtype != torch.float32 or mass.dtype != torch.float32 or X_tilde.dim() != 3:
        raise TypeError("X_tilde (B, k, d) and mass (B, k) must be float32")
    B, k, d = (int(x) for x in X_tilde.shape)
    if tuple(mass.shape) != (B, k):
        raise ValueError("mass must be (B, k)")
    if out is None:
        out = torch.empty_like(X_tilde)
    if B > 0:
        _check(lib.sa_mass_normalise(_dev_ptr(X_tilde, "X_tilde"), _dev_ptr(mass, "mass"), B, k, d,
                                     _dev_ptr(out, "out"), ctypes.c_void_p(_stream_handle(stream))),
               "sa_mass_normalise")
    return out


def read_device_status(workspace, stream=None) -> int:
    """Synchronises the stream, returns the device flag bits of the last call
    on `workspace` (0 when clean) and clears them."""
    lib = load_library()
    flags = ctypes.c_uint32(0)
    st = lib.sa_read_device_status(ctypes.c_void_p(workspace.data_ptr()),
                                   int(workspace.numel() * workspace.element_size()),
                                   ctypes.c_void_p(_stream_handle(stream)), ctypes.byref(flags))
    if st not in (SA_OK, SA_ERR_DEVICE_FLAG):
        _check(st, "sa_read_device_status")
    return int(flags.value)


class SketchCache:
    """A device pool of user sketches with a host index (sa_cache_create):
    `capacity` entries of (k, d) fp32 sketches plus (k,) masses, a
    time-to-live of `ttl` seconds.  Keys are 4-tuples (user, model_version,
    history_ts, config); `now` is the caller's clock in seconds."""

    def __init__(self, k: int, d: int, capacity: int, ttl: float):
        lib = load_library()
        handle = ctypes.c_void_p()
        _check(lib.sa_cache_create(int(k), int(d), int(capacity), float(ttl), ctypes.byref(handle)),
               "sa_cache_create")
        self._h, self._lib = handle, lib
        self.k, self.d, self.capacity, self.ttl = int(k), int(d), int(capacity), float(ttl)

    def lookup(self, keys, now: float, X_tilde, mass, stream=None) -> np.ndarray:
        """Copies the fresh entries into X_tilde[b], mass[b]; returns the hit
        mask (bool, one per key)."""
        B = len(keys)
        hit = np.zeros(max(B, 1), dtype=np.uint8)
        _check(self._lib.sa_cache_lookup(
            self._h, _keys_array(keys).ctypes.data_as(ctypes.c_void_p), B, float(now),
            hit.ctypes.data_as(ctypes.c_void_p), _dev_ptr(X_tilde, "X_tilde"), _dev_ptr(mass, "mass"),
            ctypes.c_void_p(_stream_handle(stream))), "sa_cache_lookup")
        return hit[:B].astype(bool)

    def insert(self, keys, now: float, X_tilde, mass, stream=None) -> None:
        _check(self._lib.sa_cache_insert(
            self._h, _keys_array(keys).ctypes.data_as(ctypes.c_void_p), len(keys), float(now),
            _dev_ptr(X_tilde, "X_tilde"), _dev_ptr(mass, "mass"),
            ctypes.c_void_p(_stream_handle(stream))), "sa_cache_insert")

    def stats(self) -> dict:
        vals = [ctypes.c_int64(0) for _ in range(4)]
        _check(self._lib.sa_cache_stats(self._h, *(ctypes.byref(v) for v in vals)), "sa_cache_stats")
        return dict(zip(("entries", "hits", "misses", "evictions"), (v.value for v in vals)))

    def forward(self, query: "SketchQuery", keys, now: float, X, offsets_host: np.ndarray,
                X_tilde=None, mass=None, workspace=None, stream=None):
        """One SA layer through the cache (sa_cache_forward).  offsets_host is
        an int64 numpy array (batch + 1).  Returns (X_tilde, mass, hit mask,
        workspace)."""
        torch = _torch()
        offsets_host = np.ascontiguousarray(offsets_host, dtype=np.int64)
        B, N = int(offsets_host.shape[0]) - 1, int(X.shape[0])
        if len(keys) != B:
            raise ValueError("one key per user")
        if X_tilde is None:
            X_tilde = torch.empty((B, self.k, self.d), dtype=torch.float32, device=X.device)
        if mass is None:
            mass = torch.empty((B, self.k), dtype=torch.float32, device=X.device)
        if workspace is None:
            workspace = torch.empty(int(self._lib.sa_cache_forward_workspace_bytes(query._h, B, N)),
                                    dtype=torch.uint8, device=X.device)
        hit = np.zeros(max(B, 1), dtype=np.uint8)
        _check(self._lib.sa_cache_forward(
            self._h, query._h, _keys_array(keys).ctypes.data_as(ctypes.c_void_p), float(now),
            ctypes.c_void_p(X.data_ptr() if N > 0 else 0),
            offsets_host.ctypes.data_as(ctypes.c_void_p), B, N, _dev_ptr(X_tilde, "X_tilde"),
            _dev_ptr(mass, "mass"), hit.ctypes.data_as(ctypes.c_void_p),
            _dev_ptr(workspace, "workspace"), int(workspace.numel() * workspace.element_size()),
            ctypes.c_void_p(_stream_handle(stream))), "sa_cache_forward")
        return X_tilde, mass, hit[:B].astype(bool), workspace

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._lib.sa_cache_free(self._h)
            self._h = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass


class WidthAdapter:
    """Y = X~ W_A on the tensor cores (sa_prepare_adapter): W_A is a (d, D)
    fp32 CUDA tensor; the output is bf16."""

    def __init__(self, W_A, stream=None):
        torch = _torch()
        lib = load_library()
        if W_A.dtype != torch.float32 or W_A.dim() != 2:
            raise TypeError("W_A must be a (d, D) float32 tensor")
        self.d, self.D = int(W_A.shape[0]), int(W_A.shape[1])
        handle = ctypes.c_void_p()
        _check(lib.sa_prepare_adapter(_dev_ptr(W_A, "W_A"), self.d, self.D,
                                      ctypes.c_void_p(_stream_handle(stream)), ctypes.byref(handle)),
               "sa_prepare_adapter")
        self._h, self._lib = handle, lib

    def forward(self, X_tilde, out=None, device_flags=None, stream=None):
        """X_tilde (..., d) fp32 -> (..., D) bf16."""
        torch = _torch()
        if X_tilde.dtype != torch.float32 or int(X_tilde.shape[-1]) != self.d:
            raise TypeError("X_tilde must be float32 with last dimension d")
        rows = int(X_tilde.numel()) // self.d
        if out is None:
            out = torch.empty(tuple(X_tilde.shape[:-1]) + (self.D,), dtype=torch.bfloat16,
                              device=X_tilde.device)
        fp = _dev_ptr(device_flags, "device_flags") if device_flags is not None else ctypes.c_void_p(0)
        _check(self._lib.sa_adapter_forward(self._h, _dev_ptr(X_tilde, "X_tilde"), rows,
                                             _dev_ptr(out, "out"), fp,
                                             ctypes.c_void_p(_stream_handle(stream))),
               "sa_adapter_forward")
        return out

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._lib.sa_adapter_free(self._h)
            self._h = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass


class ActionFusion:
    """The action-fusion producer (sa_prepare_action): X = E + SwiGLU-FFN of
    [E ; table[types]].  W1, W3 (d + d_a, h), W2 (h, d) and table
    (n_types, d_a) are fp32 CUDA tensors."""

    def __init__(self, W1, W3, W2, table, stream=None):
        torch = _torch()
        lib = load_library()
        for name, t in (("W1", W1), ("W3", W3), ("W2", W2), ("table", table)):
            if t.dtype != torch.float32 or t.dim() != 2:
                raise TypeError(f"{name} must be a 2-D float32 tensor")
        self.h, self.d = int(W2.shape[0]), int(W2.shape[1])
        self.n_types, self.d_a = int(table.shape[0]), int(table.shape[1])
        if tuple(W1.shape) != (self.d + self.d_a, self.h) or tuple(W3.shape) != tuple(W1.shape):
            raise ValueError("W1, W3 must be (d + d_a, h)")
        handle = ctypes.c_void_p()
        _check(lib.sa_prepare_action(_dev_ptr(W1, "W1"), _dev_ptr(W3, "W3"), _dev_ptr(W2, "W2"),
                                     _dev_ptr(table, "table"), self.d, self.d_a, self.h,
                                     self.n_types, ctypes.c_void_p(_stream_handle(stream)),
                                     ctypes.byref(handle)), "sa_prepare_action")
        self._h, self._lib = handle, lib

    def fuse(self, E, types, out=None, device_flags=None, stream=None):
        """E (rows, d) bf16 and types (rows,) uint8 CUDA tensors -> X (rows, d) bf16."""
        torch = _torch()
        if E.dtype != torch.bfloat16 or types.dtype != torch.uint8:
            raise TypeError("E must be bfloat16 and types uint8")
        rows = int(E.shape[0])
        if out is None:
            out = torch.empty_like(E)
        fp = _dev_ptr(device_flags, "device_flags") if device_flags is not None else ctypes.c_void_p(0)
        if rows > 0:
            _check(self._lib.sa_action_fuse(self._h, _dev_ptr(E, "E"), _dev_ptr(types, "types"), rows,
                                            _dev_ptr(out, "out"), fp,
                                            ctypes.c_void_p(_stream_handle(stream))),
                   "sa_action_fuse")
        return out

    def sketch_forward(self, query: "SketchQuery", E, types, offsets, X_tilde=None, mass=None,
                       workspace=None, stream=None):
        """The producer followed by one SA layer (sa_action_sketch_forward).
        Returns (X_tilde, mass, workspace)."""
        torch = _torch()
        B, N = int(offsets.shape[0]) - 1, int(E.shape[0])
        if X_tilde is None:
            X_tilde = torch.empty((B, query.k, query.d), dtype=torch.float32, device=E.device)
        if mass is None:
            mass = torch.empty((B, query.k), dtype=torch.float32, device=E.device)
        if workspace is None:
            workspace = torch.empty(int(self._lib.sa_workspace_bytes_action_sketch(query._h, B, N)),
                                    dtype=torch.uint8, device=E.device)
        _check(self._lib.sa_action_sketch_forward(
            self._h, query._h, ctypes.c_void_p(E.data_ptr() if N > 0 else 0),
            ctypes.c_void_p(types.data_ptr() if N > 0 else 0), _dev_ptr(offsets, "offsets"), B, N,
            _dev_ptr(X_tilde, "X_tilde"), _dev_ptr(mass, "mass"), _dev_ptr(workspace, "workspace"),
            int(workspace.numel() * workspace.element_size()),
            ctypes.c_void_p(_stream_handle(stream))), "sa_action_sketch_forward")
        return X_tilde, mass, workspace

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._lib.sa_action_free(self._h)
            self._h = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass
