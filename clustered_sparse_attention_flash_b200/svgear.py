"""ctypes binding of libsvgear.so (include/svgear.h).

Every function here has the name of a C entry point and only marshals
arguments: torch tensors become device pointers, streams become cudaStream_t
handles.  All arithmetic runs in the CUDA library; there is no fallback.  The
few helpers at the end allocate outputs and workspaces with torch and then call
the same entry points.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Dict, Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsvgear.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "svgear.h")

SVGEAR_OK = 0
SVGEAR_ERR_INVALID = -1
SVGEAR_ERR_UNSUPPORTED = -2
SVGEAR_ERR_CUDA = -3
SVGEAR_ERR_TIMEOUT = -4
SVGEAR_ERR_WORKSPACE = -5
SVGEAR_F32 = 0
SVGEAR_BF16 = 1
SVGEAR_ROUTE_ERROR = 0
SVGEAR_ROUTE_MASS = 1
SVGEAR_ROUTE_ERROR_NOV = 2
SVGEAR_BUDGET_ROW = 0
SVGEAR_BUDGET_GLOBAL = 1


class SvgearError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {code} ({status_string(code)})")
        self.code = code


class svgear_params(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("Nq", ctypes.c_int), ("Nk", ctypes.c_int),
                ("d", ctypes.c_int), ("Cq", ctypes.c_int), ("Ck", ctypes.c_int),
                ("iters", ctypes.c_int), ("rho", ctypes.c_float), ("scale", ctypes.c_float),
                ("dtype", ctypes.c_int), ("router", ctypes.c_int), ("budget", ctypes.c_int)]


class svgear_stats(ctypes.Structure):
    _fields_ = [("ms_kmeans_q", ctypes.c_float), ("ms_kmeans_k", ctypes.c_float),
                ("ms_permute", ctypes.c_float), ("ms_block_error", ctypes.c_float),
                ("ms_route", ctypes.c_float), ("ms_attn", ctypes.c_float),
                ("ms_total", ctypes.c_float), ("exec_pairs", ctypes.c_int64),
                ("comp_pairs", ctypes.c_int64), ("ms_attn_kernel", ctypes.c_float)]

    def as_dict(self) -> Dict[str, float]:
        return {k: getattr(self, k) for k, _ in self._fields_}


_VIEW_FIELDS = ["cent_q", "cent_k", "vbar", "labels_q", "labels_k", "counts_q", "counts_k",
                "perm_q", "perm_k", "off_q", "off_k", "Qp", "Kp", "Vp", "key_scalars", "E", "M",
                "mask", "sel", "n_sel", "exec_pairs"]


class svgear_views(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _VIEW_FIELDS]


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_PP = ctypes.POINTER(svgear_params)

_SIGS = {
    "svgear_version": (ctypes.c_char_p, []),
    "svgear_status_string": (ctypes.c_char_p, [_I]),
    "svgear_launch_count": (ctypes.c_longlong, []),
    "svgear_get_status": (_I, [_P]),
    "svgear_selftest_wait": (_I, [ctypes.c_longlong, _P]),
    "svgear_kmeans_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "svgear_kmeans": (_I, [_P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "svgear_permute_workspace_size": (_SZ, [_I, _I, _I]),
    "svgear_permute": (_I, [_P, _I, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "svgear_block_error_workspace_size": (_SZ, [_PP]),
    "svgear_block_error": (_I, [_P, _P, _P, _P, _P, _P, _P, _PP, _P, _P, _P, _SZ, _P]),
    "svgear_block_error_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _PP, _P, _P, _P]),
    "svgear_route": (_I, [_P, _P, _P, _PP, _P, _P, _P, _P, _P]),
    "svgear_route_global": (_I, [_P, _P, _P, _P, _PP, _P, _P, _P, _P, _P]),
    "svgear_hybrid_attn_workspace_size": (_SZ, [_PP]),
    "svgear_hybrid_attn": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _PP, _P, _P, _SZ, _P]),
    "svgear_workspace_size": (_SZ, [_PP]),
    "svgear_forward_views": (_I, [_PP, _P, _SZ, ctypes.POINTER(svgear_views)]),
    "svgear_forward": (_I, [_P, _P, _P, _PP, _P, _P, _P, _P, _SZ, _P, ctypes.POINTER(svgear_stats)]),
}

_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if libsvgear.so has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libsvgear.so not found at {LIB_PATH}; run "
                              "`python -m clustered_sparse_attention_flash_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def header_functions():
    """Names of the entry points declared in include/svgear.h."""
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"SVGEAR_API\s+[\w\s\*]*?\b(svgear_\w+)\s*\(", txt)))


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        if not x.is_cuda:
            raise ValueError("device tensor expected")
        if not x.is_contiguous():
            raise ValueError("contiguous tensor expected")
        return x.data_ptr()
    raise TypeError(f"cannot pass {type(x)} as a pointer")


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn: str, code: int) -> None:
    if code != SVGEAR_OK:
        raise SvgearError(fn, code)


def params(H, Nq, Nk, d, Cq, Ck, iters, rho, scale=0.0, dtype=SVGEAR_BF16,
           router=SVGEAR_ROUTE_ERROR, budget=SVGEAR_BUDGET_ROW) -> svgear_params:
    return svgear_params(H, Nq, Nk, d, Cq, Ck, iters, rho, scale, dtype, router, budget)


# ----------------------------------------------------------------- entries

def svgear_version() -> str:
    return lib().svgear_version().decode()


def svgear_launch_count() -> int:
    return int(lib().svgear_launch_count())


def status_string(code: int) -> str:
    return lib().svgear_status_string(code).decode()


svgear_status_string = status_string


def svgear_get_status(stream=None) -> int:
    return lib().svgear_get_status(_stream(stream))


def svgear_selftest_wait(limit_ns: int, stream=None) -> None:
    _check("svgear_selftest_wait", lib().svgear_selftest_wait(int(limit_ns), _stream(stream)))


def svgear_kmeans_workspace_size(H, N, d, C) -> int:
    return lib().svgear_kmeans_workspace_size(H, N, d, C)


def svgear_kmeans(X, dtype, H, N, d, C, iters, init, cent, labels, counts, ws, ws_bytes, stream=None):
    _check("svgear_kmeans", lib().svgear_kmeans(
        _ptr(X), dtype, H, N, d, C, iters, _ptr(init), _ptr(cent), _ptr(labels), _ptr(counts),
        _ptr(ws), ws_bytes, _stream(stream)))


def svgear_permute_workspace_size(H, N, C) -> int:
    return lib().svgear_permute_workspace_size(H, N, C)


def svgear_permute(X, dtype, labels, H, N, d, C, Xp, perm, offsets, V, Vp, Vbar, key_scalars,
                   ws, ws_bytes, stream=None):
    _check("svgear_permute", lib().svgear_permute(
        _ptr(X), dtype, _ptr(labels), H, N, d, C, _ptr(Xp), _ptr(perm), _ptr(offsets), _ptr(V),
        _ptr(Vp), _ptr(Vbar), _ptr(key_scalars), _ptr(ws), ws_bytes, _stream(stream)))


def svgear_block_error_workspace_size(p: svgear_params) -> int:
    return lib().svgear_block_error_workspace_size(ctypes.byref(p))


def svgear_block_error(Qbar, Kbar, Vbar, Kp, Vp, k_off, key_scalars, p, E, M, ws, ws_bytes,
                       stream=None):
    _check("svgear_block_error", lib().svgear_block_error(
        _ptr(Qbar), _ptr(Kbar), _ptr(Vbar), _ptr(Kp), _ptr(Vp), _ptr(k_off), _ptr(key_scalars),
        ctypes.byref(p), _ptr(E), _ptr(M), _ptr(ws), ws_bytes, _stream(stream)))


def svgear_block_error_noalloc(Qbar, Kbar, Vbar, Kp, Vp, k_off, key_scalars, p, E, M, stream=None):
    _check("svgear_block_error_noalloc", lib().svgear_block_error_noalloc(
        _ptr(Qbar), _ptr(Kbar), _ptr(Vbar), _ptr(Kp), _ptr(Vp), _ptr(k_off), _ptr(key_scalars),
        ctypes.byref(p), _ptr(E), _ptr(M), _stream(stream)))


def svgear_route(E, k_counts, q_counts, p, mask, sel, n_sel, exec_pairs, stream=None):
    _check("svgear_route", lib().svgear_route(
        _ptr(E), _ptr(k_counts), _ptr(q_counts), ctypes.byref(p), _ptr(mask), _ptr(sel),
        _ptr(n_sel), _ptr(exec_pairs), _stream(stream)))


def svgear_route_global(E, M, k_counts, q_counts, p, mask, sel, n_sel, exec_pairs, stream=None):
    _check("svgear_route_global", lib().svgear_route_global(
        _ptr(E), _ptr(M), _ptr(k_counts), _ptr(q_counts), ctypes.byref(p), _ptr(mask), _ptr(sel),
        _ptr(n_sel), _ptr(exec_pairs), _stream(stream)))


def svgear_hybrid_attn_workspace_size(p: svgear_params) -> int:
    return lib().svgear_hybrid_attn_workspace_size(ctypes.byref(p))


def svgear_hybrid_attn(Qp, Kp, Vp, q_off, k_off, perm_q, Kbar, Vbar, sel, n_sel, p, O, ws,
                       ws_bytes, stream=None):
    _check("svgear_hybrid_attn", lib().svgear_hybrid_attn(
        _ptr(Qp), _ptr(Kp), _ptr(Vp), _ptr(q_off), _ptr(k_off), _ptr(perm_q), _ptr(Kbar),
        _ptr(Vbar), _ptr(sel), _ptr(n_sel), ctypes.byref(p), _ptr(O), _ptr(ws), ws_bytes,
        _stream(stream)))


def svgear_workspace_size(p: svgear_params) -> int:
    return lib().svgear_workspace_size(ctypes.byref(p))


def svgear_forward_views(p: svgear_params, ws, ws_bytes) -> svgear_views:
    v = svgear_views()
    _check("svgear_forward_views", lib().svgear_forward_views(
        ctypes.byref(p), _ptr(ws), ws_bytes, ctypes.byref(v)))
    return v


def svgear_forward(Q, K, V, p, init_q, init_k, O, ws, ws_bytes, stream=None, stats=None):
    _check("svgear_forward", lib().svgear_forward(
        _ptr(Q), _ptr(K), _ptr(V), ctypes.byref(p), _ptr(init_q), _ptr(init_k), _ptr(O),
        _ptr(ws), ws_bytes, _stream(stream), ctypes.byref(stats) if stats is not None else None))


# ------------------------------------------------------- torch conveniences

def dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return SVGEAR_BF16
    if t.dtype == torch.float32:
        return SVGEAR_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def workspace(nbytes: int, device="cuda"):
    import torch
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def view_tensors(p: svgear_params, ws) -> Dict[str, "object"]:
    """torch tensors aliasing the intermediates svgear_forward leaves in `ws`."""
    import torch
    v = svgear_forward_views(p, ws, ws.numel())
    H, Nq, Nk, d, Cq, Ck = p.H, p.Nq, p.Nk, p.d, p.Cq, p.Ck
    tdt = torch.bfloat16 if p.dtype == SVGEAR_BF16 else torch.float32
    es = 2 if p.dtype == SVGEAR_BF16 else 4
    base = ws.data_ptr()
    spec = {
        "cent_q": (torch.float32, (H, Cq, d)), "cent_k": (torch.float32, (H, Ck, d)),
        "vbar": (torch.float32, (H, Ck, d)), "labels_q": (torch.int32, (H, Nq)),
        "labels_k": (torch.int32, (H, Nk)), "counts_q": (torch.int32, (H, Cq)),
        "counts_k": (torch.int32, (H, Ck)), "perm_q": (torch.int32, (H, Nq)),
        "perm_k": (torch.int32, (H, Nk)), "off_q": (torch.int32, (H, Cq + 1)),
        "off_k": (torch.int32, (H, Ck + 1)), "Qp": (tdt, (H, Nq, d)), "Kp": (tdt, (H, Nk, d)),
        "Vp": (tdt, (H, Nk, d)), "key_scalars": (torch.float32, (3, H, Nk)),
        "E": (torch.float32, (H, Cq, Ck)), "M": (torch.float32, (H, Cq)),
        "mask": (torch.uint8, (H, Cq, Ck)), "sel": (torch.int32, (H, Cq, Ck)),
        "n_sel": (torch.int32, (H, Cq)), "exec_pairs": (torch.int64, (H,)),
    }
    out = {}
    for name, (dt, shape) in spec.items():
        off = getattr(v, name) - base
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dt).element_size()
        out[name] = ws[off:off + nbytes].view(dt).view(shape)
    del es
    return out


def forward(Q, K, V, Cq: int, Ck: int, iters: int, rho: float, scale: float = 0.0,
            init_q=None, init_k=None, ws=None, stream=None, stats: bool = False,
            router: int = SVGEAR_ROUTE_ERROR, budget: int = SVGEAR_BUDGET_ROW):
    """Allocate O (and the workspace unless given) and run svgear_forward.
    Returns (O, ws, params, stats-dict or None)."""
    import torch
    H, Nq, d = Q.shape
    Nk = K.shape[1]
    p = params(H, Nq, Nk, d, Cq, Ck, iters, rho, scale, dtype_code(Q), router, budget)
    need = svgear_workspace_size(p)
    if need == 0:
        raise SvgearError("svgear_workspace_size", SVGEAR_ERR_INVALID)
    if ws is None or ws.numel() < need:
        ws = workspace(need, Q.device)
    O = torch.empty_like(Q)
    st = svgear_stats() if stats else None
    svgear_forward(Q, K, V, p, init_q, init_k, O, ws, ws.numel(), stream, st)
    return O, ws, p, (st.as_dict() if st is not None else None)
