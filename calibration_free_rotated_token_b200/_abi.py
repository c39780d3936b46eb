"""Thin ctypes binding of include/kvq.h (argument marshalling only).

Every function has the name of the C entry point it calls and takes torch
tensors (device memory) where the C call takes device pointers; it checks
shapes and dtypes, passes ``tensor.data_ptr()`` and the current (or given)
CUDA stream, and turns a negative status into ``KvqError``.  All compute
happens in the CUDA kernels of libkvq.so; if the library has not been built
or cannot be loaded, every call raises -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_OK = 0
KVQ_EINVAL = -1
KVQ_EUNSUPPORTED = -2
KVQ_ECUDA = -3
KVQ_ENOMEM = -4
KVQ_ENONFINITE = -5
KVQ_ETIMEOUT = -6
KVQ_QJL = 1
KVQ_BETA_CODEBOOK = 2
KVQ_CUDA_CORE_ROTATION = 4
KVQ_F32, KVQ_F16, KVQ_BF16 = 0, 1, 2
KVQ_LAYOUT_TOKEN, KVQ_LAYOUT_BLOCK32 = 0, 1
STATUS_NONFINITE, STATUS_NORM_OVERFLOW, STATUS_TIMEOUT = 1, 2, 4

# Every symbol include/kvq.h declares.
EXPORTED = (
    "kvq_init", "kvq_destroy", "kvq_quantize", "kvq_quantize_batch", "kvq_nsn_quantize", "kvq_decode_workspace",
    "kvq_decode_attend", "kvq_decode_attend_noalloc", "kvq_status", "kvq_last_error", "kvq_get_constants",
    "kvq_get_info", "kvq_codebook", "kvq_nsn_decode_attend", "kvq_decode_attend_ex", "kvq_probe_wait_timeout",
    "kvq_nsn_dq_side_bytes", "kvq_nsn_dq_quantize", "kvq_nsn_dq_decode_attend",
)
NOALLOC_SCRATCH_BYTES = 8 << 20

_DTYPES = {torch.float32: KVQ_F32, torch.float16: KVQ_F16, torch.bfloat16: KVQ_BF16}


class KvqError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"kvq error {code}: {msg}")
        self.code = code


class KvqCache(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("qjl", ctypes.c_void_p), ("norms", ctypes.c_void_p),
                ("capacity", ctypes.c_int64), ("layout", ctypes.c_int32)]


class KvqDecodeDesc(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("hq", ctypes.c_int32), ("hkv", ctypes.c_int32), ("k", ctypes.POINTER(KvqCache)),
                ("v", ctypes.POINTER(KvqCache)), ("k_block_mean", ctypes.c_void_p),
                ("v_block_mean", ctypes.c_void_p), ("k_window", ctypes.c_void_p), ("v_window", ctypes.c_void_p),
                ("window_cap", ctypes.c_int64), ("window_len", ctypes.c_void_p), ("seq_len", ctypes.c_void_p),
                ("max_T", ctypes.c_int64), ("scale", ctypes.c_float), ("logits", ctypes.c_void_p),
                ("logits_ld", ctypes.c_int64), ("out", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("ws_bytes", ctypes.c_size_t), ("k_side", ctypes.c_void_p), ("v_side", ctypes.c_void_p)]


class KvqQuantJob(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("n", ctypes.c_int64), ("ld", ctypes.c_int64),
                ("layout", ctypes.c_int32), ("codes", ctypes.c_void_p), ("qjl", ctypes.c_void_p),
                ("norms", ctypes.c_void_p)]


_lib = None
_lock = threading.Lock()


def load() -> ctypes.CDLL:
    """Load libkvq.so (raises if it is missing: build it with __graft_entry__.build())."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -c 'import __graft_entry__ as g; g.build()'`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, U32, U64, SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint32,
                                   ctypes.c_uint64, ctypes.c_size_t)
        L.kvq_init.argtypes = [ctypes.POINTER(P), I, I, U64, U32]
        L.kvq_destroy.argtypes = [P]
        L.kvq_quantize.argtypes = [P, P, I, I64, I64, I, P, P, P, P]
        L.kvq_nsn_quantize.argtypes = [P, P, I, I64, I64, I, P, P, P, P]
        L.kvq_quantize_batch.argtypes = [P, I, ctypes.POINTER(KvqQuantJob), P]
        L.kvq_decode_workspace.argtypes = [P, I, I, I, I64]
        L.kvq_decode_workspace.restype = SZ
        L.kvq_decode_attend.argtypes = [P, P, I, I, I, I, ctypes.POINTER(KvqCache), ctypes.POINTER(KvqCache), P,
                                        I64, ctypes.c_float, P, P, P, SZ, P]
        L.kvq_decode_attend_noalloc.argtypes = [P, P, I, I, I, I, ctypes.POINTER(KvqCache),
                                                ctypes.POINTER(KvqCache), P, I64, ctypes.c_float, P, P, P]
        L.kvq_status.argtypes = [P, P, ctypes.POINTER(U32)]
        L.kvq_last_error.restype = ctypes.c_char_p
        L.kvq_get_constants.argtypes = [P, P, P, P, P]
        L.kvq_get_info.argtypes = [P, ctypes.POINTER(I), ctypes.POINTER(I), ctypes.POINTER(I), ctypes.POINTER(U32)]
        L.kvq_codebook.argtypes = [I, I, U32, P, P]
        L.kvq_decode_attend_ex.argtypes = [P, ctypes.POINTER(KvqDecodeDesc), P]
        L.kvq_probe_wait_timeout.argtypes = [P, U32, P]
        L.kvq_nsn_decode_attend.argtypes = [P, P, I, I, I, I, ctypes.POINTER(KvqCache), ctypes.POINTER(KvqCache),
                                            P, P, P, I64, ctypes.c_float, P, P, P, SZ, P]
        L.kvq_nsn_dq_side_bytes.argtypes = [I]
        L.kvq_nsn_dq_side_bytes.restype = SZ
        L.kvq_nsn_dq_quantize.argtypes = [P, P, I, I64, I64, I, P, P, P, P]
        L.kvq_nsn_dq_decode_attend.argtypes = [P, P, I, I, I, I, ctypes.POINTER(KvqCache), ctypes.POINTER(KvqCache),
                                               P, P, P, I64, ctypes.c_float, P, P, P, SZ, P]
        for name in ("kvq_init", "kvq_destroy", "kvq_quantize", "kvq_quantize_batch", "kvq_nsn_quantize",
                     "kvq_decode_attend",
                     "kvq_decode_attend_noalloc", "kvq_status", "kvq_get_constants", "kvq_get_info",
                     "kvq_codebook", "kvq_nsn_decode_attend", "kvq_decode_attend_ex", "kvq_probe_wait_timeout",
                     "kvq_nsn_dq_quantize", "kvq_nsn_dq_decode_attend"):
            getattr(L, name).restype = I
        _lib = L
        return L


def _check(code: int):
    if code != KVQ_OK:
        raise KvqError(code, load().kvq_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t, name, dtype=None, numel=None, device=True):
    if t is None:
        raise ValueError(f"{name} is required")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements, needs {numel}")


class Handle:
    """Owns a kvq_handle; ``d``, ``b``, ``m``, ``qjl`` mirror kvq_get_info."""

    def __init__(self, d: int, b: int, seed: int, qjl: bool = True, beta: bool = False,
                 cuda_core_rotation: bool = False):
        L = load()
        h = ctypes.c_void_p()
        flags = ((KVQ_QJL if qjl else 0) | (KVQ_BETA_CODEBOOK if beta else 0) |
                 (KVQ_CUDA_CORE_ROTATION if cuda_core_rotation else 0))
        _check(L.kvq_init(ctypes.byref(h), d, b, seed & (2**64 - 1), flags))
        self._h = h
        dd, bb, mm, ff = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_uint32()
        _check(L.kvq_get_info(h, ctypes.byref(dd), ctypes.byref(bb), ctypes.byref(mm), ctypes.byref(ff)))
        self.d, self.b, self.m, self.qjl = dd.value, bb.value, mm.value, bool(ff.value & KVQ_QJL)

    @property
    def ptr(self):
        if self._h is None:
            raise RuntimeError("handle destroyed")
        return self._h

    def close(self):
        if getattr(self, "_h", None) is not None:
            load().kvq_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def kvq_init(d: int, b: int, seed: int, qjl: bool = True) -> Handle:
    return Handle(d, b, seed, qjl)


def kvq_destroy(h: Handle):
    h.close()


def kvq_get_constants(h: Handle):
    """(signs int8 [d], S fp16 [d, d], centroids fp32 [2^b], thresholds fp32 [2^b - 1]) on the host."""
    signs = torch.empty(h.d, dtype=torch.int8)
    S = torch.empty((h.m, h.d), dtype=torch.float16)
    cent = torch.empty(1 << h.b, dtype=torch.float32)
    thr = torch.empty(max((1 << h.b) - 1, 1), dtype=torch.float32)
    _check(load().kvq_get_constants(h.ptr, _ptr(signs), _ptr(S), _ptr(cent), _ptr(thr)))
    return signs, S, cent, thr[: (1 << h.b) - 1]


def packed_shapes(h: Handle, n: int, layout: int = KVQ_LAYOUT_TOKEN):
    """Shapes of (codes uint32, qjl uint32 or None, norms fp16) for n vectors in `layout`."""
    if layout == KVQ_LAYOUT_BLOCK32:
        nb = (n + 31) // 32
        return (nb, h.b, h.d), ((nb, h.m) if h.qjl else None), (n, 2)
    return (n, h.b, h.d // 32), ((n, h.m // 32) if h.qjl else None), (n, 2)


def alloc_packed(h: Handle, n: int, device="cuda", layout: int = KVQ_LAYOUT_TOKEN):
    cs, qs, ns = packed_shapes(h, n, layout)
    codes = torch.empty(cs, dtype=torch.int32, device=device)
    qjl = torch.empty(qs, dtype=torch.int32, device=device) if qs else None
    norms = torch.empty(ns, dtype=torch.float16, device=device)
    return codes, qjl, norms


def kvq_quantize(h: Handle, x: torch.Tensor, codes, qjl, norms, stream=None, layout: int = KVQ_LAYOUT_TOKEN):
    """x: [n, d] (any leading dims flattened), fp32/fp16/bf16, rows contiguous in the last dim."""
    if x.dim() < 2 or x.shape[-1] != h.d:
        raise ValueError(f"x must be [..., {h.d}]")
    x2 = x.reshape(-1, h.d)
    if x2.stride(-1) != 1:
        raise ValueError("x rows must be contiguous")
    n = x2.shape[0]
    ld = x2.stride(0) if n > 1 else h.d
    if x.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {x.dtype}")
    rows = n if layout == KVQ_LAYOUT_TOKEN else 32 * ((n + 31) // 32)
    _need(codes, "codes", numel=rows * h.b * h.d // 32)
    _need(norms, "norms", dtype=torch.float16, numel=2 * n)
    if h.qjl:
        _need(qjl, "qjl", numel=rows * h.m // 32)
    _check(load().kvq_quantize(h.ptr, _ptr(x2), _DTYPES[x.dtype], n, ld, layout, _ptr(codes),
                               _ptr(qjl) if h.qjl else None, _ptr(norms), _stream(stream)))


def kvq_codebook(d: int, b: int, beta: bool = False):
    """(centroids, thresholds) as fp32 numpy arrays, computed by the library on the host."""
    import numpy as np
    c = np.zeros(1 << b, np.float32)
    t = np.zeros(max((1 << b) - 1, 1), np.float32)
    _check(load().kvq_codebook(d, b, KVQ_BETA_CODEBOOK if beta else 0, c.ctypes.data, t.ctypes.data))
    return c, t[: (1 << b) - 1]


def _job(h: Handle, x: torch.Tensor, codes, qjl, norms, layout: int) -> KvqQuantJob:
    if x.dim() < 2 or x.shape[-1] != h.d:
        raise ValueError(f"x must be [..., {h.d}]")
    x2 = x.reshape(-1, h.d)
    if x2.stride(-1) != 1:
        raise ValueError("x rows must be contiguous")
    n = x2.shape[0]
    if x.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {x.dtype}")
    rows = n if layout == KVQ_LAYOUT_TOKEN else 32 * ((n + 31) // 32)
    _need(codes, "codes", numel=rows * h.b * h.d // 32)
    _need(norms, "norms", dtype=torch.float16, numel=2 * n)
    if h.qjl:
        _need(qjl, "qjl", numel=rows * h.m // 32)
    return KvqQuantJob(_ptr(x2), _DTYPES[x.dtype], n, x2.stride(0) if n > 1 else h.d, layout, _ptr(codes),
                       _ptr(qjl) if h.qjl else None, _ptr(norms))


def kvq_quantize_batch(h: Handle, jobs, stream=None):
    """jobs: sequence of (x, codes, qjl, norms, layout) -- kvq_quantize of each, fused launches where possible."""
    arr = (KvqQuantJob * max(len(jobs), 1))(*[_job(h, *j) for j in jobs])
    _check(load().kvq_quantize_batch(h.ptr, len(jobs), arr, _stream(stream)))


def kvq_nsn_quantize(h: Handle, x: torch.Tensor, codes, norms, block_mean, stream=None,
                     layout: int = KVQ_LAYOUT_TOKEN):
    """x: [n_heads, n_tok, d] contiguous, n_tok % 128 == 0; layout token (keys) or block-32 (values)."""
    if x.dim() != 3 or x.shape[-1] != h.d:
        raise ValueError(f"x must be [heads, tokens, {h.d}]")
    _need(x, "x")
    H, T, _ = x.shape
    _need(codes, "codes", numel=H * T * h.b * h.d // 32)
    _need(norms, "norms", dtype=torch.float16, numel=2 * H * T)
    _need(block_mean, "block_mean", dtype=torch.float16, numel=H * (T // 128) * h.d)
    _check(load().kvq_nsn_quantize(h.ptr, _ptr(x), _DTYPES[x.dtype], H, T, layout, _ptr(codes), _ptr(norms),
                                   _ptr(block_mean), _stream(stream)))


def kvq_nsn_dq_side_bytes(d: int) -> int:
    """Bytes of one side record of the double-quantized NSN front end (0 for an unsupported d)."""
    return int(load().kvq_nsn_dq_side_bytes(d))


def kvq_nsn_dq_quantize(h: Handle, x: torch.Tensor, codes, wnorms, side, stream=None,
                        layout: int = KVQ_LAYOUT_TOKEN):
    """x: [n_heads, n_tok, d] fp16/bf16, n_tok % 128 == 0; wnorms fp16 [n_heads * n_tok];
    side uint8 [n_heads * n_tok/128, kvq_nsn_dq_side_bytes(d)]."""
    if x.dim() != 3 or x.shape[-1] != h.d:
        raise ValueError(f"x must be [heads, tokens, {h.d}]")
    _need(x, "x")
    H, T, _ = x.shape
    _need(codes, "codes", numel=H * T * h.b * h.d // 32)
    _need(wnorms, "wnorms", dtype=torch.float16, numel=H * T)
    _need(side, "side", dtype=torch.uint8, numel=H * (T // 128) * kvq_nsn_dq_side_bytes(h.d))
    _check(load().kvq_nsn_dq_quantize(h.ptr, _ptr(x), _DTYPES[x.dtype], H, T, layout, _ptr(codes), _ptr(wnorms),
                                      _ptr(side), _stream(stream)))


def kvq_decode_workspace(h: Handle, batch: int, hq: int, hkv: int, max_T: int) -> int:
    return int(load().kvq_decode_workspace(h.ptr, batch, hq, hkv, max_T))


def make_cache(codes, qjl, norms, capacity: int, layout: int = KVQ_LAYOUT_TOKEN) -> KvqCache:
    """Cache descriptor; keys use KVQ_LAYOUT_TOKEN, values KVQ_LAYOUT_BLOCK32."""
    return KvqCache(codes.data_ptr(), qjl.data_ptr() if qjl is not None else None, norms.data_ptr(), capacity,
                    layout)


def kvq_decode_attend(h: Handle, q: torch.Tensor, hkv: int, kcache: KvqCache, vcache: KvqCache,
                      seq_len: torch.Tensor, max_T: int, scale: float, out: torch.Tensor,
                      workspace: torch.Tensor, logits: torch.Tensor | None = None, stream=None):
    """q: [batch, hq, d]; seq_len int32 [batch] on the device; out fp32 [batch, hq, d]."""
    if q.dim() != 3 or q.shape[-1] != h.d:
        raise ValueError(f"q must be [batch, hq, {h.d}]")
    _need(q, "q")
    B, hq, _ = q.shape
    _need(seq_len, "seq_len", dtype=torch.int32, numel=B)
    _need(out, "out", dtype=torch.float32, numel=B * hq * h.d)
    _need(workspace, "workspace")
    if logits is not None:
        _need(logits, "logits", dtype=torch.float32, numel=B * hq * max_T)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().kvq_decode_attend(h.ptr, _ptr(q), _DTYPES[q.dtype], B, hq, hkv, ctypes.byref(kcache),
                                    ctypes.byref(vcache), _ptr(seq_len), max_T, float(scale), _ptr(logits),
                                    _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)))


def kvq_nsn_decode_attend(h: Handle, q: torch.Tensor, hkv: int, kcache: KvqCache, vcache: KvqCache,
                          k_block_mean: torch.Tensor, v_block_mean: torch.Tensor, seq_len: torch.Tensor,
                          max_T: int, scale: float, out: torch.Tensor, workspace: torch.Tensor,
                          logits: torch.Tensor | None = None, stream=None):
    """kvq_decode_attend over caches from kvq_nsn_quantize; block means fp16 [streams, capacity/128, d]."""
    if q.dim() != 3 or q.shape[-1] != h.d:
        raise ValueError(f"q must be [batch, hq, {h.d}]")
    _need(q, "q")
    B, hq, _ = q.shape
    _need(seq_len, "seq_len", dtype=torch.int32, numel=B)
    _need(out, "out", dtype=torch.float32, numel=B * hq * h.d)
    _need(workspace, "workspace")
    _need(k_block_mean, "k_block_mean", dtype=torch.float16)
    _need(v_block_mean, "v_block_mean", dtype=torch.float16)
    if logits is not None:
        _need(logits, "logits", dtype=torch.float32, numel=B * hq * max_T)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().kvq_nsn_decode_attend(h.ptr, _ptr(q), _DTYPES[q.dtype], B, hq, hkv, ctypes.byref(kcache),
                                        ctypes.byref(vcache), _ptr(k_block_mean), _ptr(v_block_mean),
                                        _ptr(seq_len), max_T, float(scale), _ptr(logits), _ptr(out),
                                        _ptr(workspace), ws_bytes, _stream(stream)))


def kvq_nsn_dq_decode_attend(h: Handle, q: torch.Tensor, hkv: int, kcache: KvqCache, vcache: KvqCache,
                             k_side: torch.Tensor, v_side: torch.Tensor, seq_len: torch.Tensor, max_T: int,
                             scale: float, out: torch.Tensor, workspace: torch.Tensor,
                             logits: torch.Tensor | None = None, stream=None):
    """kvq_decode_attend over caches from kvq_nsn_dq_quantize (norms = fp16 ||w|| per token; side
    records uint8 [streams, capacity/128, kvq_nsn_dq_side_bytes(d)])."""
    if q.dim() != 3 or q.shape[-1] != h.d:
        raise ValueError(f"q must be [batch, hq, {h.d}]")
    _need(q, "q")
    B, hq, _ = q.shape
    _need(seq_len, "seq_len", dtype=torch.int32, numel=B)
    _need(out, "out", dtype=torch.float32, numel=B * hq * h.d)
    _need(workspace, "workspace")
    _need(k_side, "k_side", dtype=torch.uint8)
    _need(v_side, "v_side", dtype=torch.uint8)
    if logits is not None:
        _need(logits, "logits", dtype=torch.float32, numel=B * hq * max_T)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().kvq_nsn_dq_decode_attend(h.ptr, _ptr(q), _DTYPES[q.dtype], B, hq, hkv, ctypes.byref(kcache),
                                           ctypes.byref(vcache), _ptr(k_side), _ptr(v_side), _ptr(seq_len), max_T,
                                           float(scale), _ptr(logits), _ptr(out), _ptr(workspace), ws_bytes,
                                           _stream(stream)))


def kvq_decode_attend_ex(h: Handle, q: torch.Tensor, hkv: int, kcache: KvqCache, vcache: KvqCache,
                         seq_len: torch.Tensor, max_T: int, scale: float, out: torch.Tensor, workspace: torch.Tensor,
                         k_window: torch.Tensor | None = None, v_window: torch.Tensor | None = None,
                         window_len: torch.Tensor | None = None, k_block_mean: torch.Tensor | None = None,
                         v_block_mean: torch.Tensor | None = None, logits: torch.Tensor | None = None,
                         logits_ld: int = 0, stream=None, k_side: torch.Tensor | None = None,
                         v_side: torch.Tensor | None = None):
    """Decode over a packed cache (plain, NSN with fp16 block means, or NSN with
    double-quantized side records) and an optional fp16 residual window
    ([batch * hkv, window_cap, d]); window_len int32 [batch] on the device."""
    if q.dim() != 3 or q.shape[-1] != h.d:
        raise ValueError(f"q must be [batch, hq, {h.d}]")
    _need(q, "q")
    B, hq, _ = q.shape
    _need(seq_len, "seq_len", dtype=torch.int32, numel=B)
    _need(out, "out", dtype=torch.float32, numel=B * hq * h.d)
    _need(workspace, "workspace")
    cap = 0
    if k_window is not None or v_window is not None:
        _need(k_window, "k_window", dtype=torch.float16)
        _need(v_window, "v_window", dtype=torch.float16)
        _need(window_len, "window_len", dtype=torch.int32, numel=B)
        cap = k_window.shape[-2]
        if k_window.numel() != B * hkv * cap * h.d or v_window.shape != k_window.shape:
            raise ValueError("windows must be [batch * hkv, window_cap, d]")
    if logits is not None:
        _need(logits, "logits", dtype=torch.float32, numel=B * hq * (logits_ld or (max_T + cap)))
    d = KvqDecodeDesc(_ptr(q), _DTYPES[q.dtype], B, hq, hkv, ctypes.pointer(kcache), ctypes.pointer(vcache),
                      _ptr(k_block_mean), _ptr(v_block_mean), _ptr(k_window), _ptr(v_window), cap,
                      _ptr(window_len), _ptr(seq_len), max_T, float(scale), _ptr(logits), logits_ld, _ptr(out),
                      _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(k_side), _ptr(v_side))
    _check(load().kvq_decode_attend_ex(h.ptr, ctypes.byref(d), _stream(stream)))


def kvq_decode_attend_noalloc(h: Handle, q: torch.Tensor, hkv: int, kcache: KvqCache, vcache: KvqCache,
                              seq_len: torch.Tensor, max_T: int, scale: float, out: torch.Tensor,
                              logits: torch.Tensor | None = None, stream=None):
    """kvq_decode_attend using the library's fixed device scratch instead of a workspace.

    For callers that must not allocate device memory when they decode; the
    scratch (8 MiB per GPU, held until exit) is shared by all calls, so calls
    must not overlap on the GPU.
    """
    if q.dim() != 3 or q.shape[-1] != h.d:
        raise ValueError(f"q must be [batch, hq, {h.d}]")
    _need(q, "q")
    B, hq, _ = q.shape
    _need(seq_len, "seq_len", dtype=torch.int32, numel=B)
    _need(out, "out", dtype=torch.float32, numel=B * hq * h.d)
    if logits is not None:
        _need(logits, "logits", dtype=torch.float32, numel=B * hq * max_T)
    _check(load().kvq_decode_attend_noalloc(h.ptr, _ptr(q), _DTYPES[q.dtype], B, hq, hkv, ctypes.byref(kcache),
                                            ctypes.byref(vcache), _ptr(seq_len), max_T, float(scale), _ptr(logits),
                                            _ptr(out), _stream(stream)))


def kvq_status(h: Handle, stream=None) -> tuple[int, int]:
    """(status code, raw bits); synchronises the stream."""
    bits = ctypes.c_uint32()
    code = load().kvq_status(h.ptr, _stream(stream), ctypes.byref(bits))
    return code, bits.value


def kvq_probe_wait_timeout(h: Handle, polls: int = 4096, stream=None):
    """One kernel whose bounded mbarrier wait runs out; kvq_status then reports KVQ_ETIMEOUT."""
    _check(load().kvq_probe_wait_timeout(h.ptr, polls, _stream(stream)))


def kvq_last_error() -> str:
    return load().kvq_last_error().decode()
