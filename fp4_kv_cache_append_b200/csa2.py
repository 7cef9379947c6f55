"""ctypes binding of libcsa2 (include/csa2.h): argument marshalling only.

Every function here has the name of the C entry point it calls and does no
arithmetic of the method: torch supplies device memory and the current CUDA
stream, the library does the work.  The library is loaded on first use and a
missing or unloadable library raises immediately -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libcsa2.so")

CSA2_OK = 0
STATUS_NAMES = {0: "CSA2_OK", 1: "CSA2_ERR_INVALID_ARG", 2: "CSA2_ERR_UNSUPPORTED_SHAPE", 3: "CSA2_ERR_CUDA",
                4: "CSA2_ERR_DEVICE_CHECK", 5: "CSA2_ERR_WORKSPACE"}
DEV_INDEX_RANGE, DEV_TIMEOUT, DEV_APPEND_RANGE, DEV_BAD_POSITION = 0x1, 0x2, 0x4, 0x8


class Csa2Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class MainCacheDesc(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("ik", ctypes.c_void_p),
                ("ik_scale", ctypes.c_void_p), ("n_entries", ctypes.c_void_p), ("pending_kv", ctypes.c_void_p),
                ("pending_gate", ctypes.c_void_p), ("B", ctypes.c_int32), ("cap", ctypes.c_int32),
                ("D", ctypes.c_int32), ("d_I", ctypes.c_int32), ("m", ctypes.c_int32)]


class SwaCacheDesc(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_void_p), ("scale", ctypes.c_float), ("B", ctypes.c_int32),
                ("W_cap", ctypes.c_int32), ("D", ctypes.c_int32), ("window", ctypes.c_int32)]


_P, _I, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_PM, _PS = ctypes.POINTER(MainCacheDesc), ctypes.POINTER(SwaCacheDesc)

SIGNATURES = {
    "csa2_append_quant": (_I, [_PM, _P, _P, _P, _PS, _P, _P, _I, _P]),
    "csa2_append_quant_ex": (_I, [_PM, _P, _P, _P, _PS, _P, _P, _I, _P, _P, _I, _I, _P, _SZ, _P]),
    "csa2_append_project": (_I, [_PM, _P, _I, _P, _P, _P, _I, _P]),
    "csa2_index_full": (_I, [_PM, _P, _P, _P, _I, _I, _P, _I64, _P, _P, _SZ, _P]),
    "csa2_index_full_prepared": (_I, [_PM, _P, _I, _P, _I64, _P, _P, _SZ, _P]),
    "csa2_index_topk": (_I, [_PM, _P, _P, _P, _I, _I, _P, _I64, _P, _I, _P, _I, _P, _P, _P, _P, _SZ, _P]),
    "csa2_topk_merge": (_I, [_P, _P, _I, _I, _I, ctypes.POINTER(ctypes.c_int32), _I, _P, _P, _P]),
    "csa2_gather_entries": (_I, [_PM, _I, _P, _I, _P, _P, _I, _P, _P]),
    "csa2_index_topk_workspace_size": (_SZ, [_I, _I, _I]),
    "csa2_index_reindex": (_I, [_PM, _P, _P, _P, _I, _I, _P, _I, _P, _P, _SZ, _P]),
    "csa2_index_workspace_size": (_SZ, [_I, _I]),
    "csa2_topk": (_I, [_P, _I, _I64, _I, _P, _P, _I, _P, _I, _P, _P, _SZ, _P]),
    "csa2_topk_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "csa2_topk_noalloc": (_I, [_P, _I, _I64, _I, _P, _P, _I, _P, _I, _P, _P]),
    "csa2_sparse_attn_decode": (_I, [_PM, _PS, _P, _P, _I, _I, _P, _I, _F, _P, _P, _SZ, _P]),
    "csa2_attn_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "csa2_debug_inject_timeout": (None, [ctypes.c_uint32]),
    "csa2_last_error": (ctypes.c_char_p, []),
    "csa2_device_status": (_I, [_P, ctypes.POINTER(ctypes.c_uint32), _I]),
    "csa2_version": (_I, []),
}

_lib = None


def lib():
    """Load libcsa2.so (raises if it is missing: there is no other path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              f"`python -m fp4_kv_cache_append_b200.csrc.build` (or __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int):
    if status != CSA2_OK:
        raise Csa2Error(status, lib().csa2_last_error().decode())


_cuda = None


def _device_required() -> bool:
    """Whether tensors must live on a CUDA device: wherever CUDA is available
    (a host pointer handed to a kernel would fault the GPU).  Without CUDA the
    call goes on to the library, which reports that there is no device."""
    global _cuda
    if _cuda is None:
        _cuda = torch.cuda.is_available()
    return _cuda


def _check_device(device, what: str):
    """Where CUDA is available, `device` must be the current CUDA device: the
    kernels run there, and a pointer into another GPU's memory would be read
    across the link (or fault without peer access)."""
    if not _device_required():
        return
    if device.type != "cuda":
        raise ValueError(f"{what} must be CUDA device tensors (got one on {device})")
    cur = torch.cuda.current_device()
    if device.index is not None and device.index != cur:
        raise ValueError(f"{what} must be on the current device cuda:{cur} (got one on {device})")


def _ptr(t: torch.Tensor | None, dtype=None):
    if t is None:
        return None
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    _check_device(t.device, "tensors")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


# --------------------------------------------------------------------------- caches


class MainCache:
    """Device tensors of one FP4 main cache (layout of csa2_main_cache)."""

    def __init__(self, B, cap, D, d_I, m, device="cuda"):
        self.B, self.cap, self.D, self.d_I, self.m = B, cap, D, d_I, m
        self.codes = torch.zeros(B, cap, D // 2, dtype=torch.uint8, device=device)
        self.scales = torch.zeros(B, cap, D // 16, dtype=torch.uint8, device=device)
        self.ik = torch.zeros(B, cap, d_I, dtype=torch.uint8, device=device)
        self.ik_scale = torch.zeros(B, cap, dtype=torch.float32, device=device)
        self.n_entries = torch.zeros(B, dtype=torch.int32, device=device)
        self.pending_kv = torch.zeros(B, D, dtype=torch.bfloat16, device=device)
        self.pending_gate = torch.zeros(B, D, dtype=torch.bfloat16, device=device)

    def __setattr__(self, name, value):   # any change rebuilds the descriptor
        object.__setattr__(self, name, value)
        object.__setattr__(self, "_desc", None)

    def desc(self) -> MainCacheDesc:
        _check_device(self.codes.device, "the cache's planes")
        if self._desc is None:
            object.__setattr__(self, "_desc", MainCacheDesc(
                self.codes.data_ptr(), self.scales.data_ptr(), self.ik.data_ptr(), self.ik_scale.data_ptr(),
                self.n_entries.data_ptr(), self.pending_kv.data_ptr(), self.pending_gate.data_ptr(), self.B,
                self.cap, self.D, self.d_I, self.m))
        return self._desc

    @property
    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.codes, self.scales, self.ik, self.ik_scale, self.n_entries, self.pending_kv,
                    self.pending_gate))


class SwaCache:
    """Device ring of FP8 window rows of one layer (layout of csa2_swa_cache)."""

    def __init__(self, B, W_cap, D, scale=1.0, window=128, device="cuda"):
        self.B, self.W_cap, self.D, self.scale, self.window = B, W_cap, D, float(scale), window
        self.rows = torch.zeros(B, W_cap, D, dtype=torch.uint8, device=device)

    def __setattr__(self, name, value):   # any change rebuilds the descriptor
        object.__setattr__(self, name, value)
        object.__setattr__(self, "_desc", None)

    def desc(self) -> SwaCacheDesc:
        _check_device(self.rows.device, "the window cache's rows")
        if self._desc is None:
            object.__setattr__(self, "_desc", SwaCacheDesc(self.rows.data_ptr(), self.scale, self.B, self.W_cap,
                                                           self.D, self.window))
        return self._desc


# --------------------------------------------------------------------------- entry points


def csa2_append_quant(main: MainCache | None, kv, gate, w_ik, swa: SwaCache | None, kv_swa, pos0, T: int,
                      stream=None):
    md = ctypes.byref(main.desc()) if main is not None else None
    sd = ctypes.byref(swa.desc()) if swa is not None else None
    _check(lib().csa2_append_quant(md, _ptr(kv, torch.bfloat16), _ptr(gate, torch.bfloat16),
                                   _ptr(w_ik, torch.bfloat16), sd, _ptr(kv_swa, torch.bfloat16),
                                   _ptr(pos0, torch.int32), int(T), _stream(stream)))


def csa2_append_quant_ex(main: MainCache, kv, gate, w_ik, swa: SwaCache | None, kv_swa, pos0, T: int,
                         q_idx, w, ws, stream=None):
    """csa2_append_quant plus the preparation of the following scan's query
    (q_idx [B][T_q][H_I][d_I], w [B][T_q][H_I]) into ws."""
    sd = ctypes.byref(swa.desc()) if swa is not None else None
    T_q, H_I = q_idx.shape[-3], q_idx.shape[-2]
    _check(lib().csa2_append_quant_ex(ctypes.byref(main.desc()), _ptr(kv, torch.bfloat16), _ptr(gate, torch.bfloat16),
                                      _ptr(w_ik, torch.bfloat16), sd, _ptr(kv_swa, torch.bfloat16),
                                      _ptr(pos0, torch.int32), int(T), _ptr(q_idx, torch.bfloat16),
                                      _ptr(w, torch.float32), T_q, H_I, _ptr(ws), _nbytes(ws), _stream(stream)))


def csa2_append_project(main: MainCache, h, w_kv, w_ik, pos0, stream=None):
    """Projected append (CED producer): h [B][T][d_model] bf16, w_kv [d_model][D]."""
    T, d_model = h.shape[-2], h.shape[-1]
    _check(lib().csa2_append_project(ctypes.byref(main.desc()), _ptr(h, torch.bfloat16), int(d_model),
                                     _ptr(w_kv, torch.bfloat16), _ptr(w_ik, torch.bfloat16), _ptr(pos0, torch.int32),
                                     int(T), _stream(stream)))


def csa2_index_full_prepared(main: MainCache, q_pos, scores, n_valid=None, ws=None, stream=None):
    """csa2_index_full with the query prepared in ws by csa2_append_quant_ex."""
    T_q = q_pos.shape[-1]
    _check(lib().csa2_index_full_prepared(ctypes.byref(main.desc()), _ptr(q_pos, torch.int32), T_q,
                                          _ptr(scores, torch.float32), scores.shape[-1], _ptr(n_valid, torch.int32),
                                          _ptr(ws), _nbytes(ws), _stream(stream)))


def csa2_index_workspace_size(rows: int, d_I: int) -> int:
    return int(lib().csa2_index_workspace_size(rows, d_I))


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _ws_or_alloc(ws, nbytes, device):
    """A caller workspace, or a fresh one of the needed size (binding convenience)."""
    if ws is None:
        ws = workspace(nbytes, device)
    return ws


def csa2_index_full(main: MainCache, q_idx, w, q_pos, scores, n_valid=None, ws=None, stream=None):
    T_q = q_pos.shape[-1]
    H_I = q_idx.shape[-2]
    ws = _ws_or_alloc(ws, csa2_index_workspace_size(main.B * T_q, main.d_I), scores.device)
    _check(lib().csa2_index_full(ctypes.byref(main.desc()), _ptr(q_idx, torch.bfloat16), _ptr(w, torch.float32),
                                 _ptr(q_pos, torch.int32), T_q, H_I, _ptr(scores, torch.float32),
                                 scores.shape[-1], _ptr(n_valid, torch.int32), _ptr(ws), _nbytes(ws),
                                 _stream(stream)))


def csa2_index_topk_workspace_size(rows: int, cap: int, d_I: int) -> int:
    return int(lib().csa2_index_topk_workspace_size(rows, cap, d_I))


def csa2_index_topk(main: MainCache, q_idx, w, q_pos, scores, K: int, out_idx, n_valid=None, P_out: int = 0,
                    out_pool=None, out_scores=None, out_pool_scores=None, ws=None, stream=None):
    """Full scan fused with the first selection level, then Top-K and pool.
    q_idx and w None: the query was prepared in ws by csa2_append_quant_ex."""
    T_q = q_pos.shape[-1]
    H_I = q_idx.shape[-2] if q_idx is not None else 64
    ws = _ws_or_alloc(ws, csa2_index_topk_workspace_size(main.B * T_q, main.cap, main.d_I), scores.device)
    _check(lib().csa2_index_topk(ctypes.byref(main.desc()), _ptr(q_idx, torch.bfloat16), _ptr(w, torch.float32),
                                 _ptr(q_pos, torch.int32), T_q, H_I, _ptr(scores, torch.float32), scores.shape[-1],
                                 _ptr(n_valid, torch.int32), int(K), _ptr(out_idx, torch.int32), int(P_out),
                                 _ptr(out_pool, torch.int32), _ptr(out_scores, torch.float32),
                                 _ptr(out_pool_scores, torch.float32), _ptr(ws), _nbytes(ws), _stream(stream)))


def csa2_topk_merge(scores, ids, seg_base, K: int, out_ids, out_scores=None, stream=None):
    """scores, ids [G][rows][n_seg] device tensors; seg_base: G ints (host)."""
    G, rows, n_seg = scores.shape
    base = (ctypes.c_int32 * G)(*[int(x) for x in seg_base])
    _check(lib().csa2_topk_merge(_ptr(scores, torch.float32), _ptr(ids, torch.int32), G, rows, n_seg, base, int(K),
                                 _ptr(out_ids, torch.int32), _ptr(out_scores, torch.float32), _stream(stream)))


def csa2_gather_entries(shard: MainCache, lo: int, ids, out_codes, out_scales, out_pos=None, stream=None):
    """ids [B][K]; out_codes [B][out_cap][D/2], out_scales [B][out_cap][D/16]."""
    K = ids.shape[-1]
    _check(lib().csa2_gather_entries(ctypes.byref(shard.desc()), int(lo), _ptr(ids, torch.int32), K,
                                     _ptr(out_codes, torch.uint8), _ptr(out_scales, torch.uint8),
                                     out_codes.shape[1], _ptr(out_pos, torch.int32), _stream(stream)))


def csa2_index_reindex(main: MainCache, q_idx, w, q_pos, pool_blocks, pool_scores, ws=None, stream=None):
    T_q = q_pos.shape[-1]
    H_I = q_idx.shape[-2]
    ws = _ws_or_alloc(ws, csa2_index_workspace_size(main.B * T_q, main.d_I), pool_scores.device)
    _check(lib().csa2_index_reindex(ctypes.byref(main.desc()), _ptr(q_idx, torch.bfloat16), _ptr(w, torch.float32),
                                    _ptr(q_pos, torch.int32), T_q, H_I, _ptr(pool_blocks, torch.int32),
                                    pool_blocks.shape[-1], _ptr(pool_scores, torch.float32), _ptr(ws),
                                    _nbytes(ws), _stream(stream)))


def csa2_topk_workspace_size(rows: int, n_cols: int, K: int, P_out: int = 0) -> int:
    return int(lib().csa2_topk_workspace_size(rows, n_cols, K, P_out))


def csa2_topk(scores, n_cols: int, K: int, out_idx, n_valid=None, pool_blocks=None, P_out: int = 0,
              out_pool=None, ws=None, stream=None):
    rows = out_idx.shape[0]
    _check(lib().csa2_topk(_ptr(scores, torch.float32), rows, scores.shape[-1], int(n_cols),
                           _ptr(n_valid, torch.int32), _ptr(pool_blocks, torch.int32), int(K),
                           _ptr(out_idx, torch.int32), int(P_out), _ptr(out_pool, torch.int32),
                           _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def csa2_topk_noalloc(scores, n_cols: int, K: int, out_idx, n_valid=None, pool_blocks=None, P_out: int = 0,
                      out_pool=None, stream=None):
    """csa2_topk with the library's built-in scratch (no workspace argument)."""
    rows = out_idx.shape[0]
    _check(lib().csa2_topk_noalloc(_ptr(scores, torch.float32), rows, scores.shape[-1], int(n_cols),
                                   _ptr(n_valid, torch.int32), _ptr(pool_blocks, torch.int32), int(K),
                                   _ptr(out_idx, torch.int32), int(P_out), _ptr(out_pool, torch.int32),
                                   _stream(stream)))


def csa2_attn_workspace_size(B: int, T_q: int, H: int, D: int, K: int, window: int) -> int:
    return int(lib().csa2_attn_workspace_size(B, T_q, H, D, K, window))


def csa2_sparse_attn_decode(main: MainCache, swa: SwaCache, q, q_pos, idx, softmax_scale: float, out, ws=None,
                            stream=None):
    """idx None (or with a last dimension of 0): window-only attention (K = 0)."""
    T_q = q_pos.shape[-1]
    H = q.shape[-2]
    K = 0 if idx is None else idx.shape[-1]
    if K == 0:
        idx = None
    _check(lib().csa2_sparse_attn_decode(ctypes.byref(main.desc()), ctypes.byref(swa.desc()),
                                         _ptr(q, torch.bfloat16), _ptr(q_pos, torch.int32), T_q, H,
                                         _ptr(idx, torch.int32), K, float(softmax_scale),
                                         _ptr(out, torch.bfloat16), _ptr(ws),
                                         0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def csa2_device_status(clear: bool = True, stream=None) -> int:
    """Device status flags (CSA2_DEV_* bits) of the current device."""
    v = ctypes.c_uint32(0)
    st = lib().csa2_device_status(_stream(stream), ctypes.byref(v), 1 if clear else 0)
    if st not in (CSA2_OK, 4):
        _check(st)
    return int(v.value)


def csa2_debug_inject_timeout(polls: int):
    """Diagnostic: later indexer scans wait `polls` polls on a barrier nothing
    arrives on and take the give-up path (0 switches it off)."""
    lib().csa2_debug_inject_timeout(int(polls))


def csa2_version() -> int:
    return int(lib().csa2_version())


def workspace(nbytes: int, device="cuda") -> torch.Tensor | None:
    """A caller-owned workspace buffer (16-byte aligned torch allocation)."""
    if nbytes == 0:
        return None
    return torch.empty((nbytes + 15) // 16 * 16, dtype=torch.uint8, device=device)
