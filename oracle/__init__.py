"""CSA2 oracle -- test infrastructure only.

A thin ctypes wrapper around ``csa2_oracle.c``, the plain CPU restatement of
the CSA2 sparse-attention step over an FP4 KV cache ("DeepSeek-V4.1-Flash:
Pushing the Limits of KV Cache Compression"; jaehun.me review, sections
"2) CSA2" and "3) FP4 main KV + SWA Bounded Replay").

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares nothing with the CUDA library
``fp4_kv_cache_append_b200`` and never imports it.

Arrays are numpy: bf16 tensors are passed as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa2_oracle.c")
_LIB = os.path.join(_HERE, "libcsa2_oracle.so")

# -ffp-contract=off: no implicit fused multiply-add; -mfma only makes the
# explicit fmaf() calls a single instruction (same correctly-rounded result).
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-mfma", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc if the library is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float

_SIGS = {
    "orc_bf16_to_f32": (_F, [ctypes.c_uint16]),
    "orc_f64_to_bf16": (ctypes.c_uint16, [ctypes.c_double]),
    "orc_e2m1_value": (ctypes.c_double, [_I]),
    "orc_e4m3_value": (ctypes.c_double, [_I]),
    "orc_e4m3_encode": (ctypes.c_uint8, [_F]),
    "orc_e2m1_encode": (ctypes.c_uint8, [_F]),
    "orc_exp_neg": (_F, [_F]),
    "orc_quant_fp4_row": (None, [_P, _I, _P, _P]),
    "orc_fp4_value": (ctypes.c_double, [_P, _P, _I]),
    "orc_pool_pair": (None, [_P, _P, _P, _P, _I, _P]),
    "orc_quant_fp8_row": (None, [_P, _I, _P, _P]),
    "orc_quant_query": (None, [_P, _I, _P, _P]),
    "orc_project_key": (None, [_P, _P, _P, _I, _I, _P]),
    "orc_index_key": (None, [_P, _P, _P, _I, _I, _P, _P]),
    "orc_append": (None, [_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P,
                          _P, _P, _P, _P, _I, _F, _P, _P, _I]),
    "orc_project_kv": (None, [_P, _I, _P, _I, _P]),
    "orc_append_project": (None, [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _I]),
    "orc_n_visible": (_I, [_I, _I, _I]),
    "orc_index_scores": (None, [_P, _P, _I, _I, _P, _P, _I, _P]),
    "orc_index_scores_at": (None, [_P, _P, _P, _I, _I, _P, _P, _I, _P]),
    "orc_topk": (None, [_P, _I, _I, _P]),
    "orc_block_pool": (None, [_P, _I, _I, _P]),
    "orc_reindex_scores": (None, [_P, _P, _I, _I, _P, _P, _I, _P, _I, _P]),
    "orc_columns_to_entries": (None, [_P, _I, _P, _P]),
    "orc_attention": (None, [_P, _I, _I, _P, _P, _I, _P, _I, _P, _I, _F, _I, _I, _F, _P]),
}


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        for name, (res, args) in _SIGS.items():
            fn = getattr(_lib, name)
            fn.restype = res
            fn.argtypes = args
    return _lib


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# scalar codecs
# --------------------------------------------------------------------------

def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(int(code))


def e4m3_value(byte: int) -> float:
    return lib().orc_e4m3_value(int(byte))


def e4m3_encode(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    f = lib().orc_e4m3_encode
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint8).reshape(x.shape)


def e2m1_encode(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    f = lib().orc_e2m1_encode
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint8).reshape(x.shape)


def exp_neg(x: float) -> float:
    return lib().orc_exp_neg(float(x))


def bf16_to_f32(h) -> np.ndarray:
    h = np.asarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


def f64_to_bf16(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    f = lib().orc_f64_to_bf16
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint16).reshape(x.shape)


# --------------------------------------------------------------------------
# row codecs
# --------------------------------------------------------------------------

def quant_fp4_row(x):
    x = _c(x, np.float32)
    D = x.shape[-1]
    codes = np.zeros(D // 2, np.uint8)
    scales = np.zeros(D // 16, np.uint8)
    lib().orc_quant_fp4_row(_p(x), D, _p(codes), _p(scales))
    return codes, scales


def fp4_dequant_row(codes, scales, D):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    f = lib().orc_fp4_value
    return np.array([f(_p(codes), _p(scales), c) for c in range(D)], dtype=np.float64)


def pool_pair(kv_a, kv_b, z_a, z_b):
    kv_a, kv_b, z_a, z_b = (_c(a, np.uint16) for a in (kv_a, kv_b, z_a, z_b))
    D = kv_a.shape[-1]
    out = np.zeros(D, np.float32)
    lib().orc_pool_pair(_p(kv_a), _p(kv_b), _p(z_a), _p(z_b), D, _p(out))
    return out


def quant_fp8_row(v):
    v = _c(v, np.float32)
    codes = np.zeros(v.shape[-1], np.uint8)
    s = np.zeros(1, np.float32)
    lib().orc_quant_fp8_row(_p(v), v.shape[-1], _p(codes), _p(s))
    return codes, s[0]


def quant_query(q):
    q = _c(q, np.uint16)
    codes = np.zeros(q.shape[-1], np.uint8)
    s = np.zeros(1, np.float32)
    lib().orc_quant_query(_p(q), q.shape[-1], _p(codes), _p(s))
    return codes, s[0]


def project_key(codes, scales, W):
    """The binary32 indexer key k = W^T x^ of one entry, before FP8."""
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    W = _c(W, np.uint16)
    D, dI = W.shape
    k = np.zeros(dI, np.float32)
    lib().orc_project_key(_p(codes), _p(scales), _p(W), D, dI, _p(k))
    return k


def index_key(codes, scales, W):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    W = _c(W, np.uint16)
    D, dI = W.shape
    ik = np.zeros(dI, np.uint8)
    s = np.zeros(1, np.float32)
    lib().orc_index_key(_p(codes), _p(scales), _p(W), D, dI, _p(ik), _p(s))
    return ik, s[0]


# --------------------------------------------------------------------------
# caches
# --------------------------------------------------------------------------

class MainCache:
    """Host copy of a main (FP4) cache: the same layout as the GPU one."""

    def __init__(self, B, cap, D, dI, m):
        self.B, self.cap, self.D, self.dI, self.m = B, cap, D, dI, m
        self.codes = np.zeros((B, cap, D // 2), np.uint8)
        self.scales = np.zeros((B, cap, D // 16), np.uint8)
        self.ik = np.zeros((B, cap, dI), np.uint8)
        self.ik_scale = np.zeros((B, cap), np.float32)
        self.n_entries = np.zeros(B, np.int32)
        self.pending_kv = np.zeros((B, D), np.uint16)
        self.pending_gate = np.zeros((B, D), np.uint16)


class SwaCache:
    def __init__(self, B, W_cap, D, scale=1.0, window=128):
        self.B, self.W_cap, self.D = B, W_cap, D
        self.scale = float(scale)
        self.window = window
        self.rows = np.zeros((B, W_cap, D), np.uint8)


def append(main: MainCache | None, kv, gate, W, swa: SwaCache | None, kv_swa, pos0, T):
    """Append T tokens per sequence (see orc_append)."""
    B = main.B if main is not None else swa.B
    D = main.D if main is not None else swa.D
    pos0 = _c(pos0, np.int32)
    kv = _c(kv, np.uint16) if kv is not None else None
    gate = _c(gate, np.uint16) if gate is not None else None
    W = _c(W, np.uint16) if W is not None else None
    kv_swa = _c(kv_swa, np.uint16) if kv_swa is not None else None
    lib().orc_append(
        B, main.cap if main else 0, D, main.dI if main else 0, main.m if main else 1,
        _p(main.codes) if main else None, _p(main.scales) if main else None,
        _p(main.ik) if main else None, _p(main.ik_scale) if main else None,
        _p(main.n_entries) if main else None,
        _p(main.pending_kv) if main else None, _p(main.pending_gate) if main else None,
        _p(kv), _p(gate), _p(W),
        _p(swa.rows) if swa else None, swa.W_cap if swa else 0,
        swa.scale if swa else 1.0, _p(kv_swa), _p(pos0), int(T))


def project_kv(h, W):
    """The decoder entry of one token: kv = h W_KV rounded once to binary32."""
    h = _c(h, np.uint16)
    W = _c(W, np.uint16)
    d, D = W.shape
    kv = np.zeros(D, np.float32)
    lib().orc_project_kv(_p(h), d, _p(W), D, _p(kv))
    return kv


def append_project(main: MainCache, H, W_kv, W_ik, pos0, T):
    """Project T tokens per sequence (H [B][T][d]) into an m = 1 main cache."""
    H = _c(H, np.uint16)
    W_kv = _c(W_kv, np.uint16)
    W_ik = _c(W_ik, np.uint16)
    pos0 = _c(pos0, np.int32)
    d = W_kv.shape[0]
    lib().orc_append_project(main.B, main.cap, main.D, main.dI, _p(main.codes), _p(main.scales), _p(main.ik),
                             _p(main.ik_scale), _p(main.n_entries), _p(H), d, _p(W_kv), _p(W_ik), _p(pos0), int(T))


def n_visible(n_entries: int, t: int, m: int) -> int:
    return lib().orc_n_visible(int(n_entries), int(t), int(m))


# --------------------------------------------------------------------------
# scoring, selection, attention
# --------------------------------------------------------------------------

def index_scores(main: MainCache, b: int, q_idx, w, n: int, entries=None):
    """Indexer scores of sequence b against entries 0..n-1 (or a list)."""
    q_idx = _c(q_idx, np.uint16)
    w = _c(w, np.float32)
    H_I, dI = q_idx.shape
    ik = main.ik[b]
    iks = main.ik_scale[b]
    if entries is None:
        out = np.zeros(n, np.float64)
        lib().orc_index_scores(_p(ik), _p(iks), n, dI, _p(q_idx), _p(w), H_I, _p(out))
    else:
        ent = _c(entries, np.int32)
        out = np.zeros(ent.size, np.float64)
        lib().orc_index_scores_at(_p(ik), _p(iks), _p(ent), ent.size, dI, _p(q_idx), _p(w), H_I, _p(out))
    return out


def topk(scores, K: int):
    s = _c(scores, np.float64)
    out = np.zeros(K, np.int32)
    lib().orc_topk(_p(s), s.size, K, _p(out))
    return out


def block_pool(scores, P: int):
    s = _c(scores, np.float64)
    out = np.zeros(P, np.int32)
    lib().orc_block_pool(_p(s), s.size, P, _p(out))
    return out


def reindex_scores(main: MainCache, b: int, q_idx, w, n_vis: int, pool):
    q_idx = _c(q_idx, np.uint16)
    w = _c(w, np.float32)
    pool = _c(pool, np.int32)
    H_I, dI = q_idx.shape
    out = np.zeros(pool.size * 8, np.float64)
    lib().orc_reindex_scores(_p(main.ik[b]), _p(main.ik_scale[b]), n_vis, dI, _p(q_idx), _p(w),
                             H_I, _p(pool), pool.size, _p(out))
    return out


def columns_to_entries(cols, pool):
    cols = _c(cols, np.int32)
    pool = _c(pool, np.int32)
    out = np.zeros(cols.size, np.int32)
    lib().orc_columns_to_entries(_p(cols), cols.size, _p(pool), _p(out))
    return out


def attention(main: MainCache, swa: SwaCache, b: int, q, idx, t: int, scale: float):
    """bf16 output [H][D] of one query token of sequence b at position t."""
    q = _c(q, np.uint16)
    idx = _c(idx, np.int32)
    H, D = q.shape
    out = np.zeros((H, D), np.uint16)
    lib().orc_attention(_p(q), H, D, _p(main.codes[b]), _p(main.scales[b]), main.cap,
                        _p(idx), idx.size, _p(swa.rows[b]), swa.W_cap, swa.scale, swa.window,
                        int(t), float(scale), _p(out))
    return out
