"""fp64 CPU oracle for DuoAttention's hybrid-head attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs
of ``bench.py`` may import this package.  It is independent of the CUDA library:
it imports nothing from ``head_split_kv_duo_b200`` and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over output rows);
this module only marshals numpy arrays.  Every function cites the passage of
"DuoAttention: Efficient Long-Context LLM Inference with Retrieval and Streaming
Heads" (arXiv 2410.10819) that it follows; the readings taken where the pages are
silent are listed at the top of ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F64, F32, BF16 = 0, 1, 2

# mutation codes understood by oracle_attend (used only to show that pins can fail)
MUTANTS = {
    "window_inclusive": 1,
    "sink_off_by_one": 2,
    "no_scale": 3,
    "non_causal": 4,
    "wrong_group": 5,
    "lse_no_max": 6,
    "v_from_k": 7,
}


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, no FMA contraction, no fast-math)."""
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, i32, dbl, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
            lib.oracle_attend.restype = i32
            lib.oracle_attend.argtypes = [i32, i64, i32, i32, i32, vp, i32, i64, vp, vp, i32, i64, vp, i64, i64,
                                          dbl, vp, i64, vp, vp, i32]
            lib.oracle_gated.restype = i32
            lib.oracle_gated.argtypes = [i32, i64, i32, i32, i32, vp, i32, vp, vp, i32, vp, i64, i64, dbl, vp, i64,
                                         vp]
            lib.oracle_visible.restype = i32
            lib.oracle_visible.argtypes = [i64, i64, i32, i64, i64]
            lib.oracle_retained.restype = None
            lib.oracle_retained.argtypes = [i64, i64, i64, vp]
            lib.oracle_ring_replay.restype = None
            lib.oracle_ring_replay.argtypes = [i64, i64, i32, vp, vp]
            lib.oracle_int4_quantize.restype = None
            lib.oracle_int4_quantize.argtypes = [i64, i32, vp, i32, vp, vp, vp]
            lib.oracle_int4_dequantize.restype = None
            lib.oracle_int4_dequantize.argtypes = [i64, i32, vp, vp, vp, vp]
            lib.oracle_fp8_quantize.restype = None
            lib.oracle_fp8_quantize.argtypes = [i64, i32, vp, i32, vp, vp]
            lib.oracle_fp8_dequantize.restype = None
            lib.oracle_fp8_dequantize.argtypes = [i64, i32, vp, vp, vp]
            lib.oracle_e4m3_value.restype = dbl
            lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
            lib.oracle_layer_kv_elems.restype = dbl
            lib.oracle_layer_kv_elems.argtypes = [i64, i64, i64, i64, i64, i64]
            lib.oracle_budget_ratio.restype = dbl
            lib.oracle_budget_ratio.argtypes = [dbl, dbl, dbl]
            lib.oracle_full_kv_bytes.restype = dbl
            lib.oracle_full_kv_bytes.argtypes = [i64, i64, i64, i64, i64]
            lib.oracle_num_threads.restype = i32
            lib.oracle_num_threads.argtypes = []
            _lib = lib
    return _lib


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use."""
    return int(_load().oracle_num_threads())


def _as_input(x: np.ndarray):
    """Return (contiguous array, dtype code).  uint16 arrays are bf16 bit patterns."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float64:
        return x, F64
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"oracle inputs must be float64, float32 or uint16 (bf16 bits), got {x.dtype}")


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def visible(i: int, j: int, is_retrieval: bool, S: int, W: int) -> bool:
    """Mask predicate: causal for retrieval heads, Lambda (sinks + last W) for streaming heads
    ("The Full and Streaming Attention Masks")."""
    return bool(_load().oracle_visible(i, j, int(bool(is_retrieval)), S, W))


def attend(q, k, v, retrieval, S: int, W: int, pos0: int, scale: float | None = None, rows=None,
           mutant: str | None = None):
    """Masked softmax attention over the dense history (the plain definition).

    q: [B][nq][Hq][d]; query row r is at absolute position pos0 + r.
    k, v: [B][Lk][Hkv][d], positions 0..Lk-1, nothing evicted.
    retrieval: [Hkv] booleans (True = full causal mask, False = Lambda mask).
    rows: optional flattened (b, r, h) row ids ((b*nq + r)*Hq + h) to evaluate.
    Returns (out [rows][d] or [B][nq][Hq][d] float64, lse [rows] or [B][nq][Hq] float64).
    """
    qa, qt = _as_input(q)
    ka, kt = _as_input(k)
    va, vt = _as_input(v)
    if kt != vt:
        raise TypeError("k and v must share a dtype")
    B, nq, Hq, d = qa.shape
    Bk, Lk, Hkv, dk = ka.shape
    if Bk != B or dk != d or va.shape != ka.shape or Hq % Hkv:
        raise ValueError("shape mismatch")
    retr = np.ascontiguousarray(np.asarray(retrieval, dtype=np.uint8).reshape(Hkv))
    if rows is None:
        n = B * nq * Hq
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n = rows_arr.size
    out = np.empty((n, d), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    rc = _load().oracle_attend(B, nq, Hq, Hkv, d, _ptr(qa), qt, pos0, _ptr(ka), _ptr(va), kt, Lk, _ptr(retr), S, W,
                               0.0 if scale is None else float(scale),
                               None if rows_arr is None else _ptr(rows_arr), n, _ptr(out), _ptr(lse),
                               MUTANTS[mutant] if mutant else 0)
    if rc != 0:
        raise ValueError(f"oracle_attend failed ({rc}): need pos0 + nq <= Lk")
    if rows is None:
        return out.reshape(B, nq, Hq, d), lse.reshape(B, nq, Hq)
    return out, lse


def gated(q, k, v, alpha, S: int, W: int, scale: float | None = None, rows=None):
    """Gated mixed attention over whole sequences: alpha[g] * causal attention +
    (1 - alpha[g]) * Lambda-masked attention, per KV head g (the plain definition).

    q: [B][L][Hq][d], k, v: [B][L][Hkv][d] (positions 0..L-1); alpha: [Hkv] floats.
    Returns out [rows][d] or [B][L][Hq][d] float64.
    """
    qa, qt = _as_input(q)
    ka, kt = _as_input(k)
    va, vt = _as_input(v)
    if kt != vt:
        raise TypeError("k and v must share a dtype")
    B, L, Hq, d = qa.shape
    if ka.shape[:2] != (B, L) or ka.shape[3] != d or va.shape != ka.shape or Hq % ka.shape[2]:
        raise ValueError("shape mismatch")
    Hkv = ka.shape[2]
    al = np.ascontiguousarray(np.asarray(alpha, dtype=np.float64).reshape(Hkv))
    if rows is None:
        n = B * L * Hq
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n = rows_arr.size
    out = np.empty((n, d), dtype=np.float64)
    rc = _load().oracle_gated(B, L, Hq, Hkv, d, _ptr(qa), qt, _ptr(ka), _ptr(va), kt, _ptr(al), S, W,
                              0.0 if scale is None else float(scale),
                              None if rows_arr is None else _ptr(rows_arr), n, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_gated failed ({rc})")
    return out.reshape(B, L, Hq, d) if rows is None else out


def retained(length: int, S: int, W: int) -> np.ndarray:
    """Closed-form retained set of a streaming head after `length` tokens (bool [length])."""
    m = np.zeros(max(length, 0), dtype=np.uint8)
    if length > 0:
        _load().oracle_retained(length, S, W, _ptr(m))
    return m.astype(bool)


def ring_replay(S: int, W: int, chunk_lens) -> np.ndarray:
    """Position held by each of the S+W slots after each chunk (int64 [nchunks][S+W], -1 = empty)."""
    lens = np.ascontiguousarray(np.asarray(chunk_lens, dtype=np.int64))
    out = np.empty((lens.size, S + W), dtype=np.int64)
    _load().oracle_ring_replay(S, W, int(lens.size), _ptr(lens), _ptr(out))
    return out


def int4_quantize(x):
    """Rows [nrows][gs] (float32 or bf16 bits as uint16) -> (codes uint8 [nrows][gs/2],
    scale fp16 bits uint16 [nrows], zero fp16 bits uint16 [nrows])."""
    xa, xt = _as_input(x)
    if xt == F64:
        raise TypeError("int4_quantize takes float32 or bf16 rows")
    nrows, gs = xa.reshape(-1, xa.shape[-1]).shape
    codes = np.empty((nrows, gs // 2), dtype=np.uint8)
    sb = np.empty((nrows,), dtype=np.uint16)
    zb = np.empty((nrows,), dtype=np.uint16)
    _load().oracle_int4_quantize(nrows, gs, _ptr(xa), xt, _ptr(codes), _ptr(sb), _ptr(zb))
    return codes, sb, zb


def int4_dequantize(codes, scale_bits, zero_bits) -> np.ndarray:
    """codes [nrows][gs/2] + fp16 scale/zero bits -> float64 [nrows][gs] (code*scale + zero)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    nrows, half = c.reshape(-1, c.shape[-1]).shape
    sb = np.ascontiguousarray(scale_bits, dtype=np.uint16).reshape(nrows)
    zb = np.ascontiguousarray(zero_bits, dtype=np.uint16).reshape(nrows)
    out = np.empty((nrows, 2 * half), dtype=np.float64)
    _load().oracle_int4_dequantize(nrows, 2 * half, _ptr(c), _ptr(sb), _ptr(zb), _ptr(out))
    return out


def fp8_quantize(x):
    """Rows [nrows][gs] (float32 or bf16 bits as uint16) -> (codes uint8 [nrows][gs] in OCP
    E4M3, scales float32 [nrows] = amax / 448); reading R14 of oracle.c."""
    xa, xt = _as_input(x)
    if xt == F64:
        raise TypeError("fp8_quantize takes float32 or bf16 rows")
    xa = xa.reshape(-1, xa.shape[-1])
    nrows, gs = xa.shape
    codes = np.empty((nrows, gs), dtype=np.uint8)
    scales = np.empty((nrows,), dtype=np.float32)
    _load().oracle_fp8_quantize(nrows, gs, _ptr(np.ascontiguousarray(xa)), xt, _ptr(codes), _ptr(scales))
    return codes, scales


def fp8_dequantize(codes, scales) -> np.ndarray:
    """codes [nrows][gs] E4M3 + fp32 scales [nrows] -> float64 [nrows][gs] (value * scale)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    c = c.reshape(-1, c.shape[-1])
    nrows, gs = c.shape
    sc = np.ascontiguousarray(scales, dtype=np.float32).reshape(nrows)
    out = np.empty((nrows, gs), dtype=np.float64)
    _load().oracle_fp8_dequantize(nrows, gs, _ptr(c), _ptr(sc), _ptr(out))
    return out


def e4m3_value(code: int) -> float:
    """Value of one OCP E4M3 code."""
    return float(_load().oracle_e4m3_value(int(code)))


def e4m3_encode(y: float) -> int:
    """Nearest OCP E4M3 code of a float (ties to even, held at +-448)."""
    return int(_load().oracle_e4m3_encode(float(y)))


def layer_kv_elems(Hr: int, Hs: int, L: int, S: int, W: int, d: int) -> float:
    """(H_r L + H_s (S+W)) d elements of K (or V) per layer ("Decoding Procedure")."""
    return float(_load().oracle_layer_kv_elems(Hr, Hs, L, S, W, d))


def budget_ratio(L: float, r: float, SW: float) -> float:
    """(L r + (S+W)(1 - r)) / L (OpenReview rebuttal, "RazorAttention and Echo Heads")."""
    return float(_load().oracle_budget_ratio(L, r, SW))


def full_kv_bytes(layers: int, heads: int, d: int, L: int, elem_bytes: int) -> float:
    """2 x layers x heads x L x d elements ("The Core Problem") times bytes per element."""
    return float(_load().oracle_full_kv_bytes(layers, heads, d, L, elem_bytes))
