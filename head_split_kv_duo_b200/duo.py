"""Python binding of the C-ABI library libduo.so (include/duo.h).

Argument marshalling only: every step of the attention path runs in the CUDA
kernels of libduo.so.  The module-level functions carry the C names and return the
C status code; ``DuoCache`` owns a torch device buffer for the cache and raises
``DuoError`` on any status other than DUO_OK.  Importing this module loads (and if
needed builds) libduo.so; there is no fallback when it cannot be loaded.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

DUO_OK, DUO_ERR_INVALID, DUO_ERR_CAPACITY, DUO_ERR_CUDA, DUO_ERR_TIMEOUT, DUO_ERR_UNSUPPORTED = range(6)
DUO_BF16, DUO_FP32 = 0, 1
DUO_KV_SAME, DUO_KV_INT4_G128, DUO_KV_FP8_E4M3 = 0, 1, 2
(DUO_REGION_RETR_K, DUO_REGION_RETR_V, DUO_REGION_RETR_KSZ, DUO_REGION_RETR_VSZ, DUO_REGION_STRM_K,
 DUO_REGION_STRM_V) = range(6)

_DTYPES = {torch.bfloat16: DUO_BF16, torch.float32: DUO_FP32}
_FMTS = {"same": DUO_KV_SAME, "int4": DUO_KV_INT4_G128, "fp8": DUO_KV_FP8_E4M3}


class duo_opts(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("q_heads", ctypes.c_int), ("dtype", ctypes.c_int),
                ("retr_fmt", ctypes.c_int), ("softmax_scale", ctypes.c_float)]


class DuoError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {duo_status_str(status)} ({status})")
        self.status = status


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libduo.so (built from csrc/ first if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            L = ctypes.CDLL(path, mode=os.RTLD_NOW | getattr(os, "RTLD_LOCAL", 0))
            vp, i32, i64, u64p = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.POINTER(ctypes.c_uint64)
            L.duo_cache_bytes.restype = ctypes.c_size_t
            L.duo_cache_bytes.argtypes = [i32, i32, i32, vp, i32, i32, i64, ctypes.POINTER(duo_opts)]
            L.duo_cache_create.restype = i32
            L.duo_cache_create.argtypes = [i32, i32, i32, vp, i32, i32, i64, ctypes.POINTER(duo_opts), vp,
                                           ctypes.c_size_t, ctypes.POINTER(vp)]
            L.duo_cache_destroy.restype = None
            L.duo_cache_destroy.argtypes = [vp]
            L.duo_append_kv.restype = i32
            L.duo_append_kv.argtypes = [vp, i32, vp, vp, i32, vp]
            L.duo_prefill_chunk.restype = i32
            L.duo_prefill_chunk.argtypes = [vp, i32, vp, vp, vp, i32, vp, vp, vp]
            L.duo_append_decode.restype = i32
            L.duo_append_decode.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp]
            L.duo_decode_attention.restype = i32
            L.duo_decode_attention.argtypes = [vp, i32, vp, vp, vp, vp]
            L.duo_cache_len.restype = i32
            L.duo_cache_len.argtypes = [vp, i32, ctypes.POINTER(i64)]
            L.duo_kv_bytes.restype = i32
            L.duo_kv_bytes.argtypes = [vp, i64, u64p, u64p]
            L.duo_debug_slot_position.restype = i32
            L.duo_debug_slot_position.argtypes = [vp, i32, i32, i32, ctypes.POINTER(i64)]
            L.duo_debug_region.restype = i32
            L.duo_debug_region.argtypes = [vp, i32, i32, ctypes.POINTER(vp), u64p, ctypes.POINTER(i64)]
            L.duo_get_device_status.restype = i32
            L.duo_get_device_status.argtypes = [vp, vp]
            L.duo_status_str.restype = ctypes.c_char_p
            L.duo_status_str.argtypes = [i32]
            L.duo_gated_attention.restype = i32
            L.duo_gated_attention.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, i32, i32,
                                              ctypes.c_float, vp, vp]
            L.duo_debug_launch_controls.restype = i32
            L.duo_debug_launch_controls.argtypes = [i32, i64]
            L.duo_debug_device_stall.restype = i32
            L.duo_debug_device_stall.argtypes = [i32]
            L.duo_pool_bytes.restype = ctypes.c_size_t
            L.duo_pool_bytes.argtypes = [i32, i32, i32, vp, i32, i32, i32, i64, i64, ctypes.POINTER(duo_opts)]
            L.duo_pool_create.restype = i32
            L.duo_pool_create.argtypes = [i32, i32, i32, vp, i32, i32, i32, i64, i64, ctypes.POINTER(duo_opts), vp,
                                          ctypes.c_size_t, ctypes.POINTER(vp)]
            L.duo_pool_destroy.restype = None
            L.duo_pool_destroy.argtypes = [vp]
            L.duo_pool_open.restype = i32
            L.duo_pool_open.argtypes = [vp, vp, ctypes.POINTER(i32)]
            L.duo_pool_close.restype = i32
            L.duo_pool_close.argtypes = [vp, i32]
            L.duo_pool_len.restype = i32
            L.duo_pool_len.argtypes = [vp, i32, i32, ctypes.POINTER(i64)]
            L.duo_pool_free_pages.restype = i32
            L.duo_pool_free_pages.argtypes = [vp, ctypes.POINTER(i64)]
            L.duo_pool_append_kv.restype = i32
            L.duo_pool_append_kv.argtypes = [vp, i32, i32, vp, vp, i32, vp]
            L.duo_pool_decode_step.restype = i32
            L.duo_pool_decode_step.argtypes = [vp, i32, i32, i32, ctypes.POINTER(i32), vp, vp, vp, vp, vp, vp]
            L.duo_pool_page.restype = i32
            L.duo_pool_page.argtypes = [vp, i32, i32, ctypes.POINTER(i32)]
            L.duo_pool_region.restype = i32
            L.duo_pool_region.argtypes = [vp, i32, i32, ctypes.POINTER(vp), u64p]
            L.duo_pool_device_status.restype = i32
            L.duo_pool_device_status.argtypes = [vp, vp]
            _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.data_ptr()
    return int(x)


def _mask_buf(mask):
    if isinstance(mask, torch.Tensor):
        mask = mask.to(torch.uint8).cpu().contiguous().flatten().tolist()
    else:
        import numpy as np
        mask = np.asarray(mask, dtype=np.uint8).flatten().tolist()
    return (ctypes.c_uint8 * len(mask))(*mask)


def _opts(batch=1, q_heads=0, dtype=DUO_BF16, retr_fmt=DUO_KV_SAME, softmax_scale=0.0):
    return duo_opts(batch, q_heads, dtype, retr_fmt, softmax_scale)


# ---- the C calls, same names ----

def duo_status_str(status: int) -> str:
    return lib().duo_status_str(status).decode()


def duo_cache_bytes(layers, kv_heads, head_dim, retrieval_head_mask, S, W, max_len, opts=None) -> int:
    m = _mask_buf(retrieval_head_mask)
    return int(lib().duo_cache_bytes(layers, kv_heads, head_dim, m, S, W, max_len,
                                     ctypes.byref(opts) if opts is not None else None))


def duo_cache_create(layers, kv_heads, head_dim, retrieval_head_mask, S, W, max_len, opts, dev_buf, dev_bytes):
    """Returns (status, handle)."""
    m = _mask_buf(retrieval_head_mask)
    h = ctypes.c_void_p()
    st = lib().duo_cache_create(layers, kv_heads, head_dim, m, S, W, max_len,
                                ctypes.byref(opts) if opts is not None else None, _ptr(dev_buf), int(dev_bytes),
                                ctypes.byref(h))
    return st, h


def duo_cache_destroy(handle):
    lib().duo_cache_destroy(handle)


def duo_append_kv(handle, layer, k, v, n, stream=None) -> int:
    return lib().duo_append_kv(handle, layer, _ptr(k), _ptr(v), n, _ptr(stream))


def duo_prefill_chunk(handle, layer, q, k, v, n, out, lse, stream=None) -> int:
    return lib().duo_prefill_chunk(handle, layer, _ptr(q), _ptr(k), _ptr(v), n, _ptr(out), _ptr(lse), _ptr(stream))


def duo_decode_attention(handle, layer, q, out, lse, stream=None) -> int:
    return lib().duo_decode_attention(handle, layer, _ptr(q), _ptr(out), _ptr(lse), _ptr(stream))


def duo_append_decode(handle, layer, q, k, v, out, lse, stream=None) -> int:
    return lib().duo_append_decode(handle, layer, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(stream))


def duo_cache_len(handle, layer):
    n = ctypes.c_int64()
    st = lib().duo_cache_len(handle, layer, ctypes.byref(n))
    return st, n.value


def duo_kv_bytes(handle, L):
    r, f = ctypes.c_uint64(), ctypes.c_uint64()
    st = lib().duo_kv_bytes(handle, L, ctypes.byref(r), ctypes.byref(f))
    return st, r.value, f.value


def duo_debug_slot_position(handle, layer, kv_head, slot):
    p = ctypes.c_int64()
    st = lib().duo_debug_slot_position(handle, layer, kv_head, slot, ctypes.byref(p))
    return st, p.value


def duo_debug_region(handle, layer, which):
    p, n, cap = ctypes.c_void_p(), ctypes.c_uint64(), ctypes.c_int64()
    st = lib().duo_debug_region(handle, layer, which, ctypes.byref(p), ctypes.byref(n), ctypes.byref(cap))
    return st, (p.value or 0), n.value, cap.value


def duo_get_device_status(handle, stream=None) -> int:
    return lib().duo_get_device_status(handle, _ptr(stream))


def duo_gated_attention(q, k, v, batch, seq_len, q_heads, kv_heads, head_dim, dtype, alpha, S, W, softmax_scale,
                        out, stream=None) -> int:
    return lib().duo_gated_attention(_ptr(q), _ptr(k), _ptr(v), batch, seq_len, q_heads, kv_heads, head_dim, dtype,
                                     _ptr(alpha), S, W, float(softmax_scale), _ptr(out), _ptr(stream))


def duo_debug_launch_controls(dry_run: int, fail_after: int) -> int:
    return lib().duo_debug_launch_controls(int(dry_run), int(fail_after))


def duo_debug_device_stall(on: int) -> int:
    return lib().duo_debug_device_stall(int(on))


def duo_pool_bytes(layers, kv_heads, head_dim, retrieval_head_mask, S, W, max_seqs, max_len, num_pages,
                   opts=None) -> int:
    m = _mask_buf(retrieval_head_mask)
    return int(lib().duo_pool_bytes(layers, kv_heads, head_dim, m, S, W, max_seqs, max_len, num_pages,
                                    ctypes.byref(opts) if opts is not None else None))


def duo_pool_create(layers, kv_heads, head_dim, retrieval_head_mask, S, W, max_seqs, max_len, num_pages, opts,
                    dev_buf, dev_bytes):
    """Returns (status, handle)."""
    m = _mask_buf(retrieval_head_mask)
    h = ctypes.c_void_p()
    st = lib().duo_pool_create(layers, kv_heads, head_dim, m, S, W, max_seqs, max_len, num_pages,
                               ctypes.byref(opts) if opts is not None else None, _ptr(dev_buf), int(dev_bytes),
                               ctypes.byref(h))
    return st, h


def duo_pool_destroy(handle):
    lib().duo_pool_destroy(handle)


def duo_pool_open(handle, stream=None):
    s = ctypes.c_int()
    st = lib().duo_pool_open(handle, _ptr(stream), ctypes.byref(s))
    return st, s.value


def duo_pool_close(handle, seq) -> int:
    return lib().duo_pool_close(handle, seq)


def duo_pool_len(handle, seq, layer):
    n = ctypes.c_int64()
    st = lib().duo_pool_len(handle, seq, layer, ctypes.byref(n))
    return st, n.value


def duo_pool_free_pages(handle):
    n = ctypes.c_int64()
    st = lib().duo_pool_free_pages(handle, ctypes.byref(n))
    return st, n.value


def duo_pool_append_kv(handle, layer, seq, k, v, n, stream=None) -> int:
    return lib().duo_pool_append_kv(handle, layer, seq, _ptr(k), _ptr(v), n, _ptr(stream))


def duo_pool_decode_step(handle, layer0, nlayers, seqs, q, k, v, out, lse, stream=None) -> int:
    arr = (ctypes.c_int * len(seqs))(*[int(x) for x in seqs])
    return lib().duo_pool_decode_step(handle, layer0, nlayers, len(seqs), arr, _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                      _ptr(lse), _ptr(stream))


def duo_pool_page(handle, seq, logical_page):
    p = ctypes.c_int()
    st = lib().duo_pool_page(handle, seq, logical_page, ctypes.byref(p))
    return st, p.value


def duo_pool_region(handle, layer, which):
    p, n = ctypes.c_void_p(), ctypes.c_uint64()
    st = lib().duo_pool_region(handle, layer, which, ctypes.byref(p), ctypes.byref(n))
    return st, (p.value or 0), n.value


def duo_pool_device_status(handle, stream=None) -> int:
    return lib().duo_pool_device_status(handle, _ptr(stream))


# ---- torch-owned cache ----

def _stream_ptr(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class DuoCache:
    """A hybrid-head KV cache whose device storage is one torch uint8 buffer."""

    def __init__(self, layers, kv_heads, head_dim, retrieval_mask, S, W, max_len, *, batch=1, q_heads=0,
                 dtype=torch.bfloat16, retr_fmt="same", softmax_scale=0.0, device="cuda"):
        self.layers, self.kv_heads, self.head_dim = layers, kv_heads, head_dim
        self.S, self.W, self.max_len, self.batch = S, W, max_len, batch
        self.q_heads = q_heads or kv_heads
        self.dtype = dtype
        self.mask = torch.as_tensor(retrieval_mask, dtype=torch.uint8).reshape(layers, kv_heads).clone()
        self.opts = _opts(batch, q_heads, _DTYPES[dtype], _FMTS[retr_fmt], softmax_scale)
        nbytes = duo_cache_bytes(layers, kv_heads, head_dim, self.mask, S, W, max_len, self.opts)
        if nbytes == 0:
            raise DuoError(DUO_ERR_INVALID, "duo_cache_bytes")
        self.nbytes = nbytes
        self.buffer = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        base = self.buffer.data_ptr()
        self._base = (base + 255) // 256 * 256
        st, self.handle = duo_cache_create(layers, kv_heads, head_dim, self.mask, S, W, max_len, self.opts,
                                           self._base, nbytes)
        if st != DUO_OK:
            raise DuoError(st, "duo_cache_create")

    def close(self):
        if getattr(self, "handle", None):
            duo_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, st, what):
        if st != DUO_OK:
            raise DuoError(st, what)

    def _want(self, t, shape, name, dtype=None):
        dtype = dtype or self.dtype
        if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name}: expected contiguous {dtype} CUDA tensor of shape {tuple(shape)}, "
                             f"got {t.dtype} {tuple(t.shape)}")

    def append_kv(self, layer, k, v, stream=None):
        n = k.shape[1]
        shape = (self.batch, n, self.kv_heads, self.head_dim)
        self._want(k, shape, "k")
        self._want(v, shape, "v")
        self._check(duo_append_kv(self.handle, layer, k, v, n, _stream_ptr(stream)), "duo_append_kv")

    def prefill_chunk(self, layer, q, k, v, out=None, lse=None, want_lse=True, stream=None):
        n = q.shape[1]
        self._want(q, (self.batch, n, self.q_heads, self.head_dim), "q")
        self._want(k, (self.batch, n, self.kv_heads, self.head_dim), "k")
        self._want(v, (self.batch, n, self.kv_heads, self.head_dim), "v")
        if out is None:
            out = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty(self.batch, n, self.q_heads, dtype=torch.float32, device=q.device)
        self._want(out, q.shape, "out")
        if lse is not None:
            self._want(lse, (self.batch, n, self.q_heads), "lse", torch.float32)
        self._check(duo_prefill_chunk(self.handle, layer, q, k, v, n, out, lse, _stream_ptr(stream)),
                    "duo_prefill_chunk")
        return out, lse

    def decode_attention(self, layer, q, out=None, lse=None, want_lse=True, stream=None):
        self._want(q, (self.batch, self.q_heads, self.head_dim), "q")
        if out is None:
            out = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty(self.batch, self.q_heads, dtype=torch.float32, device=q.device)
        self._want(out, q.shape, "out")
        if lse is not None:
            self._want(lse, (self.batch, self.q_heads), "lse", torch.float32)
        self._check(duo_decode_attention(self.handle, layer, q, out, lse, _stream_ptr(stream)),
                    "duo_decode_attention")
        return out, lse

    def append_decode(self, layer, q, k, v, out=None, lse=None, want_lse=True, stream=None):
        """duo_append_decode: append one token (k, v [B][1][Hkv][d]) and attend with q."""
        self._want(q, (self.batch, self.q_heads, self.head_dim), "q")
        self._want(k, (self.batch, 1, self.kv_heads, self.head_dim), "k")
        self._want(v, (self.batch, 1, self.kv_heads, self.head_dim), "v")
        if out is None:
            out = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty(self.batch, self.q_heads, dtype=torch.float32, device=q.device)
        self._want(out, q.shape, "out")
        if lse is not None:
            self._want(lse, (self.batch, self.q_heads), "lse", torch.float32)
        self._check(duo_append_decode(self.handle, layer, q, k, v, out, lse, _stream_ptr(stream)), "duo_append_decode")
        return out, lse

    def len(self, layer) -> int:
        st, n = duo_cache_len(self.handle, layer)
        self._check(st, "duo_cache_len")
        return n

    def kv_bytes(self, L):
        st, r, f = duo_kv_bytes(self.handle, L)
        self._check(st, "duo_kv_bytes")
        return r, f

    def slot_position(self, layer, kv_head, slot) -> int:
        st, p = duo_debug_slot_position(self.handle, layer, kv_head, slot)
        self._check(st, "duo_debug_slot_position")
        return p

    def device_status(self, stream=None) -> int:
        return duo_get_device_status(self.handle, _stream_ptr(stream))

    def region(self, layer, which):
        """uint8 view of one storage array of a layer (see duo_debug_region) and the
        retrieval token stride."""
        st, ptr, nbytes, cap = duo_debug_region(self.handle, layer, which)
        self._check(st, "duo_debug_region")
        off = ptr - self.buffer.data_ptr()
        return self.buffer[off:off + nbytes], cap


class DuoPool:
    """A paged pool of sequences (ragged batching) whose device storage is one torch uint8
    buffer: bf16, head_dim 128."""

    def __init__(self, layers, kv_heads, retrieval_mask, S, W, max_seqs, max_len, num_pages, *, q_heads=0,
                 softmax_scale=0.0, device="cuda"):
        self.layers, self.kv_heads, self.head_dim = layers, kv_heads, 128
        self.S, self.W, self.max_seqs, self.max_len, self.num_pages = S, W, max_seqs, max_len, num_pages
        self.q_heads = q_heads or kv_heads
        self.mask = torch.as_tensor(retrieval_mask, dtype=torch.uint8).reshape(layers, kv_heads).clone()
        self.opts = _opts(1, q_heads, DUO_BF16, DUO_KV_SAME, softmax_scale)
        nbytes = duo_pool_bytes(layers, kv_heads, 128, self.mask, S, W, max_seqs, max_len, num_pages, self.opts)
        if nbytes == 0:
            raise DuoError(DUO_ERR_INVALID, "duo_pool_bytes")
        self.buffer = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        base = (self.buffer.data_ptr() + 255) // 256 * 256
        st, self.handle = duo_pool_create(layers, kv_heads, 128, self.mask, S, W, max_seqs, max_len, num_pages,
                                          self.opts, base, nbytes)
        if st != DUO_OK:
            raise DuoError(st, "duo_pool_create")

    def close(self):
        if getattr(self, "handle", None):
            duo_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, st, what):
        if st != DUO_OK:
            raise DuoError(st, what)

    def open(self, stream=None) -> int:
        st, s = duo_pool_open(self.handle, _stream_ptr(stream))
        self._check(st, "duo_pool_open")
        return s

    def close_seq(self, seq):
        self._check(duo_pool_close(self.handle, seq), "duo_pool_close")

    def len(self, seq, layer) -> int:
        st, n = duo_pool_len(self.handle, seq, layer)
        self._check(st, "duo_pool_len")
        return n

    def free_pages(self) -> int:
        st, n = duo_pool_free_pages(self.handle)
        self._check(st, "duo_pool_free_pages")
        return n

    def append_kv(self, layer, seq, k, v, stream=None):
        """k, v [n][Hkv][128] bf16."""
        n = k.shape[0]
        for t, name in ((k, "k"), (v, "v")):
            if t.dtype != torch.bfloat16 or tuple(t.shape) != (n, self.kv_heads, 128) or not t.is_contiguous():
                raise ValueError(f"{name}: expected contiguous bf16 [{n}][{self.kv_heads}][128]")
        self._check(duo_pool_append_kv(self.handle, layer, seq, k, v, n, _stream_ptr(stream)), "duo_pool_append_kv")

    def decode_step(self, layer0, nlayers, seqs, q, k, v, out=None, lse=None, want_lse=True, stream=None):
        """q [nlayers][nseq][Hq][128], k, v [nlayers][nseq][Hkv][128] bf16 -> (out, lse)."""
        ns = len(seqs)
        for t, name, h in ((q, "q", self.q_heads), (k, "k", self.kv_heads), (v, "v", self.kv_heads)):
            if t.dtype != torch.bfloat16 or tuple(t.shape) != (nlayers, ns, h, 128) or not t.is_contiguous():
                raise ValueError(f"{name}: expected contiguous bf16 [{nlayers}][{ns}][{h}][128]")
        if out is None:
            out = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty(nlayers, ns, self.q_heads, dtype=torch.float32, device=q.device)
        self._check(duo_pool_decode_step(self.handle, layer0, nlayers, seqs, q, k, v, out, lse, _stream_ptr(stream)),
                    "duo_pool_decode_step")
        return out, lse

    def page(self, seq, logical_page) -> int:
        st, p = duo_pool_page(self.handle, seq, logical_page)
        self._check(st, "duo_pool_page")
        return p

    def region(self, layer, which):
        st, ptr, nbytes = duo_pool_region(self.handle, layer, which)
        self._check(st, "duo_pool_region")
        off = ptr - self.buffer.data_ptr()
        return self.buffer[off:off + nbytes]

    def device_status(self, stream=None) -> int:
        return duo_pool_device_status(self.handle, _stream_ptr(stream))


def gated_attention(q, k, v, alpha, S, W, softmax_scale=0.0, out=None, stream=None):
    """Gated mixed attention over whole sequences (duo_gated_attention): q [B][L][Hq][d],
    k, v [B][L][Hkv][d] (bf16 or fp32, CUDA), alpha [Hkv] fp32 on the same device."""
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    dt = {torch.bfloat16: DUO_BF16, torch.float32: DUO_FP32}.get(q.dtype)
    if dt is None or k.dtype != q.dtype or v.dtype != q.dtype or alpha.dtype != torch.float32:
        raise DuoError(DUO_ERR_INVALID, "gated_attention dtypes")
    for t in (q, k, v, alpha):
        if not t.is_contiguous() or t.device != q.device:
            raise DuoError(DUO_ERR_INVALID, "gated_attention inputs must be contiguous on one device")
    if out is None:
        out = torch.empty_like(q)
    st = duo_gated_attention(q, k, v, B, L, Hq, Hkv, d, dt, alpha, S, W, softmax_scale, out, _stream_ptr(stream))
    if st != DUO_OK:
        raise DuoError(st, "duo_gated_attention")
    return out
