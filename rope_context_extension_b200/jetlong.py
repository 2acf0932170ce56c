"""Thin ctypes binding of libjetlong.so (include/jl_api.h), same names as the C ABI.

Argument marshalling only: tensors are torch CUDA tensors used as device
memory, their pointers and sizes go straight to the C entry points, and every
step of the computation runs in the library's kernels.  There is no CPU or
PyTorch fallback: if the shared library is missing, loading raises.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = [
    "JL_QSHIFT_NONE", "JL_QSHIFT_SELF_EXTEND", "JL_PREFILL_FP16", "JL_PREFILL_KEYS_IN_KERNEL", "JetLongError", "lib", "library_path",
    "jl_group_size", "jl_remote_positions", "jl_prefill_workspace_bytes", "jl_decode_workspace_bytes",
    "jl_bifocal_prefill", "jl_bifocal_decode", "jl_prefill_correction", "jl_prefill_attention",
    "jl_bifocal_decode_noalloc", "jl_bifocal_decode_varlen", "jl_rope_append", "jl_prefill_chunk_workspace_bytes",
    "jl_bifocal_prefill_chunk", "jl_prefill_ie_workspace_bytes", "jl_bifocal_prefill_ie", "jl_bifocal_decode_range",
    "jl_decode_combine", "jl_wait_timeout_check", "jl_prefill_tile_classes",
    "EXPORTED_SYMBOLS",
]

JL_QSHIFT_NONE = 0
JL_QSHIFT_SELF_EXTEND = 1
# Optional prefill flags OR-ed into mode (include/jl_api.h).  The default carries
# remote scores as fp16 hi + lo products: query rows corrected inside the attention
# kernel, key rows by a correction pass into the workspace.
JL_PREFILL_FP16 = 4            # one fp16 product per remote score from pre-rotated rows (workspace)
JL_PREFILL_KEYS_IN_KERNEL = 8  # default arithmetic, key tiles corrected inside the kernel too (no workspace)
EXPORTED_SYMBOLS = (
    "jl_status_string", "jl_group_size", "jl_remote_positions", "jl_prefill_workspace_bytes",
    "jl_bifocal_prefill", "jl_decode_workspace_bytes", "jl_bifocal_decode", "jl_prefill_correction",
    "jl_prefill_attention", "jl_bifocal_decode_noalloc", "jl_bifocal_decode_varlen", "jl_rope_append",
    "jl_prefill_chunk_workspace_bytes", "jl_bifocal_prefill_chunk", "jl_prefill_ie_workspace_bytes",
    "jl_bifocal_prefill_ie", "jl_bifocal_decode_range", "jl_decode_combine",
    "jl_wait_timeout_check", "jl_prefill_tile_classes",
)

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libjetlong.so")
_lib = None


class JetLongError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib().jl_status_string(status).decode()} ({status})")


def lib() -> ctypes.CDLL:
    """Load libjetlong.so (built in-tree); raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RuntimeError(f"{library_path} is missing: build it with `python -m rope_context_extension_b200.build`")
    L = ctypes.CDLL(library_path)
    c_i, c_i64, c_sz, c_p, c_d, c_f = (ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p,
                                       ctypes.c_double, ctypes.c_float)
    L.jl_status_string.argtypes = [c_i]
    L.jl_status_string.restype = ctypes.c_char_p
    L.jl_group_size.argtypes = [c_i64, c_i64, ctypes.POINTER(c_i64)]
    L.jl_group_size.restype = c_i
    L.jl_remote_positions.argtypes = [c_i64, c_i64, c_i64, c_i, c_p, c_p]
    L.jl_remote_positions.restype = c_i
    L.jl_prefill_tile_classes.argtypes = [c_i64, c_i64, c_i64, c_p]
    L.jl_prefill_tile_classes.restype = c_i
    L.jl_prefill_workspace_bytes.argtypes = [c_i, c_i, c_i, c_i, c_i]
    L.jl_prefill_workspace_bytes.restype = c_sz
    L.jl_decode_workspace_bytes.argtypes = [c_i, c_i, c_i, c_i, c_i]
    L.jl_decode_workspace_bytes.restype = c_sz
    L.jl_bifocal_prefill.argtypes = [c_p, c_p, c_p, c_p, c_p, c_i, c_i, c_i, c_i, c_i, c_i, c_i, c_d, c_f, c_i,
                                     c_p, c_sz, c_p, c_p]
    L.jl_bifocal_prefill.restype = c_i
    L.jl_prefill_correction.argtypes = [c_p, c_p, c_i, c_i, c_i, c_i, c_i, c_i, c_i, c_d, c_i, c_p, c_sz, c_p, c_p]
    L.jl_prefill_correction.restype = c_i
    L.jl_prefill_attention.argtypes = [c_p, c_p, c_p, c_p, c_p, c_i, c_i, c_i, c_i, c_i, c_i, c_i, c_d, c_f, c_i,
                                       c_p, c_sz, c_p, c_p]
    L.jl_prefill_attention.restype = c_i
    L.jl_bifocal_decode.argtypes = [c_p, c_p, c_p, c_i64, c_p, c_p, c_i, c_i, c_i, c_i, c_i, c_i, c_i, c_d, c_f,
                                    c_i, c_p, c_sz, c_p, c_p]
    L.jl_bifocal_decode.restype = c_i
    L.jl_bifocal_decode_noalloc.argtypes = [c_p, c_p, c_p, c_i64, c_p, c_p, c_i, c_i, c_i, c_i, c_i, c_i, c_i, c_d,
                                            c_f, c_i, c_p, c_p]
    L.jl_bifocal_decode_noalloc.restype = c_i
    L.jl_bifocal_decode_varlen.argtypes = [c_p, c_p, c_p, c_i64, c_p, c_i, c_p, c_p, c_i, c_i, c_i, c_i, c_i, c_i,
                                           c_d, c_f, c_i, c_p, c_sz, c_p, c_p]
    L.jl_bifocal_decode_varlen.restype = c_i
    L.jl_rope_append.argtypes = [c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_i64, c_i, c_i, c_i, c_i, c_d, c_p, c_p]
    L.jl_rope_append.restype = c_i
    L.jl_prefill_chunk_workspace_bytes.argtypes = [c_i, c_i, c_i, c_i, c_i, c_i]
    L.jl_prefill_chunk_workspace_bytes.restype = c_sz
    L.jl_bifocal_prefill_chunk.argtypes = [c_p, c_p, c_p, c_i64, c_p, c_p, c_i, c_i, c_i, c_i, c_i, c_i, c_i, c_i,
                                           c_d, c_f, c_i, c_p, c_sz, c_p, c_p]
    L.jl_bifocal_prefill_chunk.restype = c_i
    L.jl_prefill_ie_workspace_bytes.argtypes = [c_i, c_i, c_i, c_i, c_i, c_i]
    L.jl_prefill_ie_workspace_bytes.restype = c_sz
    L.jl_bifocal_prefill_ie.argtypes = list(L.jl_bifocal_prefill.argtypes)
    L.jl_bifocal_prefill_ie.restype = c_i
    L.jl_bifocal_decode_range.argtypes = [c_p, c_p, c_p, c_i64, c_i, c_i, c_i, c_p, c_p, c_i, c_i, c_i, c_i, c_i, c_i,
                                          c_d, c_f, c_i, c_p, c_sz, c_p, c_p]
    L.jl_bifocal_decode_range.restype = c_i
    L.jl_decode_combine.argtypes = [c_p, c_p, c_i, c_p, c_p, c_i, c_i, c_i, c_p]
    L.jl_decode_combine.restype = c_i
    L.jl_wait_timeout_check.argtypes = [c_p, c_d, c_p]
    L.jl_wait_timeout_check.restype = c_i
    _lib = L
    return L


def _check(status: int, where: str):
    if status != 0:
        raise JetLongError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ctypes.c_void_p(getattr(stream, "cuda_stream", stream))


def jl_group_size(L: int, w_pretrained: int) -> int:
    g = ctypes.c_int64(0)
    _check(lib().jl_group_size(L, w_pretrained, ctypes.byref(g)), "jl_group_size")
    return g.value


def jl_remote_positions(L: int, w0: int, w_pretrained: int, mode: int = JL_QSHIFT_SELF_EXTEND):
    """(p_q, f) as int32 numpy arrays of length L (host call)."""
    q = np.zeros(L, dtype=np.int32)
    k = np.zeros(L, dtype=np.int32)
    _check(lib().jl_remote_positions(L, w0, w_pretrained, mode, q.ctypes.data, k.ctypes.data),
           "jl_remote_positions")
    return q, k


def jl_prefill_tile_classes(L: int, w0: int, w_pretrained: int):
    """(local-only tiles, tiles with both passes, remote-only tiles, passes) of the
    prefill's 128 x 128 tile schedule over a length-L sequence (host call)."""
    out = np.zeros(4, dtype=np.int64)
    _check(lib().jl_prefill_tile_classes(L, w0, w_pretrained, out.ctypes.data), "jl_prefill_tile_classes")
    return tuple(int(x) for x in out)


def jl_prefill_workspace_bytes(B: int, L: int, Hq: int, Hkv: int, head_dim: int) -> int:
    return int(lib().jl_prefill_workspace_bytes(B, L, Hq, Hkv, head_dim))


def jl_decode_workspace_bytes(B: int, L: int, Hq: int, Hkv: int, head_dim: int) -> int:
    return int(lib().jl_decode_workspace_bytes(B, L, Hq, Hkv, head_dim))


def _check_tensor(t, name, dtype, shape=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def jl_bifocal_prefill(q, k, v, o, lse, *, w0: int, w_pretrained: int, rope_base: float,
                       softmax_scale: float = 0.0, mode: int = JL_QSHIFT_SELF_EXTEND, workspace=None,
                       dev_error=None, stream=None):
    """Fused bifocal prefill.  q [B, L, Hq, D], k / v [B, L, Hkv, D], o like q (bf16, CUDA);
    lse [B, Hq, L] fp32 or None; workspace: a uint8 CUDA tensor of
    jl_prefill_workspace_bytes(...) bytes (None with JL_PREFILL_KEYS_IN_KERNEL, or when
    every pair is local)."""
    import torch
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    _check_tensor(q, "q", torch.bfloat16)
    _check_tensor(k, "k", torch.bfloat16, (B, L, Hkv, D))
    _check_tensor(v, "v", torch.bfloat16, (B, L, Hkv, D))
    _check_tensor(o, "o", torch.bfloat16, (B, L, Hq, D))
    if lse is not None:
        _check_tensor(lse, "lse", torch.float32, (B, Hq, L))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().jl_bifocal_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, L, Hq, Hkv, D, int(w0),
                                  int(w_pretrained), float(rope_base), float(softmax_scale), int(mode),
                                  _ptr(workspace), ws_bytes, _ptr(dev_error), _stream(stream))
    _check(st, "jl_bifocal_prefill")


def jl_prefill_correction(q, k, *, w0: int, w_pretrained: int, rope_base: float,
                          mode: int = JL_QSHIFT_SELF_EXTEND, workspace=None, dev_error=None, stream=None):
    """Stage 1 of jl_bifocal_prefill: corrected Q / K rows into the workspace."""
    import torch
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    _check_tensor(q, "q", torch.bfloat16)
    _check_tensor(k, "k", torch.bfloat16, (B, L, Hkv, D))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().jl_prefill_correction(_ptr(q), _ptr(k), B, L, Hq, Hkv, D, int(w0), int(w_pretrained),
                                     float(rope_base), int(mode), _ptr(workspace), ws_bytes, _ptr(dev_error),
                                     _stream(stream))
    _check(st, "jl_prefill_correction")


def jl_prefill_attention(q, k, v, o, lse, *, w0: int, w_pretrained: int, rope_base: float,
                         softmax_scale: float = 0.0, mode: int = JL_QSHIFT_SELF_EXTEND, workspace=None,
                         dev_error=None, stream=None):
    """Stage 2 of jl_bifocal_prefill: the fused attention kernel."""
    import torch
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    _check_tensor(q, "q", torch.bfloat16)
    _check_tensor(k, "k", torch.bfloat16, (B, L, Hkv, D))
    _check_tensor(v, "v", torch.bfloat16, (B, L, Hkv, D))
    _check_tensor(o, "o", torch.bfloat16, (B, L, Hq, D))
    if lse is not None:
        _check_tensor(lse, "lse", torch.float32, (B, Hq, L))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().jl_prefill_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, L, Hq, Hkv, D, int(w0),
                                    int(w_pretrained), float(rope_base), float(softmax_scale), int(mode),
                                    _ptr(workspace), ws_bytes, _ptr(dev_error), _stream(stream))
    _check(st, "jl_prefill_attention")


def jl_bifocal_decode(q, k_cache, v_cache, o, lse, *, L: int, w0: int, w_pretrained: int, rope_base: float,
                      softmax_scale: float = 0.0, mode: int = JL_QSHIFT_SELF_EXTEND, workspace=None,
                      dev_error=None, stream=None):
    """Fused bifocal decode.  q / o [B, Hq, D]; caches [B, Lmax, Hkv, D] (bf16, CUDA);
    lse [B, Hq] fp32 or None; workspace: zero-initialised uint8 CUDA tensor of
    jl_decode_workspace_bytes(...) bytes."""
    import torch
    B, Hq, D = q.shape
    _, Lmax, Hkv, _ = k_cache.shape
    _check_tensor(q, "q", torch.bfloat16)
    _check_tensor(k_cache, "k_cache", torch.bfloat16)
    _check_tensor(v_cache, "v_cache", torch.bfloat16, tuple(k_cache.shape))
    _check_tensor(o, "o", torch.bfloat16, (B, Hq, D))
    if lse is not None:
        _check_tensor(lse, "lse", torch.float32, (B, Hq))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().jl_bifocal_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), Lmax, _ptr(o), _ptr(lse), B, int(L), Hq,
                                 Hkv, D, int(w0), int(w_pretrained), float(rope_base), float(softmax_scale),
                                 int(mode), _ptr(workspace), ws_bytes, _ptr(dev_error), _stream(stream))
    _check(st, "jl_bifocal_decode")


def jl_bifocal_decode_noalloc(q, k_cache, v_cache, o, lse, *, L: int, w0: int, w_pretrained: int,
                              rope_base: float, softmax_scale: float = 0.0, mode: int = JL_QSHIFT_SELF_EXTEND,
                              dev_error=None, stream=None):
    """jl_bifocal_decode for callers that cannot allocate device memory: the
    scratch is a fixed 4 MiB array inside the library (shared by every call on
    a device; calls that overlap on the GPU race).  Same tensors as
    jl_bifocal_decode, no workspace."""
    import torch
    B, Hq, D = q.shape
    _, Lmax, Hkv, _ = k_cache.shape
    _check_tensor(q, "q", torch.bfloat16)
    _check_tensor(k_cache, "k_cache", torch.bfloat16)
    _check_tensor(v_cache, "v_cache", torch.bfloat16, tuple(k_cache.shape))
    _check_tensor(o, "o", torch.bfloat16, (B, Hq, D))
    if lse is not None:
        _check_tensor(lse, "lse", torch.float32, (B, Hq))
    st = lib().jl_bifocal_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), Lmax, _ptr(o), _ptr(lse), B,
                                         int(L), Hq, Hkv, D, int(w0), int(w_pretrained), float(rope_base),
                                         float(softmax_scale), int(mode), _ptr(dev_error), _stream(stream))
    _check(st, "jl_bifocal_decode_noalloc")


def jl_bifocal_decode_varlen(q, k_cache, v_cache, o, lse, seq_lens, *, max_len: int, w0: int, w_pretrained: int,
                             rope_base: float, softmax_scale: float = 0.0, mode: int = JL_QSHIFT_SELF_EXTEND,
                             workspace=None, dev_error=None, stream=None):
    """Varlen decode: seq_lens is an int32 CUDA tensor [B] of per-sequence lengths
    (the new token of sequence b sits at seq_lens[b] - 1); max_len >= every length."""
    import torch
    B, Hq, D = q.shape
    _, Lmax, Hkv, _ = k_cache.shape
    _check_tensor(q, "q", torch.bfloat16)
    _check_tensor(k_cache, "k_cache", torch.bfloat16)
    _check_tensor(v_cache, "v_cache", torch.bfloat16, tuple(k_cache.shape))
    _check_tensor(o, "o", torch.bfloat16, (B, Hq, D))
    _check_tensor(seq_lens, "seq_lens", torch.int32, (B,))
    if lse is not None:
        _check_tensor(lse, "lse", torch.float32, (B, Hq))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().jl_bifocal_decode_varlen(_ptr(q), _ptr(k_cache), _ptr(v_cache), Lmax, _ptr(seq_lens), int(max_len),
                                        _ptr(o), _ptr(lse), B, Hq, Hkv, D, int(w0), int(w_pretrained),
                                        float(rope_base), float(softmax_scale), int(mode), _ptr(workspace),
                                        ws_bytes, _ptr(dev_error), _stream(stream))
    _check(st, "jl_bifocal_decode_varlen")


def jl_rope_append(q_raw, k_raw, v_new, positions, q_out, k_cache, v_cache, *, rope_base: float, dev_error=None,
                   stream=None):
    """Rotate each sequence's new token at positions[b] (int32 CUDA [B]) and append
    k / v to cache row positions[b]; q_out receives the rotated query."""
    import torch
    B, Hq, D = q_raw.shape
    _, Lmax, Hkv, _ = k_cache.shape
    _check_tensor(q_raw, "q_raw", torch.bfloat16)
    _check_tensor(k_raw, "k_raw", torch.bfloat16, (B, Hkv, D))
    _check_tensor(v_new, "v_new", torch.bfloat16, (B, Hkv, D))
    _check_tensor(positions, "positions", torch.int32, (B,))
    _check_tensor(q_out, "q_out", torch.bfloat16, (B, Hq, D))
    _check_tensor(k_cache, "k_cache", torch.bfloat16)
    _check_tensor(v_cache, "v_cache", torch.bfloat16, tuple(k_cache.shape))
    st = lib().jl_rope_append(_ptr(q_raw), _ptr(k_raw), _ptr(v_new), _ptr(positions), _ptr(q_out), _ptr(k_cache),
                              _ptr(v_cache), Lmax, B, Hq, Hkv, D, float(rope_base), _ptr(dev_error),
                              _stream(stream))
    _check(st, "jl_rope_append")


def jl_prefill_chunk_workspace_bytes(B: int, q_offset: int, chunk_len: int, Hq: int, Hkv: int, head_dim: int) -> int:
    return int(lib().jl_prefill_chunk_workspace_bytes(B, q_offset, chunk_len, Hq, Hkv, head_dim))


def jl_bifocal_prefill_chunk(q, k_cache, v_cache, o, lse, *, q_offset: int, w0: int, w_pretrained: int,
                             rope_base: float, softmax_scale: float = 0.0, mode: int = JL_QSHIFT_SELF_EXTEND,
                             workspace=None, dev_error=None, stream=None):
    """Chunked prefill: q [B, C, Hq, D] at positions q_offset..q_offset+C-1 against
    cache rows 0..q_offset+C-1 (the cache already holds the chunk's keys)."""
    import torch
    B, C, Hq, D = q.shape
    _, Lmax, Hkv, _ = k_cache.shape
    _check_tensor(q, "q", torch.bfloat16)
    _check_tensor(k_cache, "k_cache", torch.bfloat16)
    _check_tensor(v_cache, "v_cache", torch.bfloat16, tuple(k_cache.shape))
    _check_tensor(o, "o", torch.bfloat16, (B, C, Hq, D))
    if lse is not None:
        _check_tensor(lse, "lse", torch.float32, (B, Hq, C))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().jl_bifocal_prefill_chunk(_ptr(q), _ptr(k_cache), _ptr(v_cache), Lmax, _ptr(o), _ptr(lse), B,
                                        int(q_offset), C, Hq, Hkv, D, int(w0), int(w_pretrained), float(rope_base),
                                        float(softmax_scale), int(mode), _ptr(workspace), ws_bytes, _ptr(dev_error),
                                        _stream(stream))
    _check(st, "jl_bifocal_prefill_chunk")


def jl_prefill_ie_workspace_bytes(B: int, L: int, Hq: int, Hkv: int, head_dim: int,
                                  mode: int = JL_QSHIFT_SELF_EXTEND) -> int:
    return int(lib().jl_prefill_ie_workspace_bytes(B, L, Hq, Hkv, head_dim, mode))


def jl_bifocal_prefill_ie(q, k, v, o, lse, *, w0: int, w_pretrained: int, rope_base: float,
                          softmax_scale: float = 0.0, mode: int = JL_QSHIFT_SELF_EXTEND, workspace=None,
                          dev_error=None, stream=None):
    """The pages' three-call inclusion-exclusion prefill (unfused), same tensors as
    jl_bifocal_prefill; workspace of jl_prefill_ie_workspace_bytes(...) bytes."""
    import torch
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    _check_tensor(q, "q", torch.bfloat16)
    _check_tensor(k, "k", torch.bfloat16, (B, L, Hkv, D))
    _check_tensor(v, "v", torch.bfloat16, (B, L, Hkv, D))
    _check_tensor(o, "o", torch.bfloat16, (B, L, Hq, D))
    if lse is not None:
        _check_tensor(lse, "lse", torch.float32, (B, Hq, L))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().jl_bifocal_prefill_ie(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, L, Hq, Hkv, D, int(w0),
                                     int(w_pretrained), float(rope_base), float(softmax_scale), int(mode),
                                     _ptr(workspace), ws_bytes, _ptr(dev_error), _stream(stream))
    _check(st, "jl_bifocal_prefill_ie")


def jl_bifocal_decode_range(q, k_cache, v_cache, o, lse, *, key_offset: int, key_count: int, total_len: int, w0: int,
                            w_pretrained: int, rope_base: float, softmax_scale: float = 0.0,
                            mode: int = JL_QSHIFT_SELF_EXTEND, workspace=None, dev_error=None, stream=None):
    """Decode over cache rows holding positions key_offset..key_offset+key_count-1 of a
    sequence of total length total_len; o [B, Hq, D] bf16 and lse [B, Hq] fp32 are this
    range's normalised partial result."""
    import torch
    B, Hq, D = q.shape
    _, Lmax, Hkv, _ = k_cache.shape
    _check_tensor(q, "q", torch.bfloat16)
    _check_tensor(k_cache, "k_cache", torch.bfloat16)
    _check_tensor(v_cache, "v_cache", torch.bfloat16, tuple(k_cache.shape))
    _check_tensor(o, "o", torch.bfloat16, (B, Hq, D))
    _check_tensor(lse, "lse", torch.float32, (B, Hq))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().jl_bifocal_decode_range(_ptr(q), _ptr(k_cache), _ptr(v_cache), Lmax, int(key_offset), int(key_count),
                                       int(total_len), _ptr(o), _ptr(lse), B, Hq, Hkv, D, int(w0), int(w_pretrained),
                                       float(rope_base), float(softmax_scale), int(mode), _ptr(workspace), ws_bytes,
                                       _ptr(dev_error), _stream(stream))
    _check(st, "jl_bifocal_decode_range")


def jl_decode_combine(o_parts, lse_parts, o, lse, stream=None):
    """Log-sum-exp combine of partial results: o_parts [R, B, Hq, D] bf16,
    lse_parts [R, B, Hq] fp32 (CUDA) into o [B, Hq, D] and lse [B, Hq] (or None)."""
    import torch
    R, B, Hq, D = o_parts.shape
    _check_tensor(o_parts, "o_parts", torch.bfloat16)
    _check_tensor(lse_parts, "lse_parts", torch.float32, (R, B, Hq))
    _check_tensor(o, "o", torch.bfloat16, (B, Hq, D))
    if lse is not None:
        _check_tensor(lse, "lse", torch.float32, (B, Hq))
    st = lib().jl_decode_combine(_ptr(o_parts), _ptr(lse_parts), R, _ptr(o), _ptr(lse), B, Hq, D, _stream(stream))
    _check(st, "jl_decode_combine")


def jl_wait_timeout_check(dev_error, timeout_s: float = 0.2, stream=None):
    """Launch the bounded-wait self-test; dev_error is a device int32 tensor
    (read it after synchronising: 1 = the wait ran out as it should)."""
    import torch
    _check_tensor(dev_error, "dev_error", torch.int32)
    _check(lib().jl_wait_timeout_check(_ptr(dev_error), float(timeout_s), _stream(stream)), "jl_wait_timeout_check")
