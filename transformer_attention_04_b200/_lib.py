"""ctypes binding of libropeattn (include/ropeattn.h).

Argument marshalling only: tensors are checked for device, dtype, layout and shape,
and their data pointers plus the current CUDA stream are passed to the C ABI. Every
step of the computation runs in the library's CUDA kernels; there is no fallback,
and a missing library raises at first use.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libropeattn.so")

RA_OK, RA_ERR_INVALID_ARG, RA_ERR_UNSUPPORTED, RA_ERR_CUDA, RA_ERR_DEVICE_TIMEOUT = range(5)

# name -> (restype, argtypes), exactly the functions include/ropeattn.h declares
_P, _I, _F, _LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong
SIGNATURES = {
    "rope_attn_fwd": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "rope_attn_prefill": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I,
                               _P]),
    "rope_attn_rotate": (_I, [_P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "rope_attn_rotate_rows": (_I, [_P, _P, _I, _I, _I, _I, _F, _I, _I, _I, _P]),
    "rope_attn_fwd_partial": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I,
                                   _I, _I, _I, _I, _I, _I, _P]),
    "rope_attn_decode": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "rope_attn_decode_noalloc": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "rope_attn_decode_step": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I,
                                   _I, _P]),
    "rope_attn_decode_paged": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                    _F, _I, _I, _I, _P]),
    "rope_attn_decode_auto_splits": (_I, [_I, _I, _I, _I, _I, _I]),
    "rope_attn_get_device_status": (_I, [_P]),
    "rope_attn_set_wait_limit": (_LL, [_LL]),
    "rope_attn_status_string": (ctypes.c_char_p, [_I]),
    "rope_attn_last_cuda_error": (ctypes.c_char_p, []),
    "rope_attn_version": (_I, []),
    "rope_attn_profile_enable": (_I, [_I]),
    "rope_attn_profile_pause": (_I, [_I]),
    "rope_attn_profile_read": (_I, [_I, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I)]),
}

_lib = None


class RopeAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib().rope_attn_status_string(status).decode()
        super().__init__(f"{where}: status {status} ({msg})")
        self.status = status


def lib():
    """Load libropeattn.so (built in-tree by transformer_attention_04_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m transformer_attention_04_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype, fn.argtypes = res, args
        _lib = handle
    return _lib


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(t: torch.Tensor, name: str, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bfloat16")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (BHSD)")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _raise(status, where):
    if status != RA_OK:
        raise RopeAttnError(status, where)


def rope_attn_fwd(q, k, v, rope_base: float, pos_offset: int = 0, causal: bool = True,
                  out=None, stream=None):
    """Prefill attention. q [B,Hq,Sq,D], k/v [B,Hkv,Sk,D] bf16 CUDA; returns out [B,Hq,Sq,D]."""
    _check(q, "q")
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, H, S, D]")
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    _check(k, "k", (B, Hkv, Sk, D))
    _check(v, "v", (B, Hkv, Sk, D))
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", q.shape)
    st = lib().rope_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq, Hkv,
                             Sq, Sk, D, float(rope_base), int(pos_offset), int(bool(causal)),
                             _stream(stream))
    _raise(st, "rope_attn_fwd")
    return out


def rope_attn_prefill(q, k, v, rope_base: float, pos_offset: int = 0, causal: bool = True,
                      window: int = 0, k_cache_rot=None, v_cache=None, out=None, stream=None):
    """Prefill with an optional sliding window, optionally into a KV cache (chunked prefill).

    q [B,Hq,Sq,D], k/v [B,Hkv,Sk,D]. With caches [B,Hkv,S_cache,D] the chunk's rotated keys
    and values go to rows pos_offset.. and the queries attend all pos_offset+Sk cache rows.
    """
    _check(q, "q")
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, H, S, D]")
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    _check(k, "k", (B, Hkv, Sk, D))
    _check(v, "v", (B, Hkv, Sk, D))
    S_cache, kc, vc = 0, 0, 0
    if (k_cache_rot is None) != (v_cache is None):
        raise ValueError("give both caches or neither")
    if k_cache_rot is not None:
        S_cache = k_cache_rot.shape[2]
        _check(k_cache_rot, "k_cache_rot", (B, Hkv, S_cache, D))
        _check(v_cache, "v_cache", (B, Hkv, S_cache, D))
        kc, vc = k_cache_rot.data_ptr(), v_cache.data_ptr()
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", q.shape)
    st = lib().rope_attn_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), kc, vc,
                                 S_cache, B, Hq, Hkv, Sq, Sk, D, float(rope_base), int(pos_offset),
                                 int(bool(causal)), int(window), _stream(stream))
    _raise(st, "rope_attn_prefill")
    return out


def view_rows(shape, stride):
    """Rows between consecutive heads of a [B, H, S(, D)] layout whose rows are packed (a
    slice along S of a longer tensor qualifies), or None if the layout is not of that form."""
    B, H, S = shape[:3]
    row = shape[3] if len(shape) == 4 else 1
    if (len(shape) == 4 and stride[3] != 1 and row > 1) or (stride[2] != row and S > 1):
        return None
    if H > 1:
        if stride[1] % row:
            return None
        rows = stride[1] // row
    elif B > 1:
        if stride[0] % row:
            return None
        rows = stride[0] // row
    else:
        rows = S
    if rows < S or (B > 1 and stride[0] != H * rows * row):
        return None
    return rows


def _head_rows(t, name, dtype, shape):
    """view_rows of a CUDA tensor, after checking its dtype, device and shape."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != dtype:
        raise ValueError(f"{name} must be a {dtype} CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    rows = view_rows(tuple(shape), t.stride())
    if rows is None:
        raise ValueError(f"{name}: rows must be packed and heads evenly spaced slices of "
                         f">= {shape[2]} rows")
    return rows


def rope_attn_fwd_partial(q, k_rot, v, o_acc, lse_acc, rope_base: float, q_pos0: int,
                          k_pos0: int, causal: bool = True, accumulate: bool = False, out=None,
                          q_split: int = 0, q_pos1: int = 0, stream=None, chained: bool = False):
    """One ring-attention block: q [B,Hq,Sq,D] (rotated here to q_pos0+i; rows >= q_split at
    q_pos1 + (i - q_split) when 0 < q_split < Sq: masked calls need q_split a multiple of 128,
    of 256 for an odd group size, and q_pos1 >= k_pos0) against keys k_rot
    [B,Hkv,Sk,D] already rotated to k_pos0+j, and v. The block's normalised output and
    natural-log LSE go to o_acc [B,Hq,Sq,D] / lse_acc [B,Hq,Sq] (fp32), merged with their
    contents when ``accumulate``; ``out`` (bf16), if given, also receives the merged result.
    Every tensor may be a slice along the sequence axis of a longer one (q[:, :, a:b]).
    ``chained``: q, k_rot and v were complete before the previous kernel on the stream
    started (consecutive ring blocks whose keys were rotated up front); the block then runs
    alongside that kernel and waits for it only before its merge."""
    if q.dim() != 4 or k_rot.dim() != 4:
        raise ValueError("q, k_rot, v must be 4-D [B, H, S, D]")
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k_rot.shape[1], k_rot.shape[2]
    q_rows = _head_rows(q, "q", torch.bfloat16, (B, Hq, Sq, D))
    kv_rows = _head_rows(k_rot, "k_rot", torch.bfloat16, (B, Hkv, Sk, D))
    if _head_rows(v, "v", torch.bfloat16, (B, Hkv, Sk, D)) != kv_rows:
        raise ValueError("k_rot and v must have the same layout")
    acc_rows = _head_rows(o_acc, "o_acc", torch.float32, (B, Hq, Sq, D))
    if _head_rows(lse_acc, "lse_acc", torch.float32, (B, Hq, Sq)) != acc_rows:
        raise ValueError("o_acc and lse_acc must have the same row layout")
    o = 0
    if out is not None:
        if _head_rows(out, "out", torch.bfloat16, (B, Hq, Sq, D)) != acc_rows:
            raise ValueError("out must have the row layout of o_acc")
        o = out.data_ptr()
    st = lib().rope_attn_fwd_partial(q.data_ptr(), k_rot.data_ptr(), v.data_ptr(),
                                     o_acc.data_ptr(), lse_acc.data_ptr(), o, B, Hq, Hkv, Sq, Sk,
                                     D, float(rope_base), int(q_pos0), int(k_pos0),
                                     int(bool(causal)),
                                     (1 if accumulate else 0) | (2 if chained else 0), q_rows, kv_rows,
                                     acc_rows, int(q_split), int(q_pos1), _stream(stream))
    _raise(st, "rope_attn_fwd_partial")
    return out


def _check_pos(pos, B):
    if not isinstance(pos, torch.Tensor) or not pos.is_cuda or pos.dtype != torch.int32:
        raise ValueError("pos must be an int32 CUDA tensor")
    if tuple(pos.shape) != (B,) or not pos.is_contiguous():
        raise ValueError(f"pos must have shape ({B},)")


def rope_attn_decode_step(q, k_cache_rot, v_cache, pos, max_pos: int, rope_base: float,
                          k_new=None, v_new=None, window: int = 0, n_splits: int = 0, out=None,
                          stream=None):
    """Decode step at per-sequence positions pos [B] (int32, device), appending the new token
    (k_new/v_new [B,Hkv,1,D], keys not rotated) to the caches [B,Hkv,S_cache,D] at row pos[b]."""
    _check(q, "q")
    B, Hq, one, D = q.shape
    if one != 1:
        raise ValueError("decode takes one query row per head")
    Hkv, S_cache = k_cache_rot.shape[1], k_cache_rot.shape[2]
    _check(k_cache_rot, "k_cache_rot", (B, Hkv, S_cache, D))
    _check(v_cache, "v_cache", (B, Hkv, S_cache, D))
    _check_pos(pos, B)
    kn = vn = 0
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new or neither")
    if k_new is not None:
        _check(k_new, "k_new", (B, Hkv, 1, D))
        _check(v_new, "v_new", (B, Hkv, 1, D))
        kn, vn = k_new.data_ptr(), v_new.data_ptr()
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", q.shape)
    st = lib().rope_attn_decode_step(q.data_ptr(), kn, vn, k_cache_rot.data_ptr(),
                                     v_cache.data_ptr(), out.data_ptr(), pos.data_ptr(), B, Hq, Hkv,
                                     S_cache, D, float(rope_base), int(max_pos), int(window),
                                     int(n_splits), _stream(stream))
    _raise(st, "rope_attn_decode_step")
    return out


def rope_attn_decode_paged(q, k_pool_rot, v_pool, block_table, pos, max_pos: int,
                           rope_base: float, k_new=None, v_new=None, window: int = 0,
                           n_splits: int = 0, out=None, stream=None):
    """rope_attn_decode_step over a paged pool [num_blocks,Hkv,page,D] and a block table
    [B, max_blocks] (int32, device)."""
    _check(q, "q")
    B, Hq, one, D = q.shape
    if one != 1:
        raise ValueError("decode takes one query row per head")
    nb, Hkv, page = k_pool_rot.shape[0], k_pool_rot.shape[1], k_pool_rot.shape[2]
    _check(k_pool_rot, "k_pool_rot", (nb, Hkv, page, D))
    _check(v_pool, "v_pool", (nb, Hkv, page, D))
    _check_pos(pos, B)
    if (not isinstance(block_table, torch.Tensor) or not block_table.is_cuda or
            block_table.dtype != torch.int32 or block_table.dim() != 2 or
            block_table.shape[0] != B or not block_table.is_contiguous()):
        raise ValueError("block_table must be a contiguous int32 CUDA tensor [B, max_blocks]")
    kn = vn = 0
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new or neither")
    if k_new is not None:
        _check(k_new, "k_new", (B, Hkv, 1, D))
        _check(v_new, "v_new", (B, Hkv, 1, D))
        kn, vn = k_new.data_ptr(), v_new.data_ptr()
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", q.shape)
    st = lib().rope_attn_decode_paged(q.data_ptr(), kn, vn, k_pool_rot.data_ptr(),
                                      v_pool.data_ptr(), block_table.data_ptr(), out.data_ptr(),
                                      pos.data_ptr(), B, Hq, Hkv, D, page, block_table.shape[1], nb,
                                      float(rope_base), int(max_pos), int(window), int(n_splits),
                                      _stream(stream))
    _raise(st, "rope_attn_decode_paged")
    return out


def rope_attn_rotate(x, rope_base: float, pos_offset: int = 0, out=None, stream=None):
    """RoPE-rotate x [B,H,S,D] at positions pos_offset + s; out may be x (in place). x and out
    may be slices along the sequence axis of longer tensors (x[:, :, a:b])."""
    if not isinstance(x, torch.Tensor) or x.dim() != 4:
        raise ValueError("x must be a 4-D [B, H, S, D] tensor")
    B, H, S, D = x.shape
    x_rows = _head_rows(x, "x", torch.bfloat16, (B, H, S, D))
    if out is None:
        out = torch.empty_like(x, memory_format=torch.contiguous_format)
    out_rows = _head_rows(out, "out", torch.bfloat16, (B, H, S, D))
    st = lib().rope_attn_rotate_rows(x.data_ptr(), out.data_ptr(), B, H, S, D, float(rope_base),
                                     int(pos_offset), x_rows, out_rows, _stream(stream))
    _raise(st, "rope_attn_rotate")
    return out


def rope_attn_decode(q, k_cache_rot, v_cache, rope_base: float, pos: int, n_splits: int = 0,
                     out=None, stream=None):
    """One decode step. q [B,Hq,1,D]; caches [B,Hkv,Sk,D] (keys pre-rotated); returns out."""
    _check(q, "q")
    B, Hq, one, D = q.shape
    if one != 1:
        raise ValueError("decode takes one query row per head")
    Hkv, Sk = k_cache_rot.shape[1], k_cache_rot.shape[2]
    _check(k_cache_rot, "k_cache_rot", (B, Hkv, Sk, D))
    _check(v_cache, "v_cache", (B, Hkv, Sk, D))
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", q.shape)
    st = lib().rope_attn_decode(q.data_ptr(), k_cache_rot.data_ptr(), v_cache.data_ptr(),
                                out.data_ptr(), B, Hq, Hkv, Sk, D, float(rope_base), int(pos),
                                int(n_splits), _stream(stream))
    _raise(st, "rope_attn_decode")
    return out


def rope_attn_decode_noalloc(q, k_cache_rot, v_cache, rope_base: float, pos: int,
                             n_splits: int = 0, out=None, stream=None):
    """rope_attn_decode with its partials in the library's fixed device scratch (no device
    allocation per call); see the C header for the size limit and the sharing rules."""
    _check(q, "q")
    B, Hq, one, D = q.shape
    if one != 1:
        raise ValueError("decode takes one query row per head")
    Hkv, Sk = k_cache_rot.shape[1], k_cache_rot.shape[2]
    _check(k_cache_rot, "k_cache_rot", (B, Hkv, Sk, D))
    _check(v_cache, "v_cache", (B, Hkv, Sk, D))
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", q.shape)
    st = lib().rope_attn_decode_noalloc(q.data_ptr(), k_cache_rot.data_ptr(), v_cache.data_ptr(),
                                        out.data_ptr(), B, Hq, Hkv, Sk, D, float(rope_base),
                                        int(pos), int(n_splits), _stream(stream))
    _raise(st, "rope_attn_decode_noalloc")
    return out


def rope_attn_decode_auto_splits(B, Hq, Hkv, Sk, D, pos) -> int:
    return lib().rope_attn_decode_auto_splits(B, Hq, Hkv, Sk, D, pos)


def rope_attn_get_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the sticky kernel status."""
    return lib().rope_attn_get_device_status(_stream(stream))


def rope_attn_set_wait_limit(limit: int) -> int:
    return lib().rope_attn_set_wait_limit(int(limit))


def rope_attn_version() -> int:
    return lib().rope_attn_version()


def rope_attn_profile_enable(enable: bool = True) -> None:
    _raise(lib().rope_attn_profile_enable(int(bool(enable))), "rope_attn_profile_enable")


def rope_attn_profile_pause(pause: bool = True) -> None:
    """Stop (or resume) recording kernel events without ending the profiling session."""
    _raise(lib().rope_attn_profile_pause(int(bool(pause))), "rope_attn_profile_pause")


def rope_attn_profile_read(which: int):
    """(summed kernel ms, launches) since the last read; which 0 = prefill, 1 = decode."""
    ms, n = ctypes.c_double(0.0), ctypes.c_int(0)
    _raise(lib().rope_attn_profile_read(int(which), ctypes.byref(ms), ctypes.byref(n)),
           "rope_attn_profile_read")
    return ms.value, n.value
