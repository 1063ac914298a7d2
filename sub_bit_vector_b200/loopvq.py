"""ctypes binding of libloopvq (include/loopvq.h): argument marshalling only.

Every function has the name of the C entry point it calls.  Device buffers
are passed as torch tensors (their ``data_ptr()``); the stream defaults to
torch's current stream.  A non-OK status raises :class:`LoopVQError`.  All the
arithmetic runs in the library's CUDA kernels; if the shared library is
missing this module raises on import -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libloopvq.so")

LOOPVQ_OK = 0
LOOPVQ_ERR_INVALID_ARG = 1
LOOPVQ_ERR_UNSUPPORTED = 2
LOOPVQ_ERR_WORKSPACE_TOO_SMALL = 3
LOOPVQ_ERR_CUDA = 4
LOOPVQ_ERR_DEVICE_FAULT = 5

LOOPVQ_F32 = 0
LOOPVQ_BF16 = 1
LOOPVQ_KEYS = 0
LOOPVQ_VALUES = 1

LOOPVQ_FAULT_CODE_RANGE = 0x1
LOOPVQ_FAULT_CTX_RANGE = 0x2
LOOPVQ_FAULT_POOL_RANGE = 0x4
LOOPVQ_FAULT_TIMEOUT = 0x8

LOOPVQ_LAYOUT_STATIC_INPUTS = 0x1
LOOPVQ_LAYOUT_PAGED_BODY = 0x2
LOOPVQ_LAYOUT_RING_WINDOW = 0x4

EXPORTED = [
    "loopvq_version", "loopvq_status_string", "loopvq_validate_desc", "loopvq_ctx_split",
    "loopvq_bits_per_element",
    "loopvq_codebook_packed_bytes", "loopvq_codebook_pack", "loopvq_index_pool_bytes",
    "loopvq_index_pool_pack", "loopvq_index_pool_unpack", "loopvq_encode",
    "loopvq_codebook_update_workspace_bytes", "loopvq_codebook_update", "loopvq_codebook_grad",
    "loopvq_decode_workspace_bytes", "loopvq_decode_attn", "loopvq_decode_attn_noalloc",
    "loopvq_decode_steps_workspace_bytes", "loopvq_decode_attn_steps",
    "loopvq_residual_codes_bytes", "loopvq_residual_params_bytes", "loopvq_residual_encode",
    "loopvq_residual_decode_workspace_bytes", "loopvq_residual_decode_attn",
    "loopvq_read_device_status",
    "loopvq_clear_device_status", "loopvq_dense_decode_workspace_bytes", "loopvq_dense_decode_attn",
]


class LoopVQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {_status_text(status)} (status {status})")


class loopvq_codebook_desc(ctypes.Structure):
    _fields_ = [("n_loop", ctypes.c_int32), ("tc", ctypes.c_int32), ("n_heads_kv", ctypes.c_int32),
                ("n_heads_q", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("group_elems", ctypes.c_int32),
                ("n_codes", ctypes.c_int32), ("cb_dtype", ctypes.c_int)]


class loopvq_residual_desc(ctypes.Structure):
    _fields_ = [("n_loop", ctypes.c_int32), ("n_heads_kv", ctypes.c_int32), ("n_heads_q", ctypes.c_int32),
                ("head_dim", ctypes.c_int32)]


class loopvq_cache_layout(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_sink", ctypes.c_int32), ("n_recent", ctypes.c_int32),
                ("page", ctypes.c_int32), ("max_ctx_len", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("ctx_len", ctypes.c_void_p), ("body_off", ctypes.c_void_p), ("win_off", ctypes.c_void_p),
                ("body_pool_tokens", ctypes.c_int64), ("win_pool_tokens", ctypes.c_int64),
                ("body_pages", ctypes.c_void_p), ("body_page_tokens", ctypes.c_int32),
                ("max_body_pages", ctypes.c_int32), ("win_head", ctypes.c_void_p), ("win_ring", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("new_k", ctypes.c_void_p), ("new_v", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libloopvq.so not built ({LIB_PATH}); run python -m sub_bit_vector_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ, F, U8P = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                               ctypes.c_float, ctypes.c_void_p)
    D = ctypes.POINTER(loopvq_codebook_desc)
    L = ctypes.POINTER(loopvq_cache_layout)
    RD = ctypes.POINTER(loopvq_residual_desc)
    sig = {
        "loopvq_version": (ctypes.c_char_p, []),
        "loopvq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "loopvq_validate_desc": (ctypes.c_int, [D]),
        "loopvq_ctx_split": (ctypes.c_int, [I32, I32, I32, I32, ctypes.POINTER(I32), ctypes.POINTER(I32),
                                            ctypes.POINTER(I32)]),
        "loopvq_bits_per_element": (F, [D]),
        "loopvq_codebook_packed_bytes": (SZ, [D]),
        "loopvq_codebook_pack": (ctypes.c_int, [D, P, P, SZ, P]),
        "loopvq_index_pool_bytes": (SZ, [D, I64]),
        "loopvq_index_pool_pack": (ctypes.c_int, [D, ctypes.c_int, U8P, I64, U8P, I64, I64, P]),
        "loopvq_index_pool_unpack": (ctypes.c_int, [D, ctypes.c_int, U8P, I64, I64, I64, U8P, P]),
        "loopvq_encode": (ctypes.c_int, [D, P, ctypes.c_int, P, ctypes.c_int, I64, I64, I64, I64, U8P, I64, I64, P,
                                         P]),
        "loopvq_codebook_update_workspace_bytes": (SZ, [D]),
        "loopvq_codebook_update": (ctypes.c_int, [D, ctypes.c_int, P, ctypes.c_int, I64, I64, I64, I64, U8P, I64, I64,
                                                  P, P, P, P, SZ, P]),
        "loopvq_codebook_grad": (ctypes.c_int, [D, P, P, L, U8P, U8P, P, ctypes.c_int, I32, F, P, P, P, F, P, P,
                                                P, P, P]),
        "loopvq_residual_codes_bytes": (SZ, [RD, I64]),
        "loopvq_residual_params_bytes": (SZ, [RD, ctypes.c_int, I64]),
        "loopvq_residual_encode": (ctypes.c_int, [RD, ctypes.c_int, P, ctypes.c_int, I64, I64, I64, I64, U8P, P, I64,
                                                  I64, P]),
        "loopvq_residual_decode_workspace_bytes": (SZ, [RD, I32, I32]),
        "loopvq_residual_decode_attn": (ctypes.c_int, [RD, I32, I32, P, P, I64, U8P, P, U8P, P, P, ctypes.c_int, I32,
                                                       F, P, P, P, SZ, P]),
        "loopvq_decode_workspace_bytes": (SZ, [D, L]),
        "loopvq_decode_attn": (ctypes.c_int, [D, P, P, L, U8P, U8P, P, P, P, ctypes.c_int, I32, F, P,
                                              ctypes.c_int, P, P, SZ, P]),
        "loopvq_decode_steps_workspace_bytes": (SZ, [D, L, I32]),
        "loopvq_decode_attn_steps": (ctypes.c_int, [D, P, P, L, U8P, U8P, P, P, P, ctypes.c_int, I32, I32, F, P,
                                                    ctypes.c_int, P, P, SZ, P]),
        "loopvq_decode_attn_noalloc": (ctypes.c_int, [D, P, P, L, U8P, U8P, P, P, P, ctypes.c_int, I32, F, P,
                                                      ctypes.c_int, P, P, P]),
        "loopvq_read_device_status": (ctypes.c_int, [P, ctypes.POINTER(ctypes.c_uint32), P]),
        "loopvq_clear_device_status": (ctypes.c_int, [P, P]),
        "loopvq_dense_decode_workspace_bytes": (SZ, [I32, I32, I32, I32]),
        "loopvq_dense_decode_attn": (ctypes.c_int, [I32, I32, I32, I32, I32, P, P, I64, P, P, P, ctypes.c_int,
                                                    F, P, P, P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def _status_text(st: int) -> str:
    return _lib.loopvq_status_string(int(st)).decode()


def _check(fn: str, st: int) -> None:
    if st != LOOPVQ_OK:
        raise LoopVQError(fn, st)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return LOOPVQ_F32
    if t.dtype == torch.bfloat16:
        return LOOPVQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def make_desc(n_loop, tc, n_heads_kv, head_dim, group_elems, n_codes=256, n_heads_q=None,
              cb_dtype=LOOPVQ_BF16) -> loopvq_codebook_desc:
    return loopvq_codebook_desc(n_loop, tc, n_heads_kv, n_heads_q or n_heads_kv, head_dim, group_elems,
                                n_codes, cb_dtype)


def make_layout(batch, n_sink, n_recent, page, max_ctx_len, ctx_len, body_off, win_off,
                body_pool_tokens, win_pool_tokens, flags=0, body_pages=None, body_page_tokens=0,
                max_body_pages=0, win_head=None, win_ring=0, new_k=None, new_v=None) -> loopvq_cache_layout:
    lay = loopvq_cache_layout(batch, n_sink, n_recent, page, max_ctx_len, flags, _ptr(ctx_len), _ptr(body_off),
                              _ptr(win_off), body_pool_tokens, win_pool_tokens, _ptr(body_pages),
                              body_page_tokens, max_body_pages, _ptr(win_head), win_ring, 0, _ptr(new_k),
                              _ptr(new_v))
    # the struct holds raw device pointers: keep the arrays alive with it
    lay._keep = (ctx_len, body_off, win_off, body_pages, win_head, new_k, new_v)
    return lay


# ------------------------------------------------------------------ entry points

def loopvq_version() -> str:
    return _lib.loopvq_version().decode()


def loopvq_status_string(status: int) -> str:
    return _status_text(status)


def loopvq_validate_desc(desc) -> int:
    return _lib.loopvq_validate_desc(ctypes.byref(desc))


def loopvq_ctx_split(ctx_len, n_sink, n_recent, page):
    """Returns (sink, body, recent) token counts."""
    a, b, c = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check("loopvq_ctx_split", _lib.loopvq_ctx_split(ctx_len, n_sink, n_recent, page, ctypes.byref(a),
                                                     ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


def loopvq_bits_per_element(desc) -> float:
    return _lib.loopvq_bits_per_element(ctypes.byref(desc))


def loopvq_codebook_packed_bytes(desc) -> int:
    return _lib.loopvq_codebook_packed_bytes(ctypes.byref(desc))


def loopvq_codebook_pack(desc, canonical, packed, stream=None) -> None:
    _check("loopvq_codebook_pack", _lib.loopvq_codebook_pack(
        ctypes.byref(desc), _ptr(canonical), _ptr(packed), packed.numel() * packed.element_size(),
        _stream(stream)))


def loopvq_index_pool_bytes(desc, pool_tokens: int) -> int:
    return _lib.loopvq_index_pool_bytes(ctypes.byref(desc), pool_tokens)


def loopvq_index_pool_pack(desc, kind, codes, n_tokens, pool, tok_off, pool_tokens, stream=None) -> None:
    _check("loopvq_index_pool_pack", _lib.loopvq_index_pool_pack(
        ctypes.byref(desc), kind, _ptr(codes), n_tokens, _ptr(pool), tok_off, pool_tokens, _stream(stream)))


def loopvq_index_pool_unpack(desc, kind, pool, tok_off, pool_tokens, n_tokens, codes, stream=None) -> None:
    _check("loopvq_index_pool_unpack", _lib.loopvq_index_pool_unpack(
        ctypes.byref(desc), kind, _ptr(pool), tok_off, pool_tokens, n_tokens, _ptr(codes), _stream(stream)))


def loopvq_encode(desc, cb_packed, kind, x, n_tokens, stride_t, stride_n, stride_h, idx_pool, tok_off,
                  pool_tokens, stream=None, x_dtype=None, fault_bits=None) -> None:
    """fault_bits: an int32/uint32 device tensor of one element that receives
    the kernel's LOOPVQ_FAULT_* bits (OR-ed in), or None."""
    xd = _dtype_code(x) if x_dtype is None else x_dtype
    _check("loopvq_encode", _lib.loopvq_encode(
        ctypes.byref(desc), _ptr(cb_packed), kind, _ptr(x), xd, n_tokens, stride_t, stride_n, stride_h,
        _ptr(idx_pool), tok_off, pool_tokens, _ptr(fault_bits), _stream(stream)))


def loopvq_codebook_update_workspace_bytes(desc) -> int:
    return _lib.loopvq_codebook_update_workspace_bytes(ctypes.byref(desc))


def loopvq_codebook_update(desc, kind, x, n_tokens, stride_t, stride_n, stride_h, idx_pool, tok_off, pool_tokens,
                           cb_in, cb_out, counts_out, workspace, stream=None, x_dtype=None) -> None:
    xd = _dtype_code(x) if x_dtype is None else x_dtype
    _check("loopvq_codebook_update", _lib.loopvq_codebook_update(
        ctypes.byref(desc), kind, _ptr(x), xd, n_tokens, stride_t, stride_n, stride_h, _ptr(idx_pool), tok_off,
        pool_tokens, _ptr(cb_in), _ptr(cb_out), _ptr(counts_out) if counts_out is not None else None,
        _ptr(workspace), _nbytes(workspace), _stream(stream)))


def loopvq_codebook_grad(desc, cbK, cbV, layout, idxK_pool, idxV_pool, q, loop_step, softmax_scale, out, lse,
                         target, weight, gradK, gradV, loss_out=None, fault_bits=None, stream=None) -> None:
    """Adds the codebook gradients of weight * sum ||out - target||^2 at loop
    step ``loop_step`` to ``gradK``/``gradV`` (canonical fp32) and the loss to
    ``loss_out`` (one-element fp32 tensor, optional)."""
    _check("loopvq_codebook_grad", _lib.loopvq_codebook_grad(
        ctypes.byref(desc), _ptr(cbK), _ptr(cbV), ctypes.byref(layout), _ptr(idxK_pool), _ptr(idxV_pool), _ptr(q),
        _dtype_code(q), loop_step, softmax_scale, _ptr(out), _ptr(lse), _ptr(target), weight, _ptr(gradK),
        _ptr(gradV), _ptr(loss_out), _ptr(fault_bits), _stream(stream)))


def make_residual_desc(n_loop, n_heads_kv, head_dim, n_heads_q=None) -> loopvq_residual_desc:
    return loopvq_residual_desc(n_loop, n_heads_kv, n_heads_q or n_heads_kv, head_dim)


def loopvq_residual_codes_bytes(desc, pool_tokens) -> int:
    return _lib.loopvq_residual_codes_bytes(ctypes.byref(desc), pool_tokens)


def loopvq_residual_params_bytes(desc, kind, pool_tokens) -> int:
    return _lib.loopvq_residual_params_bytes(ctypes.byref(desc), kind, pool_tokens)


def loopvq_residual_encode(desc, kind, x, n_tokens, stride_t, stride_n, stride_h, codes, params, tok_off,
                           pool_tokens, stream=None, x_dtype=None) -> None:
    xd = _dtype_code(x) if x_dtype is None else x_dtype
    _check("loopvq_residual_encode", _lib.loopvq_residual_encode(
        ctypes.byref(desc), kind, _ptr(x), xd, n_tokens, stride_t, stride_n, stride_h, _ptr(codes), _ptr(params),
        tok_off, pool_tokens, _stream(stream)))


def loopvq_residual_decode_workspace_bytes(desc, batch, max_ctx_len) -> int:
    return _lib.loopvq_residual_decode_workspace_bytes(ctypes.byref(desc), batch, max_ctx_len)


def loopvq_residual_decode_attn(desc, batch, max_ctx_len, ctx_len, tok_off, pool_tokens, codesK, paramsK, codesV,
                                paramsV, q, loop_step, softmax_scale, out, lse_out, workspace, stream=None) -> None:
    _check("loopvq_residual_decode_attn", _lib.loopvq_residual_decode_attn(
        ctypes.byref(desc), batch, max_ctx_len, _ptr(ctx_len), _ptr(tok_off), pool_tokens, _ptr(codesK),
        _ptr(paramsK), _ptr(codesV), _ptr(paramsV), _ptr(q), _dtype_code(q), loop_step, softmax_scale, _ptr(out),
        _ptr(lse_out), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def loopvq_decode_workspace_bytes(desc, layout) -> int:
    return _lib.loopvq_decode_workspace_bytes(ctypes.byref(desc), ctypes.byref(layout))


def loopvq_decode_attn(desc, cbK_packed, cbV_packed, layout, idxK_pool, idxV_pool, winK, winV, q,
                       loop_step, softmax_scale, out, lse_out, workspace, stream=None,
                       workspace_bytes=None) -> None:
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("loopvq_decode_attn", _lib.loopvq_decode_attn(
        ctypes.byref(desc), _ptr(cbK_packed), _ptr(cbV_packed), ctypes.byref(layout), _ptr(idxK_pool),
        _ptr(idxV_pool), _ptr(winK), _ptr(winV), _ptr(q), _dtype_code(q), loop_step, softmax_scale,
        _ptr(out), _dtype_code(out), _ptr(lse_out), _ptr(workspace), wb, _stream(stream)))


def loopvq_decode_steps_workspace_bytes(desc, layout, n_steps) -> int:
    return _lib.loopvq_decode_steps_workspace_bytes(ctypes.byref(desc), ctypes.byref(layout), n_steps)


def loopvq_decode_attn_steps(desc, cbK_packed, cbV_packed, layout, idxK_pool, idxV_pool, winK, winV, q,
                             first_step, n_steps, softmax_scale, out, lse_out, workspace, stream=None) -> None:
    """Loop steps first_step .. first_step+n_steps-1 in one launch; q, out
    and lse_out carry a leading [n_steps] axis."""
    _check("loopvq_decode_attn_steps", _lib.loopvq_decode_attn_steps(
        ctypes.byref(desc), _ptr(cbK_packed), _ptr(cbV_packed), ctypes.byref(layout), _ptr(idxK_pool),
        _ptr(idxV_pool), _ptr(winK), _ptr(winV), _ptr(q), _dtype_code(q), first_step, n_steps, softmax_scale,
        _ptr(out), _dtype_code(out), _ptr(lse_out), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def prepare_decode_attn(desc, cbK_packed, cbV_packed, layout, idxK_pool, idxV_pool, winK, winV, q, loop_step,
                        softmax_scale, out, lse_out, workspace, stream=None):
    """loopvq_decode_attn with every argument marshalled once: returns a
    zero-argument callable that issues the call (for per-token loops where
    the buffers stay put and the Python-side argument conversion would cost
    more than the launch).  The tensors must stay alive and in place."""
    fn = _lib.loopvq_decode_attn
    args = (ctypes.byref(desc), _ptr(cbK_packed), _ptr(cbV_packed), ctypes.byref(layout), _ptr(idxK_pool),
            _ptr(idxV_pool), _ptr(winK), _ptr(winV), _ptr(q), _dtype_code(q), loop_step, softmax_scale, _ptr(out),
            _dtype_code(out), _ptr(lse_out), _ptr(workspace), _nbytes(workspace), _stream(stream))
    keep = (desc, layout)

    def call():
        st = fn(*args)
        if st != LOOPVQ_OK:
            raise LoopVQError("loopvq_decode_attn", st)
    call._keep = keep
    return call


def loopvq_decode_attn_noalloc(desc, cbK_packed, cbV_packed, layout, idxK_pool, idxV_pool, winK, winV, q,
                               loop_step, softmax_scale, out, lse_out, fault_bits=None, stream=None) -> None:
    """Same as loopvq_decode_attn but with no workspace: for callers that
    cannot allocate device memory (the library's fixed per-device scratch is
    used; calls must not overlap on the GPU).  ``fault_bits`` is an optional
    one-element uint32/int32 device tensor that receives the fault bits."""
    _check("loopvq_decode_attn_noalloc", _lib.loopvq_decode_attn_noalloc(
        ctypes.byref(desc), _ptr(cbK_packed), _ptr(cbV_packed), ctypes.byref(layout), _ptr(idxK_pool),
        _ptr(idxV_pool), _ptr(winK), _ptr(winV), _ptr(q), _dtype_code(q), loop_step, softmax_scale,
        _ptr(out), _dtype_code(out), _ptr(lse_out), _ptr(fault_bits), _stream(stream)))


def loopvq_read_device_status(workspace, stream=None):
    """Returns (status, fault_bits); waits for the stream."""
    bits = ctypes.c_uint32(0)
    st = _lib.loopvq_read_device_status(_ptr(workspace), ctypes.byref(bits), _stream(stream))
    if st not in (LOOPVQ_OK, LOOPVQ_ERR_DEVICE_FAULT):
        raise LoopVQError("loopvq_read_device_status", st)
    return st, bits.value


def loopvq_clear_device_status(workspace, stream=None) -> None:
    _check("loopvq_clear_device_status", _lib.loopvq_clear_device_status(_ptr(workspace), _stream(stream)))


def loopvq_dense_decode_workspace_bytes(batch, n_heads_q, head_dim, max_ctx_len) -> int:
    return _lib.loopvq_dense_decode_workspace_bytes(batch, n_heads_q, head_dim, max_ctx_len)


def loopvq_dense_decode_attn(batch, n_heads_kv, n_heads_q, head_dim, max_ctx_len, ctx_len, kv_off,
                             kv_pool_tokens, k, v, q, softmax_scale, out, lse_out, workspace,
                             stream=None) -> None:
    _check("loopvq_dense_decode_attn", _lib.loopvq_dense_decode_attn(
        batch, n_heads_kv, n_heads_q, head_dim, max_ctx_len, _ptr(ctx_len), _ptr(kv_off), kv_pool_tokens,
        _ptr(k), _ptr(v), _ptr(q), _dtype_code(q), softmax_scale, _ptr(out), _ptr(lse_out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
