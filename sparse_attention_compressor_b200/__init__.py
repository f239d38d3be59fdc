"""B200 (sm_100a) hybrid long-range attention forward of DeepSeek-V4 (CSA / HCA / sliding).

Thin Python binding of the C ABI in ``include/sac.h``: every function here marshals torch CUDA
tensors into pointers and calls the function of the same name in ``libsac.so``; all computation
runs in that library's CUDA kernels. There is no CPU path: calling into a missing or unbuilt
library raises.

Source: the "DeepSeek-V4" model documentation page (Hugging Face Transformers), sections "Hybrid
attention (section 2.3)", "Attention mask layout", "Cache layers", "DeepseekV4Config".
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsac.so")

SAC_F32, SAC_BF16 = 0, 1
SAC_KIND_SWA, SAC_KIND_HCA, SAC_KIND_CSA = 0, 1, 2
ABI_SYMBOLS = ("sac_last_error", "sac_version", "sac_workspace_size", "swa_forward",
               "hca_forward", "csa_forward", "sac_decode_workspace_size", "swa_decode",
               "hca_decode", "csa_decode", "sac_timing_begin", "sac_timing_end",
               "sac_static_scratch_bytes", "swa_forward_static", "sac_device_status",
               "decode_append", "sac_oproj_workspace_size", "o_proj_forward",
               "sac_chunk_workspace_size", "swa_prefill_chunk", "hca_prefill_chunk",
               "csa_prefill_chunk", "prefill_chunk_append")


class SacError(RuntimeError):
    """A non-zero status returned by the library, with its message."""

    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


class sac_params(ctypes.Structure):
    """Mirror of ``sac_params`` in include/sac.h."""
    _fields_ = [("B", ctypes.c_int), ("S", ctypes.c_int), ("H", ctypes.c_int),
                ("D", ctypes.c_int), ("R", ctypes.c_int), ("rope_theta", ctypes.c_double),
                ("m", ctypes.c_int), ("win_len", ctypes.c_int), ("sliding_window", ctypes.c_int),
                ("n_idx_heads", ctypes.c_int), ("idx_dim", ctypes.c_int), ("topk", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("pos0", ctypes.c_int64),
                ("dtype", ctypes.c_int), ("rope_factor", ctypes.c_double),
                ("rope_orig_max_pos", ctypes.c_int), ("yarn_beta_fast", ctypes.c_double),
                ("yarn_beta_slow", ctypes.c_double)]


def make_params(B: int, S: int, H: int, D: int, R: int, rope_theta: float, *, m: int = 0,
                win_len: int = 0, sliding_window: int = 128, n_idx_heads: int = 0,
                idx_dim: int = 0, topk: int = 0, softmax_scale: Optional[float] = None,
                pos0: int = 0, dtype: str = "bf16", rope_factor: float = 1.0,
                rope_orig_max_pos: int = 0, yarn_beta_fast: float = 32.0,
                yarn_beta_slow: float = 1.0) -> sac_params:
    scale = softmax_scale if softmax_scale is not None else D ** -0.5
    return sac_params(B, S, H, D, R, float(rope_theta), m, win_len, sliding_window, n_idx_heads,
                      idx_dim, topk, float(scale), int(pos0),
                      SAC_F32 if dtype in ("f32", "float32") else SAC_BF16, float(rope_factor),
                      int(rope_orig_max_pos), float(yarn_beta_fast), float(yarn_beta_slow))


class sac_kernel_time(ctypes.Structure):
    """Mirror of ``sac_kernel_time`` in include/sac.h."""
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int),
                ("total_ms", ctypes.c_double)]


_lib_handle = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libsac.so (raises if it is missing: build it with ``python -m
    sparse_attention_compressor_b200.build`` or ``__graft_entry__.build()``)."""
    global _lib_handle
    if _lib_handle is not None:
        return _lib_handle
    if not os.path.exists(path):
        raise RuntimeError(f"libsac.so not found at {path}; the CUDA library must be built")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(sac_params)
    vp, sz, i32p, fp = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p
    ci = ctypes.c_int
    lib.sac_last_error.restype = ctypes.c_char_p
    lib.sac_version.restype = ci
    lib.sac_workspace_size.restype = sz
    lib.sac_workspace_size.argtypes = [P, ci]
    lib.sac_decode_workspace_size.restype = sz
    lib.sac_decode_workspace_size.argtypes = [P, ci, ci]
    lib.swa_forward.argtypes = [P, vp, vp, fp, vp, vp, sz, vp]
    lib.hca_forward.argtypes = [P, vp, vp, vp, fp, fp, vp, vp, vp, sz, vp]
    lib.csa_forward.argtypes = [P, vp, vp, vp, fp, vp, fp, vp, vp, fp, fp, vp, i32p, vp, vp, vp,
                                sz, vp]
    lib.swa_decode.argtypes = [P, ci, vp, vp, i32p, ci, i32p, ci, fp, vp, vp, sz, vp]
    lib.hca_decode.argtypes = [P, ci, vp, vp, i32p, ci, i32p, ci, vp, i32p, ci, fp, vp, vp, sz,
                               vp]
    lib.csa_decode.argtypes = [P, ci, vp, vp, i32p, ci, i32p, ci, vp, vp, i32p, ci, vp, fp, fp,
                               vp, i32p, vp, sz, vp]
    lib.decode_append.argtypes = [P, ci, ci, i32p, vp, vp, vp, fp, vp, fp, vp, i32p, ci, ci, vp,
                                  vp, vp, vp, i32p, ci, vp]
    lib.sac_chunk_workspace_size.restype = sz
    lib.sac_chunk_workspace_size.argtypes = [P, ci, ci, ci]
    for name, decode_name in (("swa_prefill_chunk", "swa_decode"),
                              ("hca_prefill_chunk", "hca_decode"),
                              ("csa_prefill_chunk", "csa_decode")):
        fn = getattr(lib, name)  # the decode signature with n after nseq
        dec = getattr(lib, decode_name).argtypes
        fn.argtypes = dec[:2] + [ci] + dec[2:]
    lib.prefill_chunk_append.argtypes = lib.decode_append.argtypes[:3] + [ci] + \
        lib.decode_append.argtypes[3:]
    lib.sac_oproj_workspace_size.restype = sz
    lib.sac_oproj_workspace_size.argtypes = [P, ctypes.c_int64, ci, ci]
    lib.o_proj_forward.restype = ci
    lib.o_proj_forward.argtypes = [P, ctypes.c_int64, ci, ci, ci, vp, vp, vp, vp, vp, sz, vp]
    lib.sac_device_status.restype = ci
    lib.sac_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int), vp]
    lib.sac_static_scratch_bytes.restype = sz
    lib.swa_forward_static.restype = ci
    lib.swa_forward_static.argtypes = [P, vp, vp, fp, vp, vp]
    lib.sac_timing_begin.restype = ci
    lib.sac_timing_end.restype = ci
    lib.sac_timing_end.argtypes = [ctypes.POINTER(sac_kernel_time), ci]
    for name in ("swa_forward", "hca_forward", "csa_forward", "swa_decode", "hca_decode",
                 "csa_decode", "decode_append"):
        getattr(lib, name).restype = ci
    _lib_handle = lib
    return lib


def _ptr(t) -> Optional[int]:
    """Device pointer of a CUDA tensor (None passes NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("the library takes CUDA tensors (device pointers)")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise SacError(fn, rc, load_library().sac_last_error().decode())


def _nbytes(ws) -> int:
    return 0 if ws is None else ws.numel() * ws.element_size()


def sac_version() -> int:
    return int(load_library().sac_version())


def sac_workspace_size(p: sac_params, kind: int) -> int:
    return int(load_library().sac_workspace_size(ctypes.byref(p), kind))


def sac_decode_workspace_size(p: sac_params, kind: int, nseq: int) -> int:
    return int(load_library().sac_decode_workspace_size(ctypes.byref(p), kind, nseq))


def sac_timing_begin() -> None:
    _check("sac_timing_begin", load_library().sac_timing_begin())


def sac_timing_end(max_entries: int = 32) -> dict:
    """{kernel name: (launches, total device ms)} since sac_timing_begin()."""
    buf = (sac_kernel_time * max_entries)()
    n = load_library().sac_timing_end(buf, max_entries)
    if n < 0:
        _check("sac_timing_end", n)
    return {buf[i].name.decode(): (buf[i].launches, buf[i].total_ms)
            for i in range(min(n, max_entries))}


def swa_forward(p, q, kv, sinks, o, ws, stream=None) -> None:
    _check("swa_forward", load_library().swa_forward(
        ctypes.byref(p), _ptr(q), _ptr(kv), _ptr(sinks), _ptr(o), _ptr(ws), _nbytes(ws),
        _stream(stream)))


def sac_device_status(ws, stream=None) -> int:
    """Status word of the last prefill call on workspace ws (0 = ok); waits for the stream."""
    out = ctypes.c_int(-1)
    _check("sac_device_status", load_library().sac_device_status(_ptr(ws), ctypes.byref(out),
                                                                 _stream(stream)))
    return out.value


def sac_static_scratch_bytes() -> int:
    return int(load_library().sac_static_scratch_bytes())


def swa_forward_static(p, q, kv, sinks, o, stream=None) -> None:
    """swa_forward with the library's fixed scratch array instead of a caller workspace: for
    callers that cannot allocate device memory (see include/sac.h)."""
    _check("swa_forward_static", load_library().swa_forward_static(
        ctypes.byref(p), _ptr(q), _ptr(kv), _ptr(sinks), _ptr(o), _stream(stream)))


def hca_forward(p, q, kv, cmp_gate, cmp_bias, sinks, o, pool_out, ws, stream=None) -> None:
    _check("hca_forward", load_library().hca_forward(
        ctypes.byref(p), _ptr(q), _ptr(kv), _ptr(cmp_gate), _ptr(cmp_bias), _ptr(sinks), _ptr(o),
        _ptr(pool_out), _ptr(ws), _nbytes(ws), _stream(stream)))


def csa_forward(p, q, kv, cmp_gate, cmp_bias, q_idx, w_idx, k_idx, idx_gate, idx_bias, sinks, o,
                topk_out, pool_out, idx_pool_out, ws, stream=None) -> None:
    _check("csa_forward", load_library().csa_forward(
        ctypes.byref(p), _ptr(q), _ptr(kv), _ptr(cmp_gate), _ptr(cmp_bias), _ptr(q_idx),
        _ptr(w_idx), _ptr(k_idx), _ptr(idx_gate), _ptr(idx_bias), _ptr(sinks), _ptr(o),
        _ptr(topk_out), _ptr(pool_out), _ptr(idx_pool_out), _ptr(ws), _nbytes(ws),
        _stream(stream)))


def swa_decode(p, nseq, q, kv_pages, kv_block_table, ctx_lens, page_size, sinks, o, ws=None,
               stream=None) -> None:
    _check("swa_decode", load_library().swa_decode(
        ctypes.byref(p), nseq, _ptr(q), _ptr(kv_pages), _ptr(kv_block_table),
        kv_block_table.shape[1], _ptr(ctx_lens), page_size, _ptr(sinks), _ptr(o), _ptr(ws),
        _nbytes(ws), _stream(stream)))


def hca_decode(p, nseq, q, kv_pages, kv_block_table, ctx_lens, page_size, pool_pages,
               pool_block_table, sinks, o, ws=None, stream=None) -> None:
    _check("hca_decode", load_library().hca_decode(
        ctypes.byref(p), nseq, _ptr(q), _ptr(kv_pages), _ptr(kv_block_table),
        kv_block_table.shape[1], _ptr(ctx_lens), page_size, _ptr(pool_pages),
        _ptr(pool_block_table), pool_block_table.shape[1], _ptr(sinks), _ptr(o), _ptr(ws),
        _nbytes(ws), _stream(stream)))


def csa_decode(p, nseq, q, kv_pages, kv_block_table, ctx_lens, page_size, pool_pages,
               idx_pool_pages, pool_block_table, q_idx, w_idx, sinks, o, topk_out, ws,
               stream=None) -> None:
    _check("csa_decode", load_library().csa_decode(
        ctypes.byref(p), nseq, _ptr(q), _ptr(kv_pages), _ptr(kv_block_table),
        kv_block_table.shape[1], _ptr(ctx_lens), page_size, _ptr(pool_pages),
        _ptr(idx_pool_pages), _ptr(pool_block_table), pool_block_table.shape[1], _ptr(q_idx),
        _ptr(w_idx), _ptr(sinks), _ptr(o), _ptr(topk_out), _ptr(ws), _nbytes(ws),
        _stream(stream)))


def sac_chunk_workspace_size(p: sac_params, kind: int, nseq: int, n: int) -> int:
    return int(load_library().sac_chunk_workspace_size(ctypes.byref(p), kind, nseq, n))


def swa_prefill_chunk(p, nseq, n, q, kv_pages, kv_block_table, ctx_lens, page_size, sinks, o,
                      ws=None, stream=None) -> None:
    """Attention of each sequence's last n tokens over the paged caches (see include/sac.h)."""
    _check("swa_prefill_chunk", load_library().swa_prefill_chunk(
        ctypes.byref(p), nseq, n, _ptr(q), _ptr(kv_pages), _ptr(kv_block_table),
        kv_block_table.shape[1], _ptr(ctx_lens), page_size, _ptr(sinks), _ptr(o), _ptr(ws),
        _nbytes(ws), _stream(stream)))


def hca_prefill_chunk(p, nseq, n, q, kv_pages, kv_block_table, ctx_lens, page_size, pool_pages,
                      pool_block_table, sinks, o, ws=None, stream=None) -> None:
    _check("hca_prefill_chunk", load_library().hca_prefill_chunk(
        ctypes.byref(p), nseq, n, _ptr(q), _ptr(kv_pages), _ptr(kv_block_table),
        kv_block_table.shape[1], _ptr(ctx_lens), page_size, _ptr(pool_pages),
        _ptr(pool_block_table), pool_block_table.shape[1], _ptr(sinks), _ptr(o), _ptr(ws),
        _nbytes(ws), _stream(stream)))


def csa_prefill_chunk(p, nseq, n, q, kv_pages, kv_block_table, ctx_lens, page_size, pool_pages,
                      idx_pool_pages, pool_block_table, q_idx, w_idx, sinks, o, topk_out, ws,
                      stream=None) -> None:
    _check("csa_prefill_chunk", load_library().csa_prefill_chunk(
        ctypes.byref(p), nseq, n, _ptr(q), _ptr(kv_pages), _ptr(kv_block_table),
        kv_block_table.shape[1], _ptr(ctx_lens), page_size, _ptr(pool_pages),
        _ptr(idx_pool_pages), _ptr(pool_block_table), pool_block_table.shape[1], _ptr(q_idx),
        _ptr(w_idx), _ptr(sinks), _ptr(o), _ptr(topk_out), _ptr(ws), _nbytes(ws),
        _stream(stream)))


def prefill_chunk_append(p, kind, nseq, n, ctx_lens, kv_new, kv_pages, kv_block_table,
                         page_size, cmp_state=None, cmp_gate=None, cmp_bias=None,
                         pool_pages=None, pool_block_table=None, k_idx_new=None, idx_state=None,
                         idx_gate=None, idx_bias=None, idx_pool_pages=None, stream=None) -> None:
    """Append each sequence's last n tokens (kv_new [nseq, n, D]) to the caches: decode_append
    for a whole chunk."""
    pmax = pool_block_table.shape[1] if pool_block_table is not None else 0
    _check("prefill_chunk_append", load_library().prefill_chunk_append(
        ctypes.byref(p), kind, nseq, n, _ptr(ctx_lens), _ptr(kv_new), _ptr(k_idx_new),
        _ptr(cmp_gate), _ptr(cmp_bias), _ptr(idx_gate), _ptr(idx_bias), _ptr(kv_pages),
        _ptr(kv_block_table), kv_block_table.shape[1], page_size, _ptr(cmp_state),
        _ptr(idx_state), _ptr(pool_pages), _ptr(idx_pool_pages), _ptr(pool_block_table), pmax,
        _stream(stream)))


def decode_append(p, kind, nseq, ctx_lens, kv_new, kv_pages, kv_block_table, page_size,
                  cmp_state=None, cmp_gate=None, cmp_bias=None, pool_pages=None,
                  pool_block_table=None, k_idx_new=None, idx_state=None, idx_gate=None,
                  idx_bias=None, idx_pool_pages=None, stream=None) -> None:
    """Append each sequence's new token (at ctx - 1) to the decode caches: the rotated kv row to
    the window pages and, for HCA / CSA, the compressor ring(s), closing a pool entry whenever
    ctx is a multiple of m."""
    pmax = pool_block_table.shape[1] if pool_block_table is not None else 0
    _check("decode_append", load_library().decode_append(
        ctypes.byref(p), kind, nseq, _ptr(ctx_lens), _ptr(kv_new), _ptr(k_idx_new),
        _ptr(cmp_gate), _ptr(cmp_bias), _ptr(idx_gate), _ptr(idx_bias), _ptr(kv_pages),
        _ptr(kv_block_table), kv_block_table.shape[1], page_size, _ptr(cmp_state),
        _ptr(idx_state), _ptr(pool_pages), _ptr(idx_pool_pages), _ptr(pool_block_table), pmax,
        _stream(stream)))


def sac_oproj_workspace_size(p: sac_params, T: int, groups: int, rank: int) -> int:
    return int(load_library().sac_oproj_workspace_size(ctypes.byref(p), T, groups, rank))


def o_proj_forward(p, T, groups, rank, hidden, o, w_a, w_b, out, ws, stream=None) -> None:
    """Grouped low-rank output projection: out = concat_g(o_g w_a[g]^T) w_b^T (see include/sac.h)."""
    _check("o_proj_forward", load_library().o_proj_forward(
        ctypes.byref(p), T, groups, rank, hidden, _ptr(o), _ptr(w_a), _ptr(w_b), _ptr(out),
        _ptr(ws), _nbytes(ws), _stream(stream)))
