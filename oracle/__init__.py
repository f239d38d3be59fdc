"""fp64 CPU oracle of the DeepSeek-V4 hybrid long-range attention forward.

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It shares no code with the CUDA library: the arithmetic
lives in ``sac_oracle.c`` (plain C, IEEE fp64), this module only marshals numpy float64 arrays.

Source: the "DeepSeek-V4" model documentation page (Hugging Face Transformers), sections "Hybrid
attention (section 2.3)", "Attention mask layout" and "Cache layers". Parity status:
  - compressor gate formula: parity unpinned (a reading of the page; special cases pinned)
  - indexer score formula:   parity unpinned (a reading of the page; special cases pinned)
  - everything else is pinned by the tests under ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sac_oracle.c")
_SO = os.path.join(_HERE, "libsac_oracle.so")

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)
_lp = ctypes.POINTER(ctypes.c_int64)


class _Params(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("S", ctypes.c_int), ("H", ctypes.c_int), ("D", ctypes.c_int),
        ("R", ctypes.c_int), ("theta", ctypes.c_double), ("m", ctypes.c_int),
        ("L", ctypes.c_int), ("W", ctypes.c_int), ("nI", ctypes.c_int), ("cI", ctypes.c_int),
        ("k", ctypes.c_int), ("scale", ctypes.c_double), ("pos0", ctypes.c_int64),
        ("bf16_pools", ctypes.c_int), ("yarn_factor", ctypes.c_double),
        ("yarn_orig", ctypes.c_int), ("yarn_beta_fast", ctypes.c_double),
        ("yarn_beta_slow", ctypes.c_double),
    ]


@dataclass
class OracleParams:
    """Attention hyper-parameters of one layer (names follow the page's config)."""
    B: int
    S: int
    H: int
    D: int
    R: int
    theta: float
    W: int
    m: int = 0
    L: int = 0
    nI: int = 0
    cI: int = 0
    k: int = 0
    scale: float = 0.0
    pos0: int = 0
    bf16_pools: bool = False  # pools cached in bf16 (the layer's working dtype)
    yarn_factor: float = 1.0  # YaRN context scale s (<= 1: plain RoPE)
    yarn_orig: int = 0        # YaRN original context length
    yarn_beta_fast: float = 32.0
    yarn_beta_slow: float = 1.0

    def c(self) -> _Params:
        scale = self.scale if self.scale > 0 else 1.0 / np.sqrt(self.D)
        return _Params(self.B, self.S, self.H, self.D, self.R, float(self.theta), self.m,
                       self.L, self.W, self.nI, self.cI, self.k, float(scale), int(self.pos0),
                       int(self.bf16_pools), float(self.yarn_factor), int(self.yarn_orig),
                       float(self.yarn_beta_fast), float(self.yarn_beta_slow))


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, no fast-math, OpenMP over query rows)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


_lib_handle = None


def _lib():
    global _lib_handle
    if _lib_handle is None:
        lib = ctypes.CDLL(build())
        lib.orc_rope.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double]
        lib.orc_rope_yarn.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                      ctypes.c_double, ctypes.c_int, ctypes.c_double,
                                      ctypes.c_double, ctypes.c_double]
        lib.orc_rope_freq.restype = ctypes.c_double
        lib.orc_rope_freq.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                      ctypes.c_double, ctypes.c_int, ctypes.c_double,
                                      ctypes.c_double]
        lib.orc_compress.restype = ctypes.c_long
        lib.orc_compress.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, _dp, _dp, _dp, _dp]
        lib.orc_index_scores.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp, _dp,
                                         ctypes.c_long, _dp]
        lib.orc_topk.argtypes = [_dp, ctypes.c_long, ctypes.c_int, _ip]
        lib.orc_attend.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, _dp, ctypes.c_long,
                                   _dp, _dp, _dp]
        P = ctypes.POINTER(_Params)
        lib.orc_swa_forward.argtypes = [P, _dp, _dp, _dp, _dp, _lp, ctypes.c_long]
        lib.orc_hca_forward.argtypes = [P, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _lp, ctypes.c_long]
        lib.orc_csa_forward.argtypes = [P, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                        _ip, _dp, _dp, _ip, _lp, ctypes.c_long]
        lib.orc_csa_index_scores.argtypes = [P, _dp, _dp, _dp, _dp, _dp, _lp, ctypes.c_long, _dp]
        lib.orc_decode.argtypes = [P, ctypes.c_int, _dp, _dp, _ip, ctypes.c_int, _ip, ctypes.c_int,
                                   _dp, _dp, _ip, ctypes.c_int, _dp, _dp, _dp, _dp, _ip, _ip]
        lib.orc_oproj.restype = None
        lib.orc_oproj.argtypes = [ctypes.c_int] * 5 + [_dp, _dp, _dp, ctypes.c_int, _lp,
                                                       ctypes.c_int, _dp, _dp]
        lib.orc_round_bf16.restype = ctypes.c_double
        lib.orc_round_bf16.argtypes = [ctypes.c_double]
        lib.orc_max_threads.restype = ctypes.c_int
        lib.orc_set_threads.argtypes = [ctypes.c_int]
        _lib_handle = lib
    return _lib_handle


def _f64(x) -> np.ndarray:
    """Exact upcast to a contiguous float64 array (bf16 / fp32 values are representable)."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # a torch tensor: go through float32 (bf16 -> f32 is exact)
        x = x.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr(a, kind=_dp):
    return None if a is None else a.ctypes.data_as(kind)


def round_bf16(x: float) -> float:
    """A pool value as cached in bf16 (nearest, ties to even, from its fp32 value)."""
    return float(_lib().orc_round_bf16(float(x)))


def max_threads() -> int:
    return int(_lib().orc_max_threads())


def set_threads(n: int) -> None:
    _lib().orc_set_threads(int(n))


# --------------------------------------------------------------------------------------------
# Single steps
# --------------------------------------------------------------------------------------------
def rope(x, R: int, theta: float, pos: float) -> np.ndarray:
    """Rotate the trailing R channels of each row of x (interleaved pairs) at position pos."""
    a = _f64(x).copy()
    rows = a.reshape(-1, a.shape[-1])
    for r in rows:
        _lib().orc_rope(_ptr(r), a.shape[-1], R, float(theta), float(pos))
    return rows.reshape(a.shape)


def rope_yarn(x, R: int, theta: float, pos: float, factor: float, orig: int,
              beta_fast: float = 32.0, beta_slow: float = 1.0) -> np.ndarray:
    """rope() with YaRN frequencies (context scale `factor` over an original length `orig`)."""
    a = _f64(x).copy()
    rows = a.reshape(-1, a.shape[-1])
    for r in rows:
        _lib().orc_rope_yarn(_ptr(r), a.shape[-1], R, float(theta), float(factor), int(orig),
                             float(beta_fast), float(beta_slow), float(pos))
    return rows.reshape(a.shape)


def rope_freq(i: int, R: int, theta: float, factor: float = 1.0, orig: int = 1,
              beta_fast: float = 32.0, beta_slow: float = 1.0) -> float:
    """Frequency of rope pair i (YaRN-scaled when factor > 1)."""
    return float(_lib().orc_rope_freq(i, R, float(theta), float(factor), int(orig),
                                      float(beta_fast), float(beta_slow)))


def compress(x, u, bias, m: int, L: int) -> np.ndarray:
    """Un-rotated pool [B, floor(S/m), C] of x [B,S,C] with gate vector u [C] and bias [L]."""
    x = _f64(x)
    B, S, C = x.shape
    N = S // m
    out = np.zeros((B, max(N, 0), C))
    n = _lib().orc_compress(B, S, C, m, L, _ptr(x), _ptr(_f64(u)), _ptr(_f64(bias)),
                            _ptr(out) if N > 0 else _ptr(np.zeros(1)))
    assert n == N
    return out


def index_scores(qI_t, wI_t, KI, nvis: int) -> np.ndarray:
    """Scores [N] of one query (qI_t [nI,cI], wI_t [nI]) against KI [N,cI]; -inf past nvis."""
    qI_t, wI_t, KI = _f64(qI_t), _f64(wI_t), _f64(KI)
    nI, cI = qI_t.shape
    N = KI.shape[0]
    out = np.zeros(N)
    _lib().orc_index_scores(N, nI, cI, _ptr(qI_t), _ptr(wI_t), _ptr(KI), nvis, _ptr(out))
    return out


def topk(scores, nvis: int, k: int) -> np.ndarray:
    """Top-k of the first nvis scores: score descending, ties to the lower index, -1 fill."""
    s = _f64(scores)
    idx = np.zeros(k, dtype=np.int32)
    _lib().orc_topk(_ptr(s), nvis, k, _ptr(idx, _ip))
    return idx


def attend(qrot, keys, sinks, scale: float) -> np.ndarray:
    """One query's attention over an explicit (already rotated) key list, sink in the
    normaliser. qrot [H,D], keys [nk,D], sinks [H] -> [H,D]."""
    qrot, keys, sinks = _f64(qrot), _f64(keys), _f64(sinks)
    H, D = qrot.shape
    nk = keys.shape[0]
    o = np.zeros((H, D))
    _lib().orc_attend(H, D, float(scale), _ptr(qrot), nk,
                      _ptr(keys if nk else np.zeros((1, D))), _ptr(sinks), _ptr(o))
    return o


# --------------------------------------------------------------------------------------------
# Full forwards. Per-row arrays are given for all B*S rows, or with `rows` (flat b*S+t) only for
# the listed rows, in list order. Outputs follow the same convention.
# --------------------------------------------------------------------------------------------
def _rows(p: OracleParams, rows):
    if rows is None:
        return None, p.B * p.S
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, len(r)


def swa_forward(p: OracleParams, q, kv, sinks, rows=None) -> np.ndarray:
    r, n = _rows(p, rows)
    q = _f64(q).reshape(n, p.H, p.D)
    kv = _f64(kv).reshape(p.B, p.S, p.D)
    o = np.zeros((n, p.H, p.D))
    _lib().orc_swa_forward(ctypes.byref(p.c()), _ptr(q), _ptr(kv), _ptr(_f64(sinks)), _ptr(o),
                           _ptr(r, _lp), n)
    return o


def hca_forward(p: OracleParams, q, kv, cmp_gate, cmp_bias, sinks, rows=None):
    """Returns (o, rotated pool [B,N,D])."""
    r, n = _rows(p, rows)
    q = _f64(q).reshape(n, p.H, p.D)
    kv = _f64(kv).reshape(p.B, p.S, p.D)
    N = p.S // p.m
    o = np.zeros((n, p.H, p.D))
    pool = np.zeros((p.B, N, p.D))
    _lib().orc_hca_forward(ctypes.byref(p.c()), _ptr(q), _ptr(kv), _ptr(_f64(cmp_gate)),
                           _ptr(_f64(cmp_bias)), _ptr(_f64(sinks)), _ptr(o), _ptr(pool),
                           _ptr(r, _lp), n)
    return o, pool


def csa_forward(p: OracleParams, q, kv, cmp_gate, cmp_bias, q_idx, w_idx, k_idx, idx_gate,
                idx_bias, sinks, rows=None, topk_in=None):
    """Returns (o, topk [n,k], rotated pool [B,N,D], indexer pool [B,N,cI]). With topk_in the
    given selections replace the oracle's own (the returned topk then echoes them)."""
    r, n = _rows(p, rows)
    q = _f64(q).reshape(n, p.H, p.D)
    kv = _f64(kv).reshape(p.B, p.S, p.D)
    qI = _f64(q_idx).reshape(n, p.nI, p.cI)
    wI = _f64(w_idx).reshape(n, p.nI)
    kI = _f64(k_idx).reshape(p.B, p.S, p.cI)
    N = p.S // p.m
    o = np.zeros((n, p.H, p.D))
    tk = np.zeros((n, p.k), dtype=np.int32)
    pool = np.zeros((p.B, N, p.D))
    kpool = np.zeros((p.B, N, p.cI))
    tin = None if topk_in is None else _i32(topk_in).reshape(n, p.k)
    _lib().orc_csa_forward(ctypes.byref(p.c()), _ptr(q), _ptr(kv), _ptr(_f64(cmp_gate)),
                           _ptr(_f64(cmp_bias)), _ptr(qI), _ptr(wI), _ptr(kI),
                           _ptr(_f64(idx_gate)), _ptr(_f64(idx_bias)), _ptr(_f64(sinks)),
                           _ptr(o), _ptr(tk, _ip), _ptr(pool), _ptr(kpool), _ptr(tin, _ip),
                           _ptr(r, _lp), n)
    return o, tk, pool, kpool


def csa_index_scores(p: OracleParams, q_idx, w_idx, k_idx, idx_gate, idx_bias, rows):
    """Indexer scores [len(rows), N] of the listed rows (q_idx/w_idx given for those rows), over
    the oracle's own indexer pool (rounded to bf16 with p.bf16_pools), -inf past (t+1)//m.
    Pinned by tests/test_oracle_index_pins.py: its top-k equals csa_forward's selection, and its
    scores equal index_scores over the pool csa_forward returns."""
    r, n = _rows(p, rows)
    qI = _f64(q_idx).reshape(n, p.nI, p.cI)
    wI = _f64(w_idx).reshape(n, p.nI)
    kI = _f64(k_idx).reshape(p.B, p.S, p.cI)
    N = p.S // p.m
    out = np.zeros((n, N))
    _lib().orc_csa_index_scores(ctypes.byref(p.c()), _ptr(qI), _ptr(wI), _ptr(kI),
                                _ptr(_f64(idx_gate)), _ptr(_f64(idx_bias)), _ptr(r, _lp), n,
                                _ptr(out))
    return out


def decode(p: OracleParams, q, kv_pages, kv_block_table, ctx_lens, page_size: int,
           pool_pages=None, idx_pool_pages=None, pool_block_table=None, q_idx=None, w_idx=None,
           sinks=None, topk_in=None):
    """One decode step over a paged cache (p.m == 0: sliding only; p.k > 0: CSA; else HCA).
    Returns (o [nseq,H,D], topk [nseq,k] or None)."""
    q = _f64(q)
    nseq = q.shape[0]
    kvp = _f64(kv_pages)
    kbt = _i32(kv_block_table)
    ctx = _i32(ctx_lens)
    pp = _f64(pool_pages)
    ipp = _f64(idx_pool_pages)
    pbt = _i32(pool_block_table)
    qI = _f64(q_idx)
    wI = _f64(w_idx)
    o = np.zeros((nseq, p.H, p.D))
    tk = np.zeros((nseq, max(p.k, 1)), dtype=np.int32) if p.k > 0 else None
    tin = None if topk_in is None else _i32(topk_in)
    _lib().orc_decode(ctypes.byref(p.c()), nseq, _ptr(q), _ptr(kvp), _ptr(kbt, _ip),
                      kbt.shape[1], _ptr(ctx, _ip), page_size, _ptr(pp), _ptr(ipp),
                      _ptr(pbt, _ip), 0 if pbt is None else pbt.shape[1], _ptr(qI), _ptr(wI),
                      _ptr(_f64(sinks)), _ptr(o), _ptr(tk, _ip), _ptr(tin, _ip))
    return o, tk


def o_proj(o, w_a, w_b, groups: int, rows=None, round_mid: bool = False):
    """Grouped low-rank output projection of the listed token rows (all rows when None).
    o [T, H, D] or [T, H*D]; w_a [G, rank, (H/G)*D]; w_b [hidden, G*rank]. Returns (mid, out)
    for those rows, mid [n, G*rank] (rounded to bf16 when round_mid) and out [n, hidden]."""
    o = _f64(o)
    T = o.shape[0]
    o2 = np.ascontiguousarray(o.reshape(T, -1))
    w_a, w_b = _f64(w_a), _f64(w_b)
    G, rank, kg = w_a.shape
    hidden = w_b.shape[0]
    assert G == groups and w_b.shape[1] == G * rank and o2.shape[1] == G * kg
    HD = o2.shape[1]
    # the C routine takes H and D; only H*D and (H/G)*D matter, so pass H = G, D = kg
    rows = np.arange(T, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    mid = np.zeros((len(rows), G * rank))
    out = np.zeros((len(rows), hidden))
    _lib().orc_oproj(G, kg, G, rank, hidden, _ptr(o2), _ptr(w_a), _ptr(w_b), len(rows),
                     _ptr(rows, _lp), int(round_mid), _ptr(mid), _ptr(out))
    assert HD == G * kg
    return mid, out
