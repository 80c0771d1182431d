"""Float64 CPU reference ("the oracle") for one DSA sparse-attention prefill layer.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product path (the
CUDA library and its Python binding) never imports, links or calls it, and this
package imports nothing from the product.

The arithmetic lives in ``dsa_oracle.cpp`` (plain C++, float64, no fused
multiply-add); this module only compiles it with g++ and marshals numpy arrays.
Each function's definition and the page passages it follows are stated in the
C++ source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


class OracleDims(ctypes.Structure):
    _fields_ = [
        ("n_q", ctypes.c_int32),
        ("q_pos0", ctypes.c_int32),
        ("ctx_len", ctypes.c_int32),
        ("n_heads", ctypes.c_int32),
        ("d_latent", ctypes.c_int32),
        ("d_rope", ctypes.c_int32),
        ("n_idx_heads", ctypes.c_int32),
        ("d_idx", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("softmax_scale", ctypes.c_double),
    ]


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (-O2, no FMA contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-pthread", _SRC, "-o", _LIB + ".tmp"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, cint = ctypes.c_int32, ctypes.c_int64, ctypes.c_int
        dp = ctypes.POINTER(OracleDims)
        lib.oracle_index_scores.argtypes = [dp, P, P, P, P, i32, P, cint]
        lib.oracle_topk_select.argtypes = [dp, P, i64, P, i32, P, cint]
        lib.oracle_topk_select_f32.argtypes = [dp, P, i64, P, i32, P, cint]
        lib.oracle_sparse_attn.argtypes = [dp, P, P, P, P, P, i32, P, P, cint]
        lib.oracle_prefill_layer.argtypes = [dp, P, P, P, P, P, P, P, i32, P, P, P, cint]
        lib.oracle_quantize_fp8.argtypes = [P, i64, i32, P, P, P]
        for f in (lib.oracle_index_scores, lib.oracle_topk_select, lib.oracle_topk_select_f32,
                  lib.oracle_sparse_attn, lib.oracle_prefill_layer, lib.oracle_quantize_fp8):
            f.restype = cint
        _lib = lib
    return _lib


def _threads(n_threads):
    return int(n_threads) if n_threads else (os.cpu_count() or 1)


def dims_of(d) -> OracleDims:
    """Accepts any object with the dims attributes (e.g. workloads.Dims)."""
    return OracleDims(int(d.n_q), int(d.q_pos0), int(d.ctx_len), int(d.n_heads),
                      int(d.d_latent), int(d.d_rope), int(d.n_idx_heads), int(d.d_idx),
                      int(d.top_k), float(d.softmax_scale))


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 tensors travel as uint16 bit patterns"
    return a


def _rows(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(rows, dtype=np.int32)
    return r, int(r.size)


def index_scores(d, q_idx, k_idx, w_idx, rows=None, n_threads=None):
    """float64 scores [n_rows, ctx_len]; -inf where s > t."""
    od = dims_of(d)
    r, nr = _rows(rows)
    n = nr if r is not None else od.n_q
    out = np.empty((n, od.ctx_len), dtype=np.float64)
    q_idx, k_idx = _u16(q_idx), _u16(k_idx)
    w_idx = np.ascontiguousarray(w_idx, dtype=np.float32)
    rc = _load().oracle_index_scores(ctypes.byref(od), _ptr(q_idx), _ptr(k_idx), _ptr(w_idx),
                                     _ptr(r), nr, _ptr(out), _threads(n_threads))
    assert rc == 0
    return out


def topk_select(d, scores, rows=None, n_threads=None):
    """Selection on float64 (or float32, widened) scores [n_rows, ld]."""
    od = dims_of(d)
    r, nr = _rows(rows)
    n = nr if r is not None else od.n_q
    idx = np.empty((n, od.top_k), dtype=np.int32)
    scores = np.ascontiguousarray(scores)
    assert scores.shape[0] == n
    if scores.dtype == np.float32:
        fn = _load().oracle_topk_select_f32
    else:
        scores = scores.astype(np.float64, copy=False)
        fn = _load().oracle_topk_select
    rc = fn(ctypes.byref(od), _ptr(scores), scores.shape[1], _ptr(r), nr, _ptr(idx),
            _threads(n_threads))
    assert rc == 0
    return idx


def sparse_attn(d, q, latent, rope, idx, rows=None, n_threads=None):
    """(out float64 [n_rows, H, Dc], lse float64 [n_rows, H])."""
    od = dims_of(d)
    r, nr = _rows(rows)
    n = nr if r is not None else od.n_q
    out = np.empty((n, od.n_heads, od.d_latent), dtype=np.float64)
    lse = np.empty((n, od.n_heads), dtype=np.float64)
    q, latent, rope = _u16(q), _u16(latent), _u16(rope)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    assert idx.shape == (n, od.top_k)
    rc = _load().oracle_sparse_attn(ctypes.byref(od), _ptr(q), _ptr(latent), _ptr(rope),
                                    _ptr(idx), _ptr(r), nr, _ptr(out), _ptr(lse),
                                    _threads(n_threads))
    assert rc == 0
    return out, lse


def prefill_layer(d, q, latent, rope, q_idx, k_idx, w_idx, rows=None, n_threads=None):
    """(out float64 [n_rows,H,Dc], lse float64 [n_rows,H], idx int32 [n_rows,k])."""
    od = dims_of(d)
    r, nr = _rows(rows)
    n = nr if r is not None else od.n_q
    out = np.empty((n, od.n_heads, od.d_latent), dtype=np.float64)
    lse = np.empty((n, od.n_heads), dtype=np.float64)
    idx = np.empty((n, od.top_k), dtype=np.int32)
    q, latent, rope, q_idx, k_idx = map(_u16, (q, latent, rope, q_idx, k_idx))
    w_idx = np.ascontiguousarray(w_idx, dtype=np.float32)
    rc = _load().oracle_prefill_layer(ctypes.byref(od), _ptr(q), _ptr(latent), _ptr(rope),
                                      _ptr(q_idx), _ptr(k_idx), _ptr(w_idx), _ptr(r), nr,
                                      _ptr(out), _ptr(lse), _ptr(idx), _threads(n_threads))
    assert rc == 0
    return out, lse, idx


def quantize_fp8(x):
    """FP8 (e4m3) form of bf16 rows x [..., cols] (see dsa_oracle.cpp):
    (x8 uint8 e4m3 bits, scale float32 [...], xhat uint16 bf16 bits)."""
    x = _u16(x)
    shape = x.shape
    cols = shape[-1]
    rows = int(np.prod(shape[:-1])) if len(shape) > 1 else 1
    x8 = np.empty(shape, dtype=np.uint8)
    scale = np.empty(shape[:-1], dtype=np.float32)
    xhat = np.empty(shape, dtype=np.uint16)
    rc = _load().oracle_quantize_fp8(_ptr(x), rows, cols, _ptr(x8), _ptr(scale), _ptr(xhat))
    assert rc == 0
    return x8, scale, xhat


def index_scores_fp8(d, q_idx, k_idx, w_idx, rows=None, n_threads=None):
    """Scores of the FP8 indexer contract: the float64 scores of the
    dequantized (xhat) indexer inputs."""
    _, _, q_hat = quantize_fp8(q_idx)
    _, _, k_hat = quantize_fp8(k_idx)
    return index_scores(d, q_hat, k_hat, w_idx, rows=rows, n_threads=n_threads)
