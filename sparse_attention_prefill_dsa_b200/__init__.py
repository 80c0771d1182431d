"""Python binding of libdsa.so, the B200 (sm_100a) DSA sparse-attention prefill library.

Argument marshalling only: each function below passes its arguments to the C
entry point of the same name (declared in include/dsa.h) and returns its
status code. Every step of the layer runs in the library's CUDA kernels;
there is no other implementation to fall back to: the first call raises
RuntimeError when libdsa.so has not been built.

Tensors may be given as torch tensors (their data_ptr() is passed) or as raw
integer device addresses. ``stream`` defaults to torch's current CUDA stream.

DSA_LIBRARY=check in the environment loads libdsa_check.so instead: the same
kernels built with bounds checks that report a bad index in the workspace
status (DSA_ERR_CUDA from dsa_device_status, site 1000 + n in the header)
rather than making the access.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa_check.so" if os.environ.get("DSA_LIBRARY") == "check"
                        else "libdsa.so")

_lib = None

DSA_OK = 0
DSA_ERR_NULL = -1
DSA_ERR_ALIGN = -2
DSA_ERR_DIMS = -3
DSA_ERR_CAUSAL = -4
DSA_ERR_WORKSPACE = -5
DSA_ERR_TIMEOUT = -6
DSA_ERR_CUDA = -7
DSA_ERR_DEVICE = -8
DSA_ERR_RANGE = -9
DSA_ERR_SCRATCH_LIMIT = -10
DSA_ERR_LAYOUT = -11
DSA_NOALLOC_SCRATCH_BYTES = 32 << 20

DSA_WS_INDEX_SCORES = 0
DSA_WS_TOPK = 1
DSA_WS_ATTN = 2
DSA_WS_LAYER = 3
DSA_WS_DECODE_ATTN = 4
DSA_WS_DECODE_LAYER = 5
DSA_WS_BLOCK_ATTN = 6
DSA_FLAG_FP8_INDEXER = 1
DSA_FLAG_ATTN_PAIR = 2
DSA_FLAG_HOST_UNORDERED = 4
DSA_FLAG_L2_SCORES = 8
DSA_MAX_BLOCK_QUERIES = 2

DSA_MAX_TOPK = 2048
DSA_MAX_CTX = 131072

EXPORTED = ("dsa_workspace_size", "dsa_index_scores", "dsa_topk_select",
            "dsa_sparse_attn_prefill", "dsa_prefill_layer", "dsa_device_status",
            "dsa_status_string", "dsa_prefill_layer_noalloc", "dsa_prefill_layer_host",
            "dsa_selftest_bounded_wait", "dsa_partition_queries", "dsa_sparse_attn_decode",
            "dsa_decode_layer", "dsa_sparse_attn_block", "dsa_quantize_fp8",
            "dsa_index_scores_fp8", "dsa_selftest_mma_layout")


class dsa_dims(ctypes.Structure):
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
        ("softmax_scale", ctypes.c_float),
        ("flags", ctypes.c_uint32),
    ]


class dsa_device_tensors(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in
                ("q", "latent", "rope", "q_idx", "k_idx", "w_idx", "out", "lse", "idx")]


class DsaError(RuntimeError):
    def __init__(self, status: int):
        super().__init__(f"dsa status {status}: {dsa_status_string(status)}")
        self.status = status


_P = ctypes.c_void_p
_DP = ctypes.POINTER(dsa_dims)


def library():
    """The loaded ctypes library; raises RuntimeError if it was never built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: the DSA CUDA library has not been built "
            "(python -m sparse_attention_prefill_dsa_b200.build). There is no fallback.")
    lib = ctypes.CDLL(LIB_PATH)
    lib.dsa_workspace_size.argtypes = [_DP, ctypes.c_int32]
    lib.dsa_workspace_size.restype = ctypes.c_size_t
    lib.dsa_index_scores.argtypes = [_DP, _P, _P, _P, _P, ctypes.c_int64, _P, ctypes.c_size_t, _P]
    lib.dsa_topk_select.argtypes = [_DP, _P, ctypes.c_int64, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                    _P]
    lib.dsa_sparse_attn_prefill.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
    lib.dsa_prefill_layer.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                      ctypes.c_size_t, _P]
    lib.dsa_sparse_attn_decode.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
    lib.dsa_decode_layer.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                     ctypes.c_size_t, _P]
    lib.dsa_sparse_attn_block.argtypes = [_DP, _P, _P, _P, _P, _P, _P, ctypes.c_int32, _P,
                                          ctypes.c_size_t, _P]
    lib.dsa_quantize_fp8.argtypes = [_P, ctypes.c_int64, ctypes.c_int32, _P, _P, _P, _P]
    lib.dsa_index_scores_fp8.argtypes = [_DP, _P, _P, _P, _P, _P, _P, ctypes.c_int64, _P,
                                         ctypes.c_size_t, _P]
    lib.dsa_prefill_layer_noalloc.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]
    lib.dsa_prefill_layer_host.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                           ctypes.POINTER(dsa_device_tensors), _P, ctypes.c_size_t,
                                           ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.c_int32]
    lib.dsa_selftest_bounded_wait.argtypes = [_P, ctypes.c_size_t, _P, _P]
    lib.dsa_selftest_mma_layout.argtypes = [_P, ctypes.c_size_t, ctypes.POINTER(ctypes.c_int32),
                                            ctypes.POINTER(ctypes.c_float), _P]
    lib.dsa_partition_queries.argtypes = [_DP, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]
    lib.dsa_device_status.argtypes = [_P, _P]
    lib.dsa_status_string.argtypes = [ctypes.c_int32]
    lib.dsa_status_string.restype = ctypes.c_char_p
    for f in ("dsa_index_scores", "dsa_topk_select", "dsa_sparse_attn_prefill",
              "dsa_prefill_layer", "dsa_device_status", "dsa_prefill_layer_noalloc",
              "dsa_prefill_layer_host", "dsa_selftest_bounded_wait", "dsa_partition_queries",
              "dsa_sparse_attn_decode", "dsa_decode_layer", "dsa_sparse_attn_block",
              "dsa_quantize_fp8", "dsa_index_scores_fp8", "dsa_selftest_mma_layout"):
        getattr(lib, f).restype = ctypes.c_int32
    _lib = lib
    return lib


def make_dims(d) -> dsa_dims:
    """dsa_dims from any object with the same attribute names (flags default 0)."""
    return dsa_dims(int(d.n_q), int(d.q_pos0), int(d.ctx_len), int(d.n_heads),
                    int(d.d_latent), int(d.d_rope), int(d.n_idx_heads), int(d.d_idx),
                    int(d.top_k), float(d.softmax_scale), int(getattr(d, "flags", 0)))


def _dims(d):
    return ctypes.byref(d if isinstance(d, dsa_dims) else make_dims(d))


def _p(x):
    if x is None:
        return None
    if isinstance(x, int):
        return _P(x)
    return _P(x.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return _P(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return _P(stream)
    return _P(stream.cuda_stream)


def _nbytes(ws, ws_bytes):
    if ws_bytes is not None:
        return int(ws_bytes)
    if ws is None or isinstance(ws, int):
        return 0
    return ws.numel() * ws.element_size()


def dsa_workspace_size(dims, which: int) -> int:
    return int(library().dsa_workspace_size(_dims(dims), int(which)))


def dsa_index_scores(dims, q_idx, k_idx, w_idx, scores, ld_scores, workspace, workspace_bytes=None,
                     stream=None) -> int:
    return library().dsa_index_scores(_dims(dims), _p(q_idx), _p(k_idx), _p(w_idx), _p(scores),
                                 int(ld_scores), _p(workspace),
                                 _nbytes(workspace, workspace_bytes), _stream(stream))


def dsa_topk_select(dims, scores, ld_scores, q_idx, k_idx, w_idx, idx, workspace,
                    workspace_bytes=None, stream=None) -> int:
    return library().dsa_topk_select(_dims(dims), _p(scores), int(ld_scores), _p(q_idx), _p(k_idx),
                                _p(w_idx), _p(idx), _p(workspace),
                                _nbytes(workspace, workspace_bytes), _stream(stream))


def dsa_sparse_attn_prefill(dims, q, latent, rope, idx, out, lse, workspace, workspace_bytes=None,
                            stream=None) -> int:
    return library().dsa_sparse_attn_prefill(_dims(dims), _p(q), _p(latent), _p(rope), _p(idx),
                                        _p(out), _p(lse), _p(workspace),
                                        _nbytes(workspace, workspace_bytes), _stream(stream))


def dsa_prefill_layer(dims, q, latent, rope, q_idx, k_idx, w_idx, out, lse, idx_out, workspace,
                      workspace_bytes=None, stream=None) -> int:
    return library().dsa_prefill_layer(_dims(dims), _p(q), _p(latent), _p(rope), _p(q_idx),
                                  _p(k_idx), _p(w_idx), _p(out), _p(lse), _p(idx_out),
                                  _p(workspace), _nbytes(workspace, workspace_bytes),
                                  _stream(stream))


def dsa_sparse_attn_decode(dims, q, latent, rope, idx, out, lse, workspace, workspace_bytes=None,
                           stream=None) -> int:
    return library().dsa_sparse_attn_decode(_dims(dims), _p(q), _p(latent), _p(rope), _p(idx),
                                            _p(out), _p(lse), _p(workspace),
                                            _nbytes(workspace, workspace_bytes), _stream(stream))


def dsa_sparse_attn_block(dims, q, latent, rope, idx, out, lse, block_queries, workspace,
                          workspace_bytes=None, stream=None) -> int:
    return library().dsa_sparse_attn_block(_dims(dims), _p(q), _p(latent), _p(rope), _p(idx),
                                           _p(out), _p(lse), int(block_queries), _p(workspace),
                                           _nbytes(workspace, workspace_bytes), _stream(stream))


def dsa_quantize_fp8(x, rows, cols, x8, scale, xhat, stream=None) -> int:
    return library().dsa_quantize_fp8(_p(x), int(rows), int(cols), _p(x8), _p(scale), _p(xhat),
                                      _stream(stream))


def dsa_index_scores_fp8(dims, q8, q_scale, k8, k_scale, w_idx, scores, ld_scores, workspace,
                         workspace_bytes=None, stream=None) -> int:
    return library().dsa_index_scores_fp8(_dims(dims), _p(q8), _p(q_scale), _p(k8), _p(k_scale),
                                          _p(w_idx), _p(scores), int(ld_scores), _p(workspace),
                                          _nbytes(workspace, workspace_bytes), _stream(stream))


def dsa_decode_layer(dims, q, latent, rope, q_idx, k_idx, w_idx, out, lse, idx_out, workspace,
                     workspace_bytes=None, stream=None) -> int:
    return library().dsa_decode_layer(_dims(dims), _p(q), _p(latent), _p(rope), _p(q_idx),
                                      _p(k_idx), _p(w_idx), _p(out), _p(lse), _p(idx_out),
                                      _p(workspace), _nbytes(workspace, workspace_bytes),
                                      _stream(stream))


def dsa_prefill_layer_noalloc(dims, q, latent, rope, q_idx, k_idx, w_idx, out, lse, idx_out,
                              device_status=None, stream=None) -> int:
    """The layer on the library's static scratch array (no workspace argument)."""
    return library().dsa_prefill_layer_noalloc(_dims(dims), _p(q), _p(latent), _p(rope),
                                               _p(q_idx), _p(k_idx), _p(w_idx), _p(out), _p(lse),
                                               _p(idx_out), _p(device_status), _stream(stream))


def dsa_prefill_layer_host(dims, q, latent, rope, q_idx, k_idx, w_idx, out, lse, idx_out, dev,
                           workspace, streams, events, n_sub=4, workspace_bytes=None) -> int:
    """The layer on host buffers (q .. idx_out: page-locked host tensors or
    addresses), copies overlapped with the compute over n_sub query
    sub-chunks. dev maps the names of dsa_device_tensors to device tensors or
    addresses; streams are three CUDA streams (copy in, compute, copy out),
    events two CUDA events (torch.cuda.Event or raw cudaEvent_t addresses)."""
    d = dsa_device_tensors(*[_p(dev.get(name)) for name, _ in dsa_device_tensors._fields_])
    st = (_P * 3)(*[_stream(x) for x in streams])
    ev = (_P * 2)(*[_P(x) if isinstance(x, int) else _P(x.cuda_event) for x in events])
    return library().dsa_prefill_layer_host(_dims(dims), _p(q), _p(latent), _p(rope), _p(q_idx),
                                            _p(k_idx), _p(w_idx), _p(out), _p(lse), _p(idx_out),
                                            ctypes.byref(d), _p(workspace),
                                            _nbytes(workspace, workspace_bytes), st, ev, int(n_sub))


def dsa_selftest_bounded_wait(workspace, cycles=None, workspace_bytes=None, stream=None) -> int:
    """One CTA whose bounded waits give up (see include/dsa.h); cycles is an
    optional device int64 tensor of 2 elements."""
    return library().dsa_selftest_bounded_wait(_p(workspace), _nbytes(workspace, workspace_bytes),
                                               _p(cycles), _stream(stream))


def dsa_selftest_mma_layout(workspace, workspace_bytes=None, stream=None):
    """The tensor-core layout self-test (see include/dsa.h): returns (status,
    [wrong elements of each of the four forms], [cycles per MMA of each form])."""
    counts = (ctypes.c_int32 * 4)()
    cycles = (ctypes.c_float * 4)()
    st = library().dsa_selftest_mma_layout(_p(workspace), _nbytes(workspace, workspace_bytes),
                                           counts, cycles, _stream(stream))
    return st, list(counts), list(cycles)


def dsa_device_status(workspace, stream=None) -> int:
    return library().dsa_device_status(_p(workspace), _stream(stream))


def dsa_status_string(status: int) -> str:
    return library().dsa_status_string(int(status)).decode()


def check(status: int) -> None:
    """Raises DsaError unless status is DSA_OK."""
    if status != DSA_OK:
        raise DsaError(status)



def dsa_partition_queries(dims, n_parts: int, starts=None):
    """Query ranges of one chunk over n_parts ranks (see include/dsa.h).
    Returns (status, starts) with starts a list of n_parts + 1 row offsets."""
    arr = (ctypes.c_int32 * (int(n_parts) + 1))() if n_parts >= 1 else (ctypes.c_int32 * 1)()
    st = library().dsa_partition_queries(_dims(dims), int(n_parts), arr)
    out = list(arr)
    if starts is not None:
        starts[:] = out
    return st, out
