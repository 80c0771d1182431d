"""Seeded synthetic inputs for one DSA prefill chunk.

This module is shared by the tests, the bench and the smoke check. It draws
random tensors and nothing else: it holds none of the layer's arithmetic
(no scores, selection or attention), so neither the CUDA path nor the oracle
depends on the other through it.

Recipe (the same for every workload):
  * ``numpy.random.Generator(PCG64(seed))``;
  * draws in the order q, latent, rope, q_idx, k_idx, w_idx;
  * normal draws are ``standard_normal(dtype=float32)`` rounded to bf16 with
    round-to-nearest-even; bf16 tensors travel as uint16 bit patterns;
  * indexer head weights are float32 ``U(0,1) / sqrt(H_I)`` (drawn in float64,
    rounded once to float32), never rounded to bf16.

The five named workloads follow the layer sizes the feedman.me post
(feedman.me/posts/wy2HU) profiles: 2,048- and 8,192-token prefill chunks, a
512-wide latent KV and top-2048 selection, plus a tiny case and a tie stress.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Dims:
    n_q: int
    q_pos0: int
    ctx_len: int
    n_heads: int
    d_latent: int
    d_rope: int
    n_idx_heads: int
    d_idx: int
    top_k: int
    softmax_scale: float
    flags: int = 0  # dsa_dims.flags of the C ABI (the oracle ignores it)

    @property
    def d_qk(self) -> int:
        return self.d_latent + self.d_rope


def make_dims(n_q, q_pos0, ctx_len, n_heads, d_latent, d_rope, n_idx_heads, d_idx, top_k,
              softmax_scale=None) -> Dims:
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d_latent + d_rope)
    # The scale is a float32 value on both sides (the C ABI carries a float).
    scale = float(np.float32(softmax_scale))
    return Dims(n_q, q_pos0, ctx_len, n_heads, d_latent, d_rope, n_idx_heads, d_idx, top_k, scale)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dims: Dims
    seed: int
    kind: str  # "normal", "sin_bias", "ternary_ties"
    about: str


WORKLOADS = [
    Workload("tiny_256q", make_dims(256, 0, 256, 4, 64, 16, 2, 32, 64), 0, "normal",
             "256 queries at 0..255 (no prefix), k=64, H=4, Dc=64, Dr=16, indexer 2x32"),
    Workload("chunk2k_ctx8k", make_dims(2048, 6144, 8192, 32, 512, 64, 32, 128, 2048), 1,
             "normal", "2,048-query chunk at 6,144..8,191 of an 8,192 context, k=2048"),
    Workload("chunk8k_ctx17k", make_dims(8192, 9216, 17408, 32, 512, 64, 32, 128, 2048), 2,
             "sin_bias", "8,192-query chunk at 9,216..17,407 of a 17,408 context, k=2048, "
             "k_idx[s,0] += 0.5*sin(s/64)"),
    Workload("chunk16k_ctx48k", make_dims(16384, 32768, 49152, 32, 512, 64, 32, 128, 2048), 3,
             "normal", "16,384-query chunk at 32,768..49,151 of a 49,152 context, k=2048"),
    Workload("ties_4k_ctx8k", make_dims(4096, 4096, 8192, 32, 512, 64, 32, 128, 2048), 4,
             "ternary_ties", "4,096 queries at 4,096..8,191 of 8,192; indexer q/k in {-1,0,1}; "
             "latent/rope rows repeat in blocks of 16; w = 1 (primary) or U(0,1)/sqrt(32)"),
]
BY_NAME = {w.name: w for w in WORKLOADS}

# A longer context than the five workloads above reach: rows of more than
# 49,152 keys, which the top-k selects in two passes. Timed by the bench
# (--workload); the parity tests cover such rows with their own smaller chunks.
LONG_WORKLOADS = [
    Workload("chunk4k_ctx128k", make_dims(4096, 126976, 131072, 32, 512, 64, 32, 128, 2048), 5,
             "normal", "4,096-query chunk at 126,976..131,071 of a 131,072 context, k=2048"),
]
ALL_BY_NAME = {**BY_NAME, **{w.name: w for w in LONG_WORKLOADS}}


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even. Finite inputs."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32)
    rounded = (b + (((b >> 16) & 1) + 0x7FFF)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_bf16(rng, shape):
    return to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


def generate(d: Dims, seed: int, kind: str = "normal", w_mode: str = "uniform") -> dict:
    """Draws one chunk's inputs.

    kind: "normal" (all N(0,1)), "sin_bias" (normal plus 0.5*sin(s/64) added in
    float64 to k_idx[s,0] before rounding), "ternary_ties" (indexer q/k drawn
    uniformly from {-1,0,1}; latent and rope rows 16b..16b+15 copy row 16b).
    w_mode: "uniform" (U(0,1)/sqrt(H_I)) or "ones" (w = 1).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    n_q, T, H = d.n_q, d.ctx_len, d.n_heads
    q = _normal_bf16(rng, (n_q, H, d.d_latent + d.d_rope))
    latent = _normal_bf16(rng, (T, d.d_latent))
    rope = _normal_bf16(rng, (T, d.d_rope))
    if kind == "ternary_ties":
        q_idx = to_bf16_bits(rng.integers(-1, 2, size=(n_q, d.n_idx_heads, d.d_idx)).astype(np.float32))
        k_idx = to_bf16_bits(rng.integers(-1, 2, size=(T, d.d_idx)).astype(np.float32))
        rep = (np.arange(T) // 16) * 16
        latent = np.ascontiguousarray(latent[rep])
        rope = np.ascontiguousarray(rope[rep])
    else:
        q_idx = _normal_bf16(rng, (n_q, d.n_idx_heads, d.d_idx))
        k_f32 = rng.standard_normal(size=(T, d.d_idx), dtype=np.float32)
        if kind == "sin_bias":
            s = np.arange(T, dtype=np.float64)
            k_f32[:, 0] = (k_f32[:, 0].astype(np.float64) + 0.5 * np.sin(s / 64.0)).astype(np.float32)
        elif kind != "normal":
            raise ValueError(kind)
        k_idx = to_bf16_bits(k_f32)
    u = rng.random(size=(n_q, d.n_idx_heads), dtype=np.float64)
    if w_mode == "ones":
        w_idx = np.ones((n_q, d.n_idx_heads), dtype=np.float32)
    elif w_mode == "uniform":
        w_idx = (u / math.sqrt(d.n_idx_heads)).astype(np.float32)
    else:
        raise ValueError(w_mode)
    return dict(q=q, latent=latent, rope=rope, q_idx=q_idx, k_idx=k_idx, w_idx=w_idx)


def workload_inputs(name: str, w_mode: str | None = None) -> tuple[Dims, dict]:
    wl = ALL_BY_NAME[name]
    if w_mode is None:
        w_mode = "ones" if wl.kind == "ternary_ties" else "uniform"
    return wl.dims, generate(wl.dims, wl.seed, wl.kind, w_mode)


def useful_flops(d: Dims) -> dict:
    """Useful floating-point work of one chunk: causal indexer pairs times
    2*H_I*D_I, plus selected keys times 2*H*(Dc+Dr+Dc). Masked or padded work is
    not counted."""
    t = np.arange(d.q_pos0, d.q_pos0 + d.n_q, dtype=np.int64)
    pairs = int((t + 1).sum())
    selected = int(np.minimum(t + 1, d.top_k).sum())
    idx_fl = 2 * d.n_idx_heads * d.d_idx * pairs
    att_fl = 2 * d.n_heads * (d.d_latent + d.d_rope + d.d_latent) * selected
    return dict(pairs=pairs, selected=selected, indexer=idx_fl, attention=att_fl,
                total=idx_fl + att_fl)
