"""Helpers shared by the GPU tests: device staging and the parity metrics.

The CUDA path is reached only through the C ABI (the ctypes binding); torch
only allocates device memory and provides the stream.
"""
from __future__ import annotations

import numpy as np

# Output tolerance of the attention against the float64 oracle: bf16 inputs
# and outputs with float32 accumulation.
MAX_ABS = 2e-2
REL_L2 = 5e-3


def torch_mod():
    import torch

    return torch


def dev_bf16(a):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def dev(a):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bf16_as_f32(t):
    torch = torch_mod()
    bits = t.view(torch.int16).cpu().numpy().view(np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def empty_bf16(*shape):
    torch = torch_mod()
    return torch.empty(*shape, dtype=torch.bfloat16, device="cuda")


def workspace(nbytes):
    torch = torch_mod()
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device="cuda")


def stage(x):
    """Moves one chunk's inputs (numpy, bf16 as uint16) to the device."""
    return dict(q=dev_bf16(x["q"]), latent=dev_bf16(x["latent"]), rope=dev_bf16(x["rope"]),
                q_idx=dev_bf16(x["q_idx"]), k_idx=dev_bf16(x["k_idx"]), w_idx=dev(x["w_idx"]))


def run_layer(dsa, d, xd, want_lse=True):
    """dsa_prefill_layer through the C ABI. Returns (out f32 [n_q,H,Dc], lse, idx)."""
    torch = torch_mod()
    out = empty_bf16(d.n_q, d.n_heads, d.d_latent)
    lse = torch.empty(d.n_q, d.n_heads, dtype=torch.float32, device="cuda") if want_lse else None
    idx = torch.empty(d.n_q, d.top_k, dtype=torch.int32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_LAYER))
    dsa.check(dsa.dsa_prefill_layer(d, xd["q"], xd["latent"], xd["rope"], xd["q_idx"],
                                    xd["k_idx"], xd["w_idx"], out, lse, idx, ws))
    dsa.check(dsa.dsa_device_status(ws))
    return (host_bf16_as_f32(out), lse.cpu().numpy() if want_lse else None, idx.cpu().numpy())


def attn_errors(out_gpu, out_ref):
    diff = out_gpu.astype(np.float64) - out_ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    ref_norm = float(np.linalg.norm(out_ref))
    rel = float(np.linalg.norm(diff) / ref_norm) if ref_norm > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_attn_close(out_gpu, out_ref):
    max_abs, rel = attn_errors(out_gpu, out_ref)
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel
