"""Decode-side DSA (chunks of a few queries; a decode step is one query)
through the C ABI against the float64 oracle: dsa_decode_layer and
dsa_sparse_attn_decode spread each query's key tiles over SMs and merge the
partial softmax sums. Selections are bit-exact; outputs are within the
attention tolerance; selections equal those of dsa_prefill_layer."""
import numpy as np
import pytest

import workloads
from workloads import make_dims

from dsa_test_util import (assert_attn_close, dev, empty_bf16, host_bf16_as_f32, run_layer, stage,
                           workspace)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_prefill_dsa_b200 as m

    m.library()
    return m


def _decode_layer(dsa, d, xd):
    import torch

    out = empty_bf16(d.n_q, d.n_heads, d.d_latent)
    lse = torch.empty(d.n_q, d.n_heads, dtype=torch.float32, device="cuda")
    idx = torch.empty(d.n_q, d.top_k, dtype=torch.int32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_DECODE_LAYER))
    dsa.check(dsa.dsa_decode_layer(d, xd["q"], xd["latent"], xd["rope"], xd["q_idx"], xd["k_idx"],
                                   xd["w_idx"], out, lse, idx, ws))
    dsa.check(dsa.dsa_device_status(ws))
    return host_bf16_as_f32(out), lse.cpu().numpy(), idx.cpu().numpy()


@pytest.mark.parametrize("n_q,T,k", [
    (1, 49152, 2048),   # one decode step at the longest context
    (1, 300, 2048),     # fewer causal keys than k: every key kept, three tiles
    (3, 8192, 2048),
    (16, 17408, 2048),  # n_split = 9: ranges of two tiles
    (40, 8192, 500),    # ragged last tile, n_split = 3
])
def test_decode_layer_matches_oracle(dsa, oracle_lib, n_q, T, k):
    d = make_dims(n_q, T - n_q, T, 32, 512, 64, 32, 128, k)
    x = workloads.generate(d, 40 + n_q, "normal", "uniform")
    xd = stage(x)
    out, lse, idx = _decode_layer(dsa, d, xd)
    ref_out, ref_lse, ref_idx = oracle_lib.prefill_layer(d, **x)
    assert np.array_equal(idx, ref_idx)
    assert_attn_close(out, ref_out)
    finite = np.isfinite(ref_lse)
    np.testing.assert_allclose(lse[finite], ref_lse[finite], rtol=0, atol=2e-3)
    _, _, idx_p = run_layer(dsa, d, xd)
    assert np.array_equal(idx, idx_p)


def test_decode_layer_tiny_shape(dsa, oracle_lib):
    d0 = workloads.BY_NAME["tiny_256q"].dims
    d = make_dims(2, 254, 256, d0.n_heads, d0.d_latent, d0.d_rope, d0.n_idx_heads, d0.d_idx,
                  d0.top_k, d0.softmax_scale)
    x = workloads.generate(d, 5, "normal", "uniform")
    out, lse, idx = _decode_layer(dsa, d, stage(x))
    ref_out, ref_lse, ref_idx = oracle_lib.prefill_layer(d, **x)
    assert np.array_equal(idx, ref_idx)
    assert_attn_close(out, ref_out)


def test_sparse_attn_decode_on_given_sets(dsa, oracle_lib):
    """Shuffled order, a short list and a row with no key (out 0, lse -inf)."""
    import torch

    d = make_dims(6, 8186, 8192, 32, 512, 64, 32, 128, 2048)
    x = workloads.generate(d, 6, "normal", "uniform")
    _, _, ref_idx = oracle_lib.prefill_layer(d, **x)
    rng = np.random.default_rng(4)
    idx = np.stack([rng.permutation(r) for r in ref_idx]).astype(np.int32)
    idx[2, 300:] = -1
    idx[4, :] = -1
    ref_out, ref_lse = oracle_lib.sparse_attn(d, x["q"], x["latent"], x["rope"], idx)
    xd = stage(x)
    out = empty_bf16(d.n_q, d.n_heads, d.d_latent)
    lse = torch.empty(d.n_q, d.n_heads, dtype=torch.float32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_DECODE_ATTN))
    dsa.check(dsa.dsa_sparse_attn_decode(d, xd["q"], xd["latent"], xd["rope"], dev(idx), out, lse,
                                         ws))
    dsa.check(dsa.dsa_device_status(ws))
    o = host_bf16_as_f32(out)
    assert_attn_close(o, ref_out)
    l = lse.cpu().numpy()
    assert np.all(o[4] == 0) and np.all(np.isneginf(l[4]))
    finite = np.isfinite(ref_lse)
    np.testing.assert_allclose(l[finite], ref_lse[finite], rtol=0, atol=2e-3)
