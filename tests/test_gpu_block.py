"""Block-sparse attention (dsa_sparse_attn_block): groups of 1 or 2
neighbouring queries share the gather of the union of their selections, with
per-query masks. Outputs against the float64 oracle on the same selections."""
import numpy as np
import pytest

import workloads
from workloads import make_dims

from dsa_test_util import assert_attn_close, dev, empty_bf16, host_bf16_as_f32, stage, workspace

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_prefill_dsa_b200 as m

    m.library()
    return m


def _block(dsa, d, xd, idx, qb):
    import torch

    out = empty_bf16(d.n_q, d.n_heads, d.d_latent)
    lse = torch.empty(d.n_q, d.n_heads, dtype=torch.float32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_BLOCK_ATTN))
    dsa.check(dsa.dsa_sparse_attn_block(d, xd["q"], xd["latent"], xd["rope"], dev(idx), out, lse,
                                        qb, ws))
    dsa.check(dsa.dsa_device_status(ws))
    return host_bf16_as_f32(out), lse.cpu().numpy()


def _reduced(name, n_q, w_mode=None):
    wl = workloads.BY_NAME[name]
    d0 = wl.dims
    d = make_dims(n_q, d0.ctx_len - n_q, d0.ctx_len, d0.n_heads, d0.d_latent, d0.d_rope,
                  d0.n_idx_heads, d0.d_idx, d0.top_k, d0.softmax_scale)
    if w_mode is None:
        w_mode = "ones" if wl.kind == "ternary_ties" else "uniform"
    return d, workloads.generate(d, wl.seed + 300, wl.kind, w_mode)


@pytest.mark.parametrize("qb", [1, 2])
@pytest.mark.parametrize("name,n_q", [
    ("tiny_256q", 75),        # k = 64, 4 heads (padded MMA columns), odd query count
    ("chunk8k_ctx17k", 41),   # sin-biased keys: the neighbours' selections overlap most here
    ("ties_4k_ctx8k", 36),    # repeated latent rows, integer indexer scores
])
def test_block_attn_matches_oracle(dsa, oracle_lib, qb, name, n_q):
    d, x = _reduced(name, n_q)
    _, _, ref_idx = oracle_lib.prefill_layer(d, **x)
    ref_out, ref_lse = oracle_lib.sparse_attn(d, x["q"], x["latent"], x["rope"], ref_idx)
    out, lse = _block(dsa, d, stage(x), ref_idx, qb)
    assert_attn_close(out, ref_out)
    finite = np.isfinite(ref_lse)
    np.testing.assert_allclose(lse[finite], ref_lse[finite], rtol=0, atol=2e-3)


@pytest.mark.parametrize("qb", [1, 2])
def test_block_attn_on_given_sets(dsa, oracle_lib, qb):
    """Shuffled order, a short list, a row with no key (out 0, lse -inf) and a
    group whose two rows share no key."""
    d, x = _reduced("chunk2k_ctx8k", 10)
    _, _, ref_idx = oracle_lib.prefill_layer(d, **x)
    rng = np.random.default_rng(8)
    idx = np.stack([rng.permutation(r) for r in ref_idx]).astype(np.int32)
    idx[3, 200:] = -1
    idx[5, :] = -1
    idx[6, :] = -1
    idx[6, :100] = np.arange(100)           # row 6 keeps keys 0..99 only,
    idx[7, :] = -1
    idx[7, :100] = np.arange(100, 200)      # row 7 keys 100..199: disjoint from its neighbour
    ref_out, ref_lse = oracle_lib.sparse_attn(d, x["q"], x["latent"], x["rope"], idx)
    out, lse = _block(dsa, d, stage(x), idx, qb)
    assert_attn_close(out, ref_out)
    assert np.all(out[5] == 0) and np.all(np.isneginf(lse[5]))
    finite = np.isfinite(ref_lse)
    np.testing.assert_allclose(lse[finite], ref_lse[finite], rtol=0, atol=2e-3)


def test_block_attn_reports_future_keys(dsa):
    d, x = _reduced("chunk2k_ctx8k", 4)
    idx = np.tile(np.arange(d.top_k, dtype=np.int32), (d.n_q, 1))
    idx[0, 3] = d.q_pos0 + 2
    import torch

    out = empty_bf16(d.n_q, d.n_heads, d.d_latent)
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_BLOCK_ATTN))
    xd = stage(x)
    dsa.check(dsa.dsa_sparse_attn_block(d, xd["q"], xd["latent"], xd["rope"], dev(idx), out, None,
                                        2, ws))
    assert dsa.dsa_device_status(ws) == dsa.DSA_ERR_RANGE
    assert dsa.dsa_sparse_attn_block(d, xd["q"], xd["latent"], xd["rope"], dev(idx), out, None,
                                     3, ws) == dsa.DSA_ERR_DIMS
    torch.cuda.synchronize()
