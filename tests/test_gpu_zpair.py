"""The attention on SM pairs (DSA_FLAG_ATTN_PAIR: a cluster of two CTAs per
query, each gathering half of every key's dims, S and P halves exchanged
through distributed shared memory) against the float64 oracle, on the layer
and on given sets. Collected after the other parity files, since it is the
newest kernel."""
import dataclasses

import numpy as np
import pytest

import workloads
from workloads import make_dims

from dsa_test_util import assert_attn_close, dev, empty_bf16, host_bf16_as_f32, run_layer, stage, workspace

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_prefill_dsa_b200 as m

    m.library()
    return m


def _reduced(name, n_q):
    wl = workloads.BY_NAME[name]
    d0 = wl.dims
    d = make_dims(n_q, d0.ctx_len - n_q, d0.ctx_len, d0.n_heads, d0.d_latent, d0.d_rope,
                  d0.n_idx_heads, d0.d_idx, d0.top_k, d0.softmax_scale)
    w_mode = "ones" if wl.kind == "ternary_ties" else "uniform"
    return d, workloads.generate(d, wl.seed + 700, wl.kind, w_mode)


@pytest.mark.parametrize("name,n_q", [("chunk2k_ctx8k", 157), ("chunk8k_ctx17k", 131),
                                      ("ties_4k_ctx8k", 149), ("chunk16k_ctx48k", 40)])
def test_pair_layer_matches_oracle(dsa, oracle_lib, name, n_q):
    d, x = _reduced(name, n_q)
    dp = dataclasses.replace(d, flags=dsa.DSA_FLAG_ATTN_PAIR)
    xd = stage(x)
    out, lse, idx = run_layer(dsa, dp, xd)
    ref_out, ref_lse, ref_idx = oracle_lib.prefill_layer(d, **x)
    assert np.array_equal(idx, ref_idx)
    assert_attn_close(out, ref_out)
    finite = np.isfinite(ref_lse)
    np.testing.assert_allclose(lse[finite], ref_lse[finite], rtol=0, atol=2e-3)


@pytest.mark.parametrize("n_q,q_pos0,T,k", [(1, 0, 1, 2048), (70, 930, 1000, 500), (33, 0, 33, 2048)])
def test_pair_layer_edge_shapes(dsa, oracle_lib, n_q, q_pos0, T, k):
    d = make_dims(n_q, q_pos0, T, 32, 512, 64, 32, 128, k)
    x = workloads.generate(d, 21, "normal", "uniform")
    out, lse, idx = run_layer(dsa, dataclasses.replace(d, flags=dsa.DSA_FLAG_ATTN_PAIR), stage(x))
    ref_out, ref_lse, ref_idx = oracle_lib.prefill_layer(d, **x)
    assert np.array_equal(idx, ref_idx)
    assert_attn_close(out, ref_out)


def test_pair_attn_on_given_sets(dsa, oracle_lib):
    """Shuffled order, a short list and a row with no key (out 0, lse -inf)."""
    import torch

    d, x = _reduced("chunk2k_ctx8k", 50)
    _, _, ref_idx = oracle_lib.prefill_layer(d, **x)
    rng = np.random.default_rng(3)
    idx = np.stack([rng.permutation(r) for r in ref_idx]).astype(np.int32)
    idx[7, 100:] = -1
    idx[8, :] = -1
    ref_out, ref_lse = oracle_lib.sparse_attn(d, x["q"], x["latent"], x["rope"], idx)
    xd = stage(x)
    out = empty_bf16(d.n_q, d.n_heads, d.d_latent)
    lse = torch.empty(d.n_q, d.n_heads, dtype=torch.float32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_ATTN))
    dp = dataclasses.replace(d, flags=dsa.DSA_FLAG_ATTN_PAIR)
    dsa.check(dsa.dsa_sparse_attn_prefill(dp, xd["q"], xd["latent"], xd["rope"], dev(idx), out, lse, ws))
    dsa.check(dsa.dsa_device_status(ws))
    o = host_bf16_as_f32(out)
    assert_attn_close(o, ref_out)
    assert np.all(o[8] == 0) and np.all(np.isneginf(lse.cpu().numpy()[8]))


def test_pair_and_single_sm_agree_on_the_bench_chunk(dsa):
    """The full 8,192-query chunk in the bench's launch configuration: the
    pair kernel's outputs against the one-SM kernel's, within the attention
    tolerance, and the same selections."""
    d, x = workloads.workload_inputs("chunk8k_ctx17k")
    xd = stage(x)
    out1, lse1, idx1 = run_layer(dsa, d, xd)
    out2, lse2, idx2 = run_layer(dsa, dataclasses.replace(d, flags=dsa.DSA_FLAG_ATTN_PAIR), xd)
    assert np.array_equal(idx1, idx2)
    assert_attn_close(out2, out1.astype(np.float64))
