"""GPU parity at contexts past 49,152 keys.

A row of more than 49,152 keys does not fit one CTA's shared memory, so the
top-k selects in two passes: the top-k of every segment of at most 32,768 keys,
then the top-k among those candidates. The selections must still be the
oracle's, bit for bit: across segment boundaries, with ties spanning segments,
for rows that end in the first segment of a two-pass launch, and through the
whole layer and the decode step at the longest supported context.
"""
import numpy as np
import pytest

import workloads
from workloads import make_dims

from dsa_test_util import assert_attn_close, dev, run_layer, stage, workspace

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_prefill_dsa_b200 as m

    m.library()
    return m


def _select_f32(dsa, d, s32):
    import torch

    idx = torch.empty(d.n_q, d.top_k, dtype=torch.int32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_TOPK))
    dsa.check(dsa.dsa_topk_select(d, dev(s32), s32.shape[1], None, None, None, idx, ws))
    dsa.check(dsa.dsa_device_status(ws))
    return idx.cpu().numpy()


@pytest.mark.parametrize("n_q,q_pos0,T,k", [
    (8, 131064, 131072, 2048),   # four segments of 32,768 keys
    (12, 49146, 49158, 2048),    # two segments of 24,580; rows on both sides of 49,152
    (40, 65500, 65540, 2048),    # three segments of 21,848
    (6, 98300, 98306, 1),        # k = 1
    (5, 70000, 70005, 777),      # an odd k
])
def test_two_level_on_float32_scores_is_bitexact(dsa, oracle_lib, n_q, q_pos0, T, k):
    rng = np.random.default_rng(n_q * 7919 + T)
    d = make_dims(n_q, q_pos0, T, 32, 512, 64, 32, 128, k)
    ld = (T + 3) // 4 * 4
    # a few dozen distinct values: every segment holds many ties of the k-th value
    s32 = rng.integers(0, 40, size=(n_q, ld)).astype(np.float32) * np.float32(0.25)
    s32[:, ::5] = -s32[:, ::5]
    s32[0, :] = 0.0                                   # all tied: the lowest keys win
    s32[1, ::2] = -0.0                                # -0 and +0 tie
    s32[1, 1::2] = 0.0
    if n_q > 2:
        s32[2, :] = np.float32(-1.0)                  # the winners all in the last segment
        s32[2, q_pos0 + 2 - 3 * k // 2:q_pos0 + 3] = np.float32(1.0)
    if n_q > 3:
        s32[3, :] = -np.arange(ld, dtype=np.float32)  # strictly decreasing: keys 0..k-1
    if n_q > 4:
        s32[4, 32767:32770] = np.float32(1e30)        # a maximum on a segment boundary
    got = _select_f32(dsa, d, s32)
    ref = oracle_lib.topk_select(d, s32)
    assert np.array_equal(got, ref)


def test_two_level_exact_mode_longest_context(dsa, oracle_lib):
    """Indexer scores and the exact float64 order at 131,072 keys."""
    import torch

    n_q, T = 8, 131072
    d = make_dims(n_q, T - n_q, T, 32, 512, 64, 32, 128, 2048)
    x = workloads.generate(d, 41, "sin_bias", "uniform")
    xd = stage(x)
    ld = T
    sc = torch.empty(n_q, ld, dtype=torch.float32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_TOPK))
    dsa.check(dsa.dsa_index_scores(d, xd["q_idx"], xd["k_idx"], xd["w_idx"], sc, ld, ws))
    idx = torch.empty(n_q, d.top_k, dtype=torch.int32, device="cuda")
    dsa.check(dsa.dsa_topk_select(d, sc, ld, xd["q_idx"], xd["k_idx"], xd["w_idx"], idx, ws))
    dsa.check(dsa.dsa_device_status(ws))
    ref = oracle_lib.topk_select(d, oracle_lib.index_scores(d, x["q_idx"], x["k_idx"], x["w_idx"]))
    assert np.array_equal(idx.cpu().numpy(), ref)


@pytest.mark.parametrize("k,kind", [(64, "normal"), (2048, "normal"), (2048, "ternary_ties")])
def test_layer_one_chunk_of_49160_queries(dsa, oracle_lib, k, kind):
    """A 49,160-token prompt in one chunk (small head shapes): the two-pass
    launch holds rows of every length, from one key to 49,160; sampled rows on
    both sides of the segment boundary (24,580) match the oracle."""
    T = 49160
    d = make_dims(T, 0, T, 4, 64, 16, 2, 32, k)
    x = workloads.generate(d, 43 + k, kind, "uniform")
    out, lse, idx = run_layer(dsa, d, stage(x))
    rows = np.array([0, 1, k - 1, k, k + 1, 24579, 24580, 24581, 24580 + k - 1, 24580 + k,
                     24580 + k + 1, 30001, 49151, 49152, 49159], dtype=np.int32)
    ref_out, ref_lse, ref_idx = oracle_lib.prefill_layer(d, **x, rows=rows)
    bad = np.nonzero(~np.all(idx[rows] == ref_idx, axis=1))[0]
    assert bad.size == 0, f"rows {rows[bad]} differ in their selected sets"
    assert_attn_close(out[rows], ref_out)
    finite = np.isfinite(ref_lse)
    np.testing.assert_allclose(lse[rows][finite], ref_lse[finite], rtol=0, atol=2e-3)


def test_layer_at_the_longest_context(dsa, oracle_lib):
    """The whole layer, full head shapes, 131,072-token context: sampled rows."""
    n_q, T = 16, 131072
    d = make_dims(n_q, T - n_q, T, 32, 512, 64, 32, 128, 2048)
    x = workloads.generate(d, 47, "normal", "uniform")
    out, lse, idx = run_layer(dsa, d, stage(x))
    rows = np.array([0, 7, 15], dtype=np.int32)
    ref_out, ref_lse, ref_idx = oracle_lib.prefill_layer(d, **x, rows=rows)
    assert np.array_equal(idx[rows], ref_idx)
    assert_attn_close(out[rows], ref_out)
    finite = np.isfinite(ref_lse)
    np.testing.assert_allclose(lse[rows][finite], ref_lse[finite], rtol=0, atol=2e-3)


def test_decode_step_at_the_longest_context(dsa, oracle_lib):
    import torch

    from dsa_test_util import empty_bf16, host_bf16_as_f32

    T = 131072
    d = make_dims(1, T - 1, T, 32, 512, 64, 32, 128, 2048)
    x = workloads.generate(d, 53, "normal", "uniform")
    xd = stage(x)
    out = empty_bf16(1, d.n_heads, d.d_latent)
    lse = torch.empty(1, d.n_heads, dtype=torch.float32, device="cuda")
    idx = torch.empty(1, d.top_k, dtype=torch.int32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_DECODE_LAYER))
    dsa.check(dsa.dsa_decode_layer(d, xd["q"], xd["latent"], xd["rope"], xd["q_idx"],
                                   xd["k_idx"], xd["w_idx"], out, lse, idx, ws))
    dsa.check(dsa.dsa_device_status(ws))
    ref_out, ref_lse, ref_idx = oracle_lib.prefill_layer(d, **x)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert_attn_close(host_bf16_as_f32(out), ref_out)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=2e-3)
