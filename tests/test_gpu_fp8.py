"""The FP8 indexer variant through the C ABI against the float64 oracle: e4m3
codes, scales and dequantized rows bit-exact; FP8 scores within the certified
bound of the oracle's scores of the dequantized rows; the exact top-k under the
FP8 contract bit-exact on reduced chunks; the layer's outputs within the
attention tolerance."""
import dataclasses

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


def _quantize(dsa, x_bits):
    import torch

    rows, cols = int(np.prod(x_bits.shape[:-1])), x_bits.shape[-1]
    x8 = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    sc = torch.empty(rows, dtype=torch.float32, device="cuda")
    xh = torch.empty(rows, cols, dtype=torch.int16, device="cuda")
    dsa.check(dsa.dsa_quantize_fp8(dev(x_bits.view(np.int16).reshape(rows, cols)), rows, cols,
                                   x8, sc, xh))
    torch.cuda.synchronize()
    return (x8.cpu().numpy().reshape(x_bits.shape), sc.cpu().numpy().reshape(x_bits.shape[:-1]),
            xh.cpu().numpy().view(np.uint16).reshape(x_bits.shape))


def test_quantize_matches_oracle(dsa, oracle_lib):
    d, x = workloads.workload_inputs("chunk2k_ctx8k")
    rng = np.random.default_rng(3)
    extra = rng.standard_normal((8, 128)).astype(np.float32)
    extra[0] = 0.0
    extra[1] *= 1e-30
    extra[2, ::2] = -0.0
    extra[3] = np.round(extra[3] * 16) / 16
    for arr in (x["k_idx"], x["q_idx"], workloads.to_bf16_bits(extra)):
        g8, gs, gh = _quantize(dsa, arr)
        r8, rs, rh = oracle_lib.quantize_fp8(arr)
        assert np.array_equal(g8, r8) and np.array_equal(gs, rs) and np.array_equal(gh, rh)


def _reduced(name, n_q, w_mode=None):
    wl = workloads.BY_NAME[name]
    d0 = wl.dims
    d = make_dims(n_q, d0.ctx_len - n_q, d0.ctx_len, d0.n_heads, d0.d_latent, d0.d_rope,
                  d0.n_idx_heads, d0.d_idx, d0.top_k, d0.softmax_scale)
    if w_mode is None:
        w_mode = "ones" if wl.kind == "ternary_ties" else "uniform"
    return d, workloads.generate(d, wl.seed + 500, wl.kind, w_mode)


@pytest.mark.parametrize("name,n_q", [("chunk2k_ctx8k", 64), ("chunk16k_ctx48k", 16),
                                      ("ties_4k_ctx8k", 64)])
def test_fp8_scores_within_certified_bound(dsa, oracle_lib, name, n_q):
    import torch

    d, x = _reduced(name, n_q)
    q8, qs, qh = oracle_lib.quantize_fp8(x["q_idx"])
    k8, ks, kh = oracle_lib.quantize_fp8(x["k_idx"])
    ld = (d.ctx_len + 3) // 4 * 4
    sc = torch.full((d.n_q, ld), float("nan"), dtype=torch.float32, device="cuda")
    ws = workspace(256)
    dsa.check(dsa.dsa_index_scores_fp8(d, dev(q8), dev(qs), dev(k8), dev(ks), dev(x["w_idx"]), sc,
                                       ld, ws))
    torch.cuda.synchronize()
    f32 = sc.cpu().numpy()
    ref = oracle_lib.index_scores(d, qh, kh, x["w_idx"])
    qi = workloads.bf16_bits_to_f32(qh).astype(np.float64)
    ki = workloads.bf16_bits_to_f32(kh).astype(np.float64)
    A = (np.abs(x["w_idx"].astype(np.float64)) * np.linalg.norm(qi, axis=2)).sum(axis=1)
    kmax = np.linalg.norm(ki, axis=1).max()
    worst = 0.0
    for i in range(d.n_q):
        t = d.q_pos0 + i
        err = np.abs(f32[i, : t + 1].astype(np.float64) - ref[i, : t + 1]).max()
        worst = max(worst, err / (A[i] * kmax))
    print(f"\n{name} fp8: worst |F-X| / (A_t Kmax) = {worst:.3e}")
    assert worst <= (2.0 ** -15 + 2.0 ** -17) / 16


@pytest.mark.parametrize("name,n_q", [("tiny_256q", 256), ("chunk8k_ctx17k", 131),
                                      ("ties_4k_ctx8k", 149), ("chunk16k_ctx48k", 24)])
def test_fp8_layer_matches_oracle(dsa, oracle_lib, name, n_q):
    if name == "tiny_256q":
        d, x = workloads.workload_inputs(name)
    else:
        d, x = _reduced(name, n_q)
    _, _, qh = oracle_lib.quantize_fp8(x["q_idx"])
    _, _, kh = oracle_lib.quantize_fp8(x["k_idx"])
    ref_idx = oracle_lib.topk_select(d, oracle_lib.index_scores(d, qh, kh, x["w_idx"]))
    ref_out, ref_lse = oracle_lib.sparse_attn(d, x["q"], x["latent"], x["rope"], ref_idx)
    df = dataclasses.replace(d, flags=dsa.DSA_FLAG_FP8_INDEXER)
    out, lse, idx = run_layer(dsa, df, stage(x))
    assert np.array_equal(idx, ref_idx)
    assert_attn_close(out, ref_out)
    finite = np.isfinite(ref_lse)
    np.testing.assert_allclose(lse[finite], ref_lse[finite], rtol=0, atol=2e-3)


def test_fp8_flag_is_refused_by_single_step_calls(dsa):
    d = dataclasses.replace(make_dims(4, 60, 64, 32, 512, 64, 32, 128, 16),
                            flags=dsa.DSA_FLAG_FP8_INDEXER)
    ws = workspace(256)
    assert dsa.dsa_index_scores(d, 16, 16, 16, 16, 64, ws) == dsa.DSA_ERR_DIMS
    assert dsa.dsa_workspace_size(d, dsa.DSA_WS_LAYER) > dsa.dsa_workspace_size(
        dataclasses.replace(d, flags=0), dsa.DSA_WS_LAYER)
