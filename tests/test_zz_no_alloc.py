"""dsa_prefill_layer_noalloc: the layer for callers that cannot allocate device
memory (plugin or callback code handed only its input and output buffers, or
code that must not touch the allocator while a pool is shared or captured).
Its scratch is a static device array inside the library; this file checks
that the call matches dsa_prefill_layer on two calls in a row and that it
refuses chunks larger than that array. It sits last in collection order."""
import numpy as np
import pytest

import workloads
from workloads import make_dims

from dsa_test_util import empty_bf16, host_bf16_as_f32, run_layer, stage

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_prefill_dsa_b200 as m

    m.library()
    return m


def _noalloc(dsa, d, xd):
    import torch

    out = empty_bf16(d.n_q, d.n_heads, d.d_latent)
    lse = torch.empty(d.n_q, d.n_heads, dtype=torch.float32, device="cuda")
    idx = torch.empty(d.n_q, d.top_k, dtype=torch.int32, device="cuda")
    status = torch.full((1,), 77, dtype=torch.int32, device="cuda")
    dsa.check(dsa.dsa_prefill_layer_noalloc(d, xd["q"], xd["latent"], xd["rope"], xd["q_idx"],
                                            xd["k_idx"], xd["w_idx"], out, lse, idx, status))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return host_bf16_as_f32(out), lse.cpu().numpy(), idx.cpu().numpy()


def _reduced_chunk():
    wl = workloads.BY_NAME["chunk2k_ctx8k"]
    d0 = wl.dims
    d = make_dims(157, d0.ctx_len - 157, d0.ctx_len, d0.n_heads, d0.d_latent, d0.d_rope,
                  d0.n_idx_heads, d0.d_idx, d0.top_k, d0.softmax_scale)
    return d, workloads.generate(d, 77, "normal", "uniform")


def test_noalloc_matches_layer_on_two_calls_in_a_row(dsa):
    """Both calls run the same kernels on the same inputs, so the results are
    the same bits, not merely within the attention tolerance."""
    cases = [workloads.workload_inputs("tiny_256q"), _reduced_chunk()]
    staged = [(d, stage(x)) for d, x in cases]
    results = [_noalloc(dsa, d, xd) for d, xd in staged]  # two calls in a row
    for (d, xd), (out, lse, idx) in zip(staged, results):
        ref_out, ref_lse, ref_idx = run_layer(dsa, d, xd)
        assert np.array_equal(idx, ref_idx)
        assert np.array_equal(out, ref_out)
        assert np.array_equal(lse, ref_lse)


def test_noalloc_accepts_the_l2_sub_block_schedule(dsa):
    """DSA_FLAG_L2_SCORES through the call without allocation: the same bits as
    dsa_prefill_layer with and without the flag (the 157-query chunk is one
    sub-block, so the schedule and workspace equal the default's)."""
    import dataclasses

    d, x = _reduced_chunk()
    xd = stage(x)
    dl2 = dataclasses.replace(d, flags=dsa.DSA_FLAG_L2_SCORES)
    out, lse, idx = _noalloc(dsa, dl2, xd)
    ref_out, ref_lse, ref_idx = run_layer(dsa, d, xd)
    assert np.array_equal(idx, ref_idx)
    assert np.array_equal(out, ref_out)
    assert np.array_equal(lse, ref_lse)


def _scratch_bytes(n_q, T, k):
    return 256 + n_q * ((T + 127) // 128 * 128 + k) * 4


def test_noalloc_at_its_scratch_limit(dsa):
    """1,024 queries at top_k 2048 fit up to a 6,016-token context: the
    largest such chunk runs (bit-identical to dsa_prefill_layer); one more
    token needs 128 more score columns per row and is refused."""
    import torch

    fits = make_dims(1024, 6016 - 1024, 6016, 32, 512, 64, 32, 128, 2048)
    over = make_dims(1024, 6017 - 1024, 6017, 32, 512, 64, 32, 128, 2048)
    assert _scratch_bytes(1024, 6016, 2048) <= dsa.DSA_NOALLOC_SCRATCH_BYTES
    assert _scratch_bytes(1024, 6017, 2048) > dsa.DSA_NOALLOC_SCRATCH_BYTES
    assert dsa.dsa_workspace_size(fits, dsa.DSA_WS_LAYER) == _scratch_bytes(1024, 6016, 2048)
    xd = stage(workloads.generate(fits, 78, "normal", "uniform"))
    out, lse, idx = _noalloc(dsa, fits, xd)
    ref_out, ref_lse, ref_idx = run_layer(dsa, fits, xd)
    assert np.array_equal(idx, ref_idx) and np.array_equal(out, ref_out)
    assert np.array_equal(lse, ref_lse)
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(16, dtype=torch.float32, device="cuda")
    assert (dsa.dsa_prefill_layer_noalloc(over, x, x, x, x, x, w, x, None, None, None)
            == dsa.DSA_ERR_SCRATCH_LIMIT)


def test_noalloc_refuses_chunks_beyond_its_scratch(dsa):
    import torch

    d = workloads.BY_NAME["chunk8k_ctx17k"].dims
    assert dsa.dsa_workspace_size(d, dsa.DSA_WS_LAYER) > dsa.DSA_NOALLOC_SCRATCH_BYTES
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(16, dtype=torch.float32, device="cuda")
    out = torch.full((16,), 5.0, dtype=torch.bfloat16, device="cuda")
    st = dsa.dsa_prefill_layer_noalloc(d, x, x, x, x, x, w, out, None, None, None)
    assert st == dsa.DSA_ERR_SCRATCH_LIMIT
    assert "static array" in dsa.dsa_status_string(st)
    torch.cuda.synchronize()
    assert torch.all(out == 5.0)
