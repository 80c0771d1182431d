"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Bar: selected index sets bit-exact; attention outputs within max-abs 2e-2 and
relative L2 5e-3 of the oracle (bf16 in/out, float32 accumulation).
Full element-wise comparisons run on reduced chunks of each workload (the
oracle finishes them in seconds; they still span several tiles and end on a
ragged tail); the full-size workloads, in the launch configuration the bench
times, are compared on sampled query rows that the oracle computes one by one.
"""
import numpy as np
import pytest

import workloads
from workloads import make_dims

from dsa_test_util import (assert_attn_close, attn_errors, dev, dev_bf16, empty_bf16,
                           host_bf16_as_f32, run_layer, stage, workspace)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_prefill_dsa_b200 as m

    m.library()
    return m


def _reduced(name, n_q, w_mode=None):
    wl = workloads.BY_NAME[name]
    d0 = wl.dims
    d = make_dims(n_q, d0.ctx_len - n_q, d0.ctx_len, d0.n_heads, d0.d_latent, d0.d_rope,
                  d0.n_idx_heads, d0.d_idx, d0.top_k, d0.softmax_scale)
    if w_mode is None:
        w_mode = "ones" if wl.kind == "ternary_ties" else "uniform"
    return d, workloads.generate(d, wl.seed + 100, wl.kind, w_mode)


def _compare_layer(oracle_lib, d, x, out, lse, idx, rows=None):
    ref_out, ref_lse, ref_idx = oracle_lib.prefill_layer(d, **x, rows=rows)
    sel = slice(None) if rows is None else rows
    bad = np.nonzero(~np.all(idx[sel] == ref_idx, axis=1))[0]
    assert bad.size == 0, f"{bad.size} rows differ in their selected sets, first row {bad[:4]}"
    assert_attn_close(out[sel], ref_out)
    finite = np.isfinite(ref_lse)
    np.testing.assert_allclose(lse[sel][finite], ref_lse[finite], rtol=0, atol=2e-3)


def test_layer_tiny_workload_full(dsa, oracle_lib):
    d, x = workloads.workload_inputs("tiny_256q")
    out, lse, idx = run_layer(dsa, d, stage(x))
    _compare_layer(oracle_lib, d, x, out, lse, idx)


@pytest.mark.parametrize("name,n_q,w_mode", [
    ("chunk2k_ctx8k", 157, None),
    ("chunk8k_ctx17k", 131, None),
    ("chunk16k_ctx48k", 40, None),
    ("ties_4k_ctx8k", 149, None),
    ("ties_4k_ctx8k", 77, "uniform"),
])
def test_layer_reduced_elementwise(dsa, oracle_lib, name, n_q, w_mode):
    d, x = _reduced(name, n_q, w_mode)
    out, lse, idx = run_layer(dsa, d, stage(x))
    _compare_layer(oracle_lib, d, x, out, lse, idx)


def _golden_selections():
    import importlib.util
    import json
    import os

    here = os.path.join(os.path.dirname(__file__), "golden")
    spec = importlib.util.spec_from_file_location(
        "make_selection_hashes", os.path.join(here, "make_selection_hashes.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    with open(os.path.join(here, "selection_hashes.json")) as f:
        return mod, json.load(f)


_GOLDEN_MOD, _GOLDEN = _golden_selections()
# workloads whose attention outputs are compared on every row; the two large
# chunks are compared on 512 rows spread over the chunk (their selections are
# still checked on every row)
_ALL_ROWS = {"tiny_256q", "chunk2k_ctx8k", "ties_4k_ctx8k"}


@pytest.mark.parametrize("case", sorted(_GOLDEN["cases"]))
def test_layer_full_size_every_row(dsa, oracle_lib, case):
    """The full-size workloads in the bench's launch configuration.

    Selections: every row of the GPU's [n_q, top_k] selection hashes to the
    digest of the float64 oracle's full selection (tests/golden, written from
    oracle/ alone). On a mismatch the oracle recomputes the first differing
    block of rows to name the first wrong row.
    Outputs: the oracle's attention over those (proven identical) selections,
    element-wise on every row of the 256-, 2,048- and 4,096-query chunks and on
    512 rows spread over the 8,192- and 16,384-query chunks.
    """
    import dataclasses

    g = _GOLDEN["cases"][case]
    name, w_mode = g["workload"], g["w_mode"]
    fp8 = g.get("variant", "") == "fp8"
    d, x = workloads.workload_inputs(name, w_mode)
    assert _GOLDEN_MOD.inputs_digest(x) == g["inputs_sha256"], \
        "input recipe changed since the digests were written: rerun make_selection_hashes.py"
    if fp8:  # the FP8 indexer's contract: the dequantized e4m3 rows
        d = dataclasses.replace(d, flags=dsa.DSA_FLAG_FP8_INDEXER)
    out, lse, idx = run_layer(dsa, d, stage(x))
    whole, blocks = _GOLDEN_MOD.selection_digests(idx)
    if whole != g["selection_sha256"]:
        nb = _GOLDEN["block_rows"]
        bad = [b for b, (a, e) in enumerate(zip(blocks, g["block_sha256"])) if a != e]
        rows = np.arange(bad[0] * nb, min(d.n_q, (bad[0] + 1) * nb), dtype=np.int32)
        ref = _GOLDEN_MOD.oracle_selection(d, x, rows=rows, fp8=fp8)
        wrong = rows[~np.all(idx[rows] == ref, axis=1)]
        pytest.fail(f"{len(bad)} blocks of {nb} rows differ; first wrong rows {wrong[:8].tolist()}")
    if name in _ALL_ROWS:
        rows = np.arange(d.n_q, dtype=np.int32)
    else:
        rows = np.unique(np.linspace(0, d.n_q - 1, 512).round().astype(np.int32))
        assert rows.size == 512
    ref_out, ref_lse = oracle_lib.sparse_attn(d, x["q"], x["latent"], x["rope"], idx[rows],
                                              rows=rows)
    assert_attn_close(out[rows], ref_out)
    finite = np.isfinite(ref_lse)
    np.testing.assert_allclose(lse[rows][finite], ref_lse[finite], rtol=0, atol=2e-3)


@pytest.mark.parametrize("name,n_q,w_mode", [
    ("chunk2k_ctx8k", 64, None),
    ("chunk8k_ctx17k", 64, None),    # keys with the sin bias
    ("chunk16k_ctx48k", 24, None),   # 48K-key rows
    ("ties_4k_ctx8k", 64, "ones"),   # integer scores
    ("ties_4k_ctx8k", 64, "uniform"),
])
def test_index_scores_within_certified_bound(dsa, oracle_lib, name, n_q, w_mode):
    """float32 indexer scores stay far inside the bound the exact top-k relies
    on: |F - X| <= (2^-15 + 2^-17) * A_t * max_s ||k_s||, with A_t the sum over
    heads of |w| * ||q||. The bound assumes the tensor core's float32
    accumulation loses no more than one float32 rounding per addition; the
    margin measured here is the evidence for that assumption."""
    import torch

    d, x = _reduced(name, n_q, w_mode)
    xd = stage(x)
    ld = (d.ctx_len + 3) // 4 * 4
    sc = torch.full((d.n_q, ld), float("nan"), dtype=torch.float32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_INDEX_SCORES))
    dsa.check(dsa.dsa_index_scores(d, xd["q_idx"], xd["k_idx"], xd["w_idx"], sc, ld, ws))
    torch.cuda.synchronize()
    f32 = sc.cpu().numpy()
    ref = oracle_lib.index_scores(d, x["q_idx"], x["k_idx"], x["w_idx"])
    qi = workloads.bf16_bits_to_f32(x["q_idx"]).astype(np.float64)
    ki = workloads.bf16_bits_to_f32(x["k_idx"]).astype(np.float64)
    A = (np.abs(x["w_idx"].astype(np.float64)) * np.linalg.norm(qi, axis=2)).sum(axis=1)
    kmax = np.linalg.norm(ki, axis=1).max()
    worst = 0.0
    for i in range(d.n_q):
        t = d.q_pos0 + i
        err = np.abs(f32[i, : t + 1].astype(np.float64) - ref[i, : t + 1]).max()
        if A[i] * kmax > 0:
            worst = max(worst, err / (A[i] * kmax))
    bound = 2.0 ** -15 + 2.0 ** -17
    ratio = bound / worst if worst > 0 else float("inf")
    print(f"\n{name}:{w_mode}: worst |F-X| / (A_t Kmax) = {worst:.3e} "
          f"(bound {bound:.3e}, margin {ratio:.0f}x)")
    assert worst <= bound / 16


def test_topk_on_float32_scores_is_bitexact(dsa, oracle_lib):
    """With no indexer inputs the select orders the given float32 scores."""
    import torch

    rng = np.random.default_rng(7)
    d = make_dims(300, 700, 1000, 32, 512, 64, 32, 128, 256)
    ld = 1000
    s32 = rng.integers(0, 50, size=(d.n_q, ld)).astype(np.float32) * np.float32(0.125)
    s32[:, ::7] = -s32[:, ::7]           # negatives too
    s32[5, :] = 0.0                      # a row of exact ties
    s32[6, ::2] = -0.0                   # -0 and +0 tie
    idx = torch.empty(d.n_q, d.top_k, dtype=torch.int32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_TOPK))
    dsa.check(dsa.dsa_topk_select(d, dev(s32), ld, None, None, None, idx, ws))
    dsa.check(dsa.dsa_device_status(ws))
    ref = oracle_lib.topk_select(d, s32)
    assert np.array_equal(idx.cpu().numpy(), ref)


def test_topk_exact_mode_on_gpu_scores(dsa, oracle_lib):
    """dsa_topk_select with indexer inputs reproduces the float64 order."""
    import torch

    d, x = _reduced("ties_4k_ctx8k", 96)
    xd = stage(x)
    ld = d.ctx_len
    sc = torch.empty(d.n_q, ld, dtype=torch.float32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_TOPK))
    dsa.check(dsa.dsa_index_scores(d, xd["q_idx"], xd["k_idx"], xd["w_idx"], sc, ld, ws))
    idx = torch.empty(d.n_q, d.top_k, dtype=torch.int32, device="cuda")
    dsa.check(dsa.dsa_topk_select(d, sc, ld, xd["q_idx"], xd["k_idx"], xd["w_idx"], idx, ws))
    dsa.check(dsa.dsa_device_status(ws))
    ref = oracle_lib.topk_select(d, oracle_lib.index_scores(d, x["q_idx"], x["k_idx"], x["w_idx"]))
    assert np.array_equal(idx.cpu().numpy(), ref)


@pytest.mark.parametrize("T,kind", [
    (18400, "normal"),          # the window select
    (30000, "normal"),
    (18400, "repeated_keys"),   # 40 distinct key rows: every score ties with hundreds of others,
    (30000, "repeated_keys"),   # the window overflows and the rows are handed back to the bucket
])                              # select (two CTAs per SM at 18,400 keys, one at 30,000)
def test_topk_exact_mode_launch_variants(dsa, oracle_lib, T, kind):
    """The exact mode's kernels and shared-memory layouts by context length:
    the window select, and the bucket select on the rows it hands back; each
    reproduces the float64 order."""
    import torch

    n_q = 6
    d = make_dims(n_q, T - n_q, T, 32, 512, 64, 32, 128, 2048)
    x = workloads.generate(d, 31, "normal", "uniform")
    if kind == "repeated_keys":
        x["k_idx"] = np.ascontiguousarray(x["k_idx"][np.arange(T) % 40])
    xd = stage(x)
    ld = (T + 3) // 4 * 4
    sc = torch.empty(d.n_q, ld, dtype=torch.float32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_TOPK))
    dsa.check(dsa.dsa_index_scores(d, xd["q_idx"], xd["k_idx"], xd["w_idx"], sc, ld, ws))
    idx = torch.empty(d.n_q, d.top_k, dtype=torch.int32, device="cuda")
    dsa.check(dsa.dsa_topk_select(d, sc, ld, xd["q_idx"], xd["k_idx"], xd["w_idx"], idx, ws))
    torch.cuda.synchronize()
    # the workspace header counts the rows the window select handed back
    # (a 32-bit word at byte 24)
    handed_back = int(ws[24:28].cpu().numpy().view(np.uint32)[0])
    dsa.check(dsa.dsa_device_status(ws))
    ref = oracle_lib.topk_select(d, oracle_lib.index_scores(d, x["q_idx"], x["k_idx"], x["w_idx"]))
    assert np.array_equal(idx.cpu().numpy(), ref)
    if kind == "repeated_keys":
        assert handed_back > 0


@pytest.mark.parametrize("n_q,n_sub", [
    (203, 3),   # sub-chunks of 68, 68 and 67 rows
    (8, 8),     # rows per sub-chunk rounded up to 4: two sub-chunks
    (64, 1),    # one sub-chunk
])
def test_host_entry_matches_device_entry(dsa, n_q, n_sub):
    """dsa_prefill_layer_host (host buffers, copies overlapped with the layer
    over query sub-chunks) gives the bits of one dsa_prefill_layer call."""
    import torch

    d, x = _reduced("chunk2k_ctx8k", n_q)
    xd = stage(x)
    out_ref, lse_ref, idx_ref = run_layer(dsa, d, xd)
    pinned = {k: v.cpu().pin_memory() for k, v in xd.items()}
    dev_t = {k: torch.empty_like(v) for k, v in xd.items()}
    dev_t["out"] = empty_bf16(d.n_q, d.n_heads, d.d_latent)
    dev_t["lse"] = torch.empty(d.n_q, d.n_heads, dtype=torch.float32, device="cuda")
    dev_t["idx"] = torch.empty(d.n_q, d.top_k, dtype=torch.int32, device="cuda")
    out_h = torch.empty(d.n_q, d.n_heads, d.d_latent, dtype=torch.bfloat16).pin_memory()
    lse_h = torch.empty(d.n_q, d.n_heads, dtype=torch.float32).pin_memory()
    idx_h = torch.full((d.n_q, d.top_k), -7, dtype=torch.int32).pin_memory()
    streams = (torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream())
    events = (torch.cuda.Event(), torch.cuda.Event())
    for ev in events:
        ev.record()
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_LAYER))
    dsa.check(dsa.dsa_prefill_layer_host(d, pinned["q"], pinned["latent"], pinned["rope"],
                                         pinned["q_idx"], pinned["k_idx"], pinned["w_idx"], out_h,
                                         lse_h, idx_h, dev_t, ws, streams, events, n_sub))
    streams[2].synchronize()
    dsa.check(dsa.dsa_device_status(ws, stream=streams[1]))
    assert np.array_equal(host_bf16_as_f32(out_h), out_ref)
    assert np.array_equal(lse_h.numpy(), lse_ref)
    assert np.array_equal(idx_h.numpy(), idx_ref)


def test_host_entry_unordered_calls_alternating_buffers(dsa):
    """DSA_FLAG_HOST_UNORDERED: four back-to-back host calls on two chunks,
    alternating two sets of device tensors (each reused after an event at the
    end of the call that last used it), overlap one call's copy-in with the
    previous call's layers; every call's outputs keep the bits of
    dsa_prefill_layer on its own chunk."""
    import dataclasses

    import torch

    chunks = []
    for n_q, seed_shift in ((96, 0), (133, 1)):
        d, x = _reduced("chunk2k_ctx8k", n_q)
        if seed_shift:  # a second chunk with other inputs of another length
            x = workloads.generate(d, 977, "normal", "uniform")
        xd = stage(x)
        chunks.append((d, {k: v.cpu().pin_memory() for k, v in xd.items()}, run_layer(dsa, d, xd)))
    d_max = max((c[0] for c in chunks), key=lambda d_: d_.n_q)
    sets = []
    for _ in range(2):
        dev_t = {k: torch.empty(d_max.ctx_len if k in ("latent", "rope", "k_idx") else d_max.n_q,
                                *v.shape[1:], dtype=v.dtype, device="cuda")
                 for k, v in chunks[1][1].items()}
        dev_t["out"] = empty_bf16(d_max.n_q, d_max.n_heads, d_max.d_latent)
        sets.append(dev_t)
    streams = (torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream())
    events = (torch.cuda.Event(), torch.cuda.Event())
    free = [torch.cuda.Event(), torch.cuda.Event()]
    for ev in (*events, *free):
        ev.record()
    ws = workspace(dsa.dsa_workspace_size(d_max, dsa.DSA_WS_LAYER))
    outs = []
    for call in range(4):
        d, pinned, _ = chunks[call % 2]
        b = call % 2
        streams[0].wait_event(free[b])
        streams[1].wait_event(free[b])
        out_h = torch.empty(d.n_q, d.n_heads, d.d_latent, dtype=torch.bfloat16).pin_memory()
        dh = dataclasses.replace(d, flags=dsa.DSA_FLAG_HOST_UNORDERED)
        dsa.check(dsa.dsa_prefill_layer_host(dh, pinned["q"], pinned["latent"], pinned["rope"],
                                             pinned["q_idx"], pinned["k_idx"], pinned["w_idx"],
                                             out_h, None, None, sets[b], ws, streams, events, 8))
        free[b].record(streams[2])
        outs.append(out_h)
    torch.cuda.synchronize()
    dsa.check(dsa.dsa_device_status(ws, stream=streams[1]))
    for call, out_h in enumerate(outs):
        assert np.array_equal(host_bf16_as_f32(out_h), chunks[call % 2][2][0]), call
    # the flag belongs to the host call alone
    d0 = dataclasses.replace(chunks[0][0], flags=dsa.DSA_FLAG_HOST_UNORDERED)
    assert dsa.dsa_prefill_layer(d0, *[chunks[0][1][k].cuda() for k in
                                       ("q", "latent", "rope", "q_idx", "k_idx", "w_idx")],
                                 sets[0]["out"], None, None, ws) == dsa.DSA_ERR_DIMS


def test_sparse_attn_entry_point_on_given_sets(dsa, oracle_lib):
    """dsa_sparse_attn_prefill on oracle-chosen sets, with padding and shuffled order."""
    import torch

    d, x = _reduced("chunk2k_ctx8k", 50)
    _, _, ref_idx = oracle_lib.prefill_layer(d, **x)
    rng = np.random.default_rng(3)
    idx = np.stack([rng.permutation(r) for r in ref_idx]).astype(np.int32)
    idx[7, 100:] = -1                     # a row with a short list
    idx[8, :] = -1                        # a row with no key: out 0, lse -inf
    ref_out, ref_lse = oracle_lib.sparse_attn(d, x["q"], x["latent"], x["rope"], idx)
    xd = stage(x)
    out = empty_bf16(d.n_q, d.n_heads, d.d_latent)
    lse = torch.empty(d.n_q, d.n_heads, dtype=torch.float32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_ATTN))
    dsa.check(dsa.dsa_sparse_attn_prefill(d, xd["q"], xd["latent"], xd["rope"], dev(idx), out,
                                          lse, ws))
    dsa.check(dsa.dsa_device_status(ws))
    o = host_bf16_as_f32(out)
    assert_attn_close(o, ref_out)
    assert np.all(o[8] == 0) and np.all(np.isneginf(lse.cpu().numpy()[8]))


# ----------------------------------------------------------------- edge cases


def test_bounded_wait_gives_up_cleanly(dsa, oracle_lib):
    """The failure path the kernels share: a device wait that runs out records
    DSA_ERR_TIMEOUT with its site, the CTA's other waits leave through the
    abort flag instead of their own one-second limit, and the context stays
    usable (no fault, no hang)."""
    import time

    import torch

    ws = workspace(256)
    cycles = torch.zeros(2, dtype=torch.int64, device="cuda")
    torch.cuda.synchronize()
    t0 = time.time()
    dsa.check(dsa.dsa_selftest_bounded_wait(ws, cycles))
    torch.cuda.synchronize()
    assert time.time() - t0 < 1.0
    status, site = ws[:8].cpu().numpy().view(np.uint32)
    assert status == 1 and site == 101  # timeout, at the short-limit wait
    c = cycles.cpu().numpy()
    assert c[0] >= 1_000_000            # warp 0 waited out its limit
    assert 0 <= c[1] < 20_000_000       # warp 1 followed the abort, far below 2e9 cycles
    assert dsa.dsa_device_status(ws) == dsa.DSA_ERR_TIMEOUT
    assert dsa.dsa_device_status(ws) == dsa.DSA_OK  # read once, then cleared
    d, x = _reduced("tiny_256q", 64)
    out, lse, idx = run_layer(dsa, d, stage(x))
    _compare_layer(oracle_lib, d, x, out, lse, idx)


@pytest.mark.parametrize("name,n_rows", [("chunk8k_ctx17k", None), ("chunk4k_ctx128k", 1100)])
def test_l2_scores_schedule_is_bit_identical(dsa, name, n_rows):
    """DSA_FLAG_L2_SCORES (indexer and top-k over query sub-blocks whose
    scores stay in L2): selections, outputs and lse equal the default
    schedule's bit for bit, on the full 8K chunk (nine sub-blocks) and on rows
    of the 131,072-token context (two-pass top-k, 128-row sub-blocks)."""
    import dataclasses

    d, x = workloads.workload_inputs(name)
    if n_rows is not None:
        d = dataclasses.replace(d, n_q=n_rows, q_pos0=d.ctx_len - n_rows)
        x = workloads.generate(d, 5, "normal", "uniform")
    xd = stage(x)
    out0, lse0, idx0 = run_layer(dsa, d, xd)
    out1, lse1, idx1 = run_layer(dsa, dataclasses.replace(d, flags=dsa.DSA_FLAG_L2_SCORES), xd)
    assert np.array_equal(idx0, idx1)
    assert np.array_equal(out0, out1)
    assert np.array_equal(lse0, lse1)


def test_mma_layout_selftest_passes(dsa):
    """The start-up check of the tensor-core operand layouts: every accumulator
    element of the four forms (indexer bf16, attention QK^T and PV, FP8
    indexer) equals the exact integer product, and nothing is reported."""
    ws = workspace(512)
    st, counts, cycles = dsa.dsa_selftest_mma_layout(ws)
    dsa.check(st)
    assert counts == [0, 0, 0, 0]
    assert dsa.dsa_device_status(ws) == dsa.DSA_OK
    # the timed runs, for the record: an N = 256 MMA is bound by its math (128
    # cycles at 4,096 bf16 multiply-adds per clock; an e4m3 MMA does twice the
    # multiply-adds, K = 32, at twice the rate), an N = 32 MMA by its 5 KB of
    # shared-memory operands
    print(f"cycles per MMA: indexer bf16 N=256 {cycles[0]:.1f}, QK^T N=32 {cycles[1]:.1f}, "
          f"PV N=32 MN-major {cycles[2]:.1f}, FP8 N=256 {cycles[3]:.1f}")
    assert all(c > 0 for c in cycles)


def test_empty_chunk_launches_nothing(dsa):
    import torch

    d = make_dims(0, 10, 10, 32, 512, 64, 32, 128, 2048)
    one = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(16, dtype=torch.float32, device="cuda")
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_LAYER))
    assert dsa.dsa_prefill_layer(d, one, one, one, one, one, w, one, None, None, ws) == dsa.DSA_OK
    assert dsa.dsa_device_status(ws) == dsa.DSA_OK


@pytest.mark.parametrize("n_q,q_pos0,T,k", [
    (1, 0, 1, 2048),        # one query that sees only itself
    (3, 0, 3, 1),           # k = 1
    (70, 930, 1000, 500),   # ragged context, partial key tiles
    (33, 0, 33, 2048),      # every row keeps all causal keys, -1 padding
])
def test_layer_edge_shapes(dsa, oracle_lib, n_q, q_pos0, T, k):
    d = make_dims(n_q, q_pos0, T, 32, 512, 64, 32, 128, k)
    x = workloads.generate(d, 21, "normal", "uniform")
    out, lse, idx = run_layer(dsa, d, stage(x))
    _compare_layer(oracle_lib, d, x, out, lse, idx)


def test_layer_all_keys_tied(dsa, oracle_lib):
    """Identical indexer keys: every score of a row ties, so the band holds
    the whole row (larger than the kernel's band cache) and the lowest
    indices must win."""
    d = make_dims(6, 6000, 6006, 32, 512, 64, 32, 128, 2048)
    x = workloads.generate(d, 22, "normal", "uniform")
    x["k_idx"] = np.ascontiguousarray(np.broadcast_to(x["k_idx"][:1], x["k_idx"].shape))
    out, lse, idx = run_layer(dsa, d, stage(x))
    for i in range(d.n_q):
        assert idx[i].tolist() == list(range(d.top_k))
    _compare_layer(oracle_lib, d, x, out, lse, idx)


def test_layer_zero_weights(dsa, oracle_lib):
    d = make_dims(20, 980, 1000, 32, 512, 64, 32, 128, 300)
    x = workloads.generate(d, 23, "normal", "uniform")
    x["w_idx"] = np.zeros_like(x["w_idx"])
    out, lse, idx = run_layer(dsa, d, stage(x))
    assert np.all(idx == np.arange(d.top_k)[None, :])
    _compare_layer(oracle_lib, d, x, out, lse, idx)


def test_chunk_split_is_invariant(dsa):
    """Two half chunks give the same selections and bit-identical outputs."""
    d, x = _reduced("chunk2k_ctx8k", 128)
    out, lse, idx = run_layer(dsa, d, stage(x))
    h = d.n_q // 2
    for part in range(2):
        sl = slice(part * h, (part + 1) * h)
        dp = make_dims(h, d.q_pos0 + part * h, d.ctx_len, d.n_heads, d.d_latent, d.d_rope,
                       d.n_idx_heads, d.d_idx, d.top_k, d.softmax_scale)
        xp = dict(x)
        for key in ("q", "q_idx", "w_idx"):
            xp[key] = np.ascontiguousarray(x[key][sl])
        o, l, ix = run_layer(dsa, dp, stage(xp))
        assert np.array_equal(ix, idx[sl])
        assert np.array_equal(o, out[sl])
        assert np.array_equal(l, lse[sl])


@pytest.mark.parametrize("where", ["past_cache", "future_token"])
def test_out_of_range_index_is_reported(dsa, where):
    """An index past the cache, or past the query's own position t while still
    inside the cache (a future token of the chunk), is reported and skipped."""
    d, x = _reduced("chunk2k_ctx8k", 4)
    xd = stage(x)
    idx = np.tile(np.arange(d.top_k, dtype=np.int32), (d.n_q, 1))
    if where == "past_cache":
        idx[2, 5] = d.ctx_len + 7
    else:
        idx[0, 5] = d.q_pos0 + 1  # row 0 sits at t = q_pos0 < q_pos0 + 1 < ctx_len
    out = empty_bf16(d.n_q, d.n_heads, d.d_latent)
    ws = workspace(dsa.dsa_workspace_size(d, dsa.DSA_WS_ATTN))
    dsa.check(dsa.dsa_sparse_attn_prefill(d, xd["q"], xd["latent"], xd["rope"], dev(idx), out,
                                          None, ws))
    assert dsa.dsa_device_status(ws) == dsa.DSA_ERR_RANGE
    assert dsa.dsa_device_status(ws) == dsa.DSA_OK  # cleared by the read


def test_argument_errors_launch_nothing(dsa):
    import torch

    d, x = _reduced("chunk2k_ctx8k", 8)
    xd = stage(x)
    out = torch.full((d.n_q, d.n_heads, d.d_latent), 3.0, dtype=torch.bfloat16, device="cuda")
    nbytes = dsa.dsa_workspace_size(d, dsa.DSA_WS_LAYER)
    ws = workspace(nbytes)
    args = [xd["q"], xd["latent"], xd["rope"], xd["q_idx"], xd["k_idx"], xd["w_idx"], out, None,
            None, ws]
    assert dsa.dsa_prefill_layer(d, *args[:6], None, None, None, ws) == dsa.DSA_ERR_NULL
    bad = list(args); bad[0] = xd["q"].data_ptr() + 2
    assert dsa.dsa_prefill_layer(d, *bad) == dsa.DSA_ERR_ALIGN
    assert dsa.dsa_prefill_layer(d, *args, workspace_bytes=nbytes - 1) == dsa.DSA_ERR_WORKSPACE
    for field, val, code in (("top_k", 4096, dsa.DSA_ERR_DIMS), ("n_heads", 16, dsa.DSA_ERR_DIMS),
                             ("d_idx", 64, dsa.DSA_ERR_DIMS), ("flags", 4, dsa.DSA_ERR_DIMS),
                             ("n_q", d.n_q + 1, dsa.DSA_ERR_CAUSAL)):
        dd = dsa.make_dims(d)
        setattr(dd, field, val)
        assert dsa.dsa_prefill_layer(dd, *args) == code
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)  # nothing ran
