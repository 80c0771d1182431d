"""Pins for the float64 oracle, on the CPU only.

None of these checks re-types the oracle's own formulas. Each one ties the
oracle to something outside it:
  * a hand-worked 4-token case (tests/golden/hand_case_4tok.json);
  * library routines the definitions reduce to in a special case: torch's
    float64 scaled-dot-product attention when every causal key is kept
    (k >= t+1), torch float64 matmuls for the indexer, numpy lexsort for the
    selection order, exact integer matmuls when every score is an integer;
  * exact rational arithmetic on tiny inputs;
  * invariants (set sizes, causality, softmax normalisation, convex hull,
    permutation, duplicate rows, exact weight scaling, chunk splitting).
Each is chosen so that a plausible slip in the oracle fails at least one: a
dropped rope term or head, a wrong sign, s < t instead of s <= t, a transposed
operand, the wrong tie order.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import workloads
from workloads import bf16_bits_to_f32, make_dims, to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a):
    return to_bf16_bits(np.asarray(a, dtype=np.float32))


def _f64(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


def _small_inputs(n_q=24, q_pos0=8, T=32, H=3, Dc=16, Dr=8, HI=4, DI=8, k=7, seed=5,
                  kind="normal", w_mode="uniform"):
    d = make_dims(n_q, q_pos0, T, H, Dc, Dr, HI, DI, k)
    return d, workloads.generate(d, seed, kind, w_mode)


# ---------------------------------------------------------------- hand case


def _hand_case():
    with open(os.path.join(GOLDEN, "hand_case_4tok.json")) as f:
        g = json.load(f)
    dd = g["dims"]
    d = make_dims(dd["n_q"], dd["q_pos0"], dd["ctx_len"], dd["n_heads"], dd["d_latent"],
                  dd["d_rope"], dd["n_idx_heads"], dd["d_idx"], dd["top_k"], dd["softmax_scale"])
    x = dict(q=_bf16(g["q"]), latent=_bf16(g["latent"]), rope=_bf16(g["rope"]),
             q_idx=_bf16(g["q_idx"]), k_idx=_bf16(g["k_idx"]),
             w_idx=np.asarray(g["w_idx"], dtype=np.float32))
    return g, d, x


def _closed_form(expr):
    return eval(expr, {"__builtins__": {}}, {"e": math.e, "ln2": math.log(2.0), "log": math.log})


def test_hand_case_scores_and_selection(oracle_lib):
    g, d, x = _hand_case()
    sc = oracle_lib.index_scores(d, x["q_idx"], x["k_idx"], x["w_idx"])
    for i, row in enumerate(g["expected_scores"]):
        for s, v in enumerate(row):
            if v is None:
                assert sc[i, s] == -math.inf
            else:
                assert sc[i, s] == v
    idx = oracle_lib.topk_select(d, sc)
    assert idx.tolist() == g["expected_idx"]


def test_hand_case_attention(oracle_lib):
    g, d, x = _hand_case()
    out, lse, idx = oracle_lib.prefill_layer(d, **x)
    assert idx.tolist() == g["expected_idx"]
    for i in range(d.n_q):
        assert out[i, 0, 0] == pytest.approx(_closed_form(g["expected_out"][i]), abs=1e-14)
        assert lse[i, 0] == pytest.approx(_closed_form(g["expected_lse"][i]), abs=1e-14)


# ------------------------------------------------------------ indexer scores


def test_scores_match_torch_float64_matmul(oracle_lib):
    d, x = _small_inputs()
    sc = oracle_lib.index_scores(d, x["q_idx"], x["k_idx"], x["w_idx"])
    qi = torch.from_numpy(_f64(x["q_idx"]))           # [n_q, HI, DI]
    ki = torch.from_numpy(_f64(x["k_idx"]))           # [T, DI]
    w = torch.from_numpy(x["w_idx"].astype(np.float64))
    dots = torch.einsum("njc,sc->njs", qi, ki)
    ref = torch.einsum("nj,njs->ns", w, torch.relu(dots)).numpy()
    t = d.q_pos0 + np.arange(d.n_q)[:, None]
    s = np.arange(d.ctx_len)[None, :]
    causal = s <= t
    np.testing.assert_allclose(sc[causal], ref[causal], rtol=1e-13, atol=1e-13)
    assert np.all(np.isneginf(sc[~causal]))


def test_scores_exact_rational_tiny(oracle_lib):
    """Exact rational value vs the float64 result: within a few ulps of the
    exact score, so the float64 order matches the exact order here."""
    d, x = _small_inputs(n_q=5, q_pos0=3, T=8, HI=3, DI=6, seed=11)
    sc = oracle_lib.index_scores(d, x["q_idx"], x["k_idx"], x["w_idx"])
    qi, ki = _f64(x["q_idx"]), _f64(x["k_idx"])
    for i in range(d.n_q):
        t = d.q_pos0 + i
        exact = []
        for s in range(t + 1):
            tot = Fraction(0)
            for j in range(d.n_idx_heads):
                dot = sum(Fraction(float(qi[i, j, c])) * Fraction(float(ki[s, c]))
                          for c in range(d.d_idx))
                tot += Fraction(float(x["w_idx"][i, j])) * max(dot, Fraction(0))
            exact.append(tot)
            assert abs(Fraction(sc[i, s]) - tot) <= Fraction(abs(float(tot))) * Fraction(1, 2**48) + Fraction(1, 2**80)
        order_exact = sorted(range(t + 1), key=lambda s: (-exact[s], s))
        order_f64 = sorted(range(t + 1), key=lambda s: (-sc[i, s], s))
        assert order_exact == order_f64


def test_scores_integer_inputs_exact(oracle_lib):
    """Ternary indexer inputs and w = 1: every score is an integer, so the
    float64 result must equal an exact int64 matmul."""
    d, x = _small_inputs(n_q=16, q_pos0=16, T=32, HI=4, DI=16, kind="ternary_ties", w_mode="ones")
    sc = oracle_lib.index_scores(d, x["q_idx"], x["k_idx"], x["w_idx"])
    qi = _f64(x["q_idx"]).astype(np.int64)
    ki = _f64(x["k_idx"]).astype(np.int64)
    ref = np.maximum(np.einsum("njc,sc->njs", qi, ki), 0).sum(axis=1)
    for i in range(d.n_q):
        t = d.q_pos0 + i
        assert np.array_equal(sc[i, : t + 1], ref[i, : t + 1].astype(np.float64))


# ---------------------------------------------------------------- selection


def _lexsort_select(row, t, k):
    cand = np.arange(t + 1)
    order = np.lexsort((cand, -row[: t + 1]))  # last key primary: score desc, then index asc
    keep = np.sort(order[: min(k, t + 1)])
    out = -np.ones(k, dtype=np.int64)
    out[: keep.size] = keep
    return out


@pytest.mark.parametrize("k", [1, 5, 16, 40])
def test_selection_matches_lexsort_with_heavy_ties(oracle_lib, k):
    rng = np.random.default_rng(3)
    d = make_dims(30, 10, 40, 1, 8, 0, 1, 8, k)
    scores = rng.integers(0, 4, size=(d.n_q, d.ctx_len)).astype(np.float64)  # many ties
    idx = oracle_lib.topk_select(d, scores)
    for i in range(d.n_q):
        t = d.q_pos0 + i
        assert np.array_equal(idx[i], _lexsort_select(scores[i], t, k))


def test_selection_characterisation(oracle_lib):
    """Every kept key beats every dropped causal key under (score desc, index asc)."""
    rng = np.random.default_rng(4)
    d = make_dims(50, 0, 50, 1, 8, 0, 1, 8, 9)
    scores = np.round(rng.standard_normal((d.n_q, d.ctx_len)), 1)
    idx = oracle_lib.topk_select(d, scores)
    for i in range(d.n_q):
        t = i
        kept = [s for s in idx[i] if s >= 0]
        assert len(kept) == min(d.top_k, t + 1)
        assert kept == sorted(set(kept)) and all(0 <= s <= t for s in kept)
        assert all(s == -1 for s in idx[i][len(kept):])
        dropped = set(range(t + 1)) - set(kept)
        for a in kept:
            for b in dropped:
                assert (scores[i, a], -a) > (scores[i, b], -b)


def test_selection_f32_equals_widened_f64(oracle_lib):
    rng = np.random.default_rng(6)
    d = make_dims(20, 30, 50, 1, 8, 0, 1, 8, 12)
    s32 = rng.integers(0, 6, size=(d.n_q, 52)).astype(np.float32) * np.float32(0.25)
    assert np.array_equal(oracle_lib.topk_select(d, s32),
                          oracle_lib.topk_select(d, s32.astype(np.float64)))


# ---------------------------------------------------------------- attention


def _sdpa_reference(d, x):
    """Full causal softmax attention through torch's float64 SDPA (value = latent)."""
    q = torch.from_numpy(_f64(x["q"])).permute(1, 0, 2).unsqueeze(0)          # [1,H,n_q,Dc+Dr]
    kv = np.concatenate([_f64(x["latent"]), _f64(x["rope"])], axis=1)
    k = torch.from_numpy(kv)[None, None].expand(1, d.n_heads, -1, -1)        # [1,H,T,Dc+Dr]
    v = torch.from_numpy(_f64(x["latent"]))[None, None].expand(1, d.n_heads, -1, -1)
    t = d.q_pos0 + torch.arange(d.n_q)[:, None]
    mask = torch.arange(d.ctx_len)[None, :] <= t                              # [n_q, T]
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                           scale=d.softmax_scale)
    logits = torch.einsum("bhqc,bhsc->bhqs", q, k) * d.softmax_scale
    lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1)
    return out[0].permute(1, 0, 2).numpy(), lse[0].permute(1, 0).numpy()


@pytest.mark.parametrize("q_pos0,k", [(0, 64), (16, 48), (5, 200)])
def test_attention_equals_full_causal_sdpa_when_k_covers_context(oracle_lib, q_pos0, k):
    d, x = _small_inputs(n_q=32, q_pos0=q_pos0, T=q_pos0 + 32, H=3, Dc=16, Dr=8, k=k, seed=7)
    out, lse, idx = oracle_lib.prefill_layer(d, **x)
    ref_out, ref_lse = _sdpa_reference(d, x)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)
    for i in range(d.n_q):  # every causal key kept
        t = q_pos0 + i
        assert idx[i][: t + 1].tolist() == list(range(t + 1))


def test_tiny_workload_rows_below_k_take_full_causal_attention(oracle_lib):
    """The tiny 256-query workload keeps k=64 keys: rows t < 64 keep every causal key."""
    d, x = workloads.workload_inputs("tiny_256q")
    rows = np.arange(64)
    out, lse, idx = oracle_lib.prefill_layer(d, **x, rows=rows)
    d64 = make_dims(64, 0, 64, d.n_heads, d.d_latent, d.d_rope, d.n_idx_heads, d.d_idx, 64,
                    d.softmax_scale)
    x64 = dict(q=x["q"][:64], latent=x["latent"][:64], rope=x["rope"][:64])
    ref_out, ref_lse = _sdpa_reference(d64, x64)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_attention_softmax_normalised_and_convex(oracle_lib):
    d, x = _small_inputs(seed=9)
    out, lse, idx = oracle_lib.prefill_layer(d, **x)
    lat = _f64(x["latent"])
    for i in range(d.n_q):
        sel = idx[i][idx[i] >= 0]
        lo, hi = lat[sel].min(axis=0), lat[sel].max(axis=0)
        assert np.all(out[i] >= lo - 1e-12) and np.all(out[i] <= hi + 1e-12)
    # constant latent rows -> output is that constant (softmax weights sum to 1)
    x2 = dict(x)
    x2["latent"] = np.broadcast_to(_bf16(np.full(d.d_latent, 1.5)), x["latent"].shape).copy()
    out2, _, _ = oracle_lib.prefill_layer(d, **x2)
    np.testing.assert_allclose(out2, 1.5, rtol=0, atol=1e-13)


def test_attention_permutation_and_duplicate_rows(oracle_lib):
    d, x = _small_inputs(seed=12)
    _, _, idx = oracle_lib.prefill_layer(d, **x)
    out, lse = oracle_lib.sparse_attn(d, x["q"], x["latent"], x["rope"], idx)
    rng = np.random.default_rng(0)
    perm_idx = np.stack([rng.permutation(r) for r in idx])
    out_p, lse_p = oracle_lib.sparse_attn(d, x["q"], x["latent"], x["rope"], perm_idx)
    np.testing.assert_allclose(out_p, out, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse_p, lse, rtol=0, atol=1e-13)
    # two identical cache rows count twice: a list holding row a twice equals a
    # list holding a and an exact copy of a
    x3 = {k: v.copy() for k, v in x.items()}
    a, b = 2, 3
    x3["latent"][b] = x3["latent"][a]
    x3["rope"][b] = x3["rope"][a]
    k = d.top_k
    twice = np.full((d.n_q, k), -1, np.int32); twice[:, 0] = a; twice[:, 1] = a
    pair = np.full((d.n_q, k), -1, np.int32); pair[:, 0] = a; pair[:, 1] = b
    o1, l1 = oracle_lib.sparse_attn(d, x3["q"], x3["latent"], x3["rope"], twice)
    o2, l2 = oracle_lib.sparse_attn(d, x3["q"], x3["latent"], x3["rope"], pair)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    np.testing.assert_allclose(o1, np.broadcast_to(_f64(x3["latent"][a]), o1.shape), atol=1e-13)


# --------------------------------------------------------------- invariants


def test_layer_invariants_tiny_workload(oracle_lib):
    d, x = workloads.workload_inputs("tiny_256q")
    out, lse, idx = oracle_lib.prefill_layer(d, **x)
    for i in range(d.n_q):
        t = d.q_pos0 + i
        kept = idx[i][idx[i] >= 0]
        assert kept.size == min(d.top_k, t + 1)
        assert np.all(np.diff(kept) > 0) and kept.min() >= 0 and kept.max() <= t
        assert np.all(idx[i][kept.size:] == -1)
    # scaling w by 2 is exact in float32 and float64: the selection cannot move
    x2 = dict(x); x2["w_idx"] = x["w_idx"] * np.float32(2)
    _, _, idx2 = oracle_lib.prefill_layer(d, **x2)
    assert np.array_equal(idx, idx2)


def test_chunk_split_equals_whole(oracle_lib):
    """Two half chunks (q_pos0 and q_pos0 + n_q/2) reproduce the whole chunk."""
    d, x = _small_inputs(n_q=20, q_pos0=12, T=32, k=9, seed=13)
    out, lse, idx = oracle_lib.prefill_layer(d, **x)
    h = d.n_q // 2
    for part, sl in ((0, slice(0, h)), (1, slice(h, d.n_q))):
        dp = make_dims(h, d.q_pos0 + part * h, d.ctx_len, d.n_heads, d.d_latent, d.d_rope,
                       d.n_idx_heads, d.d_idx, d.top_k, d.softmax_scale)
        xp = dict(x)
        for key in ("q", "q_idx", "w_idx"):
            xp[key] = np.ascontiguousarray(x[key][sl])
        o, l, ix = oracle_lib.prefill_layer(dp, **xp)
        assert np.array_equal(ix, idx[sl])
        np.testing.assert_array_equal(o, out[sl])
        np.testing.assert_array_equal(l, lse[sl])


def test_rows_subset_equals_full(oracle_lib):
    d, x = _small_inputs(seed=14)
    out, lse, idx = oracle_lib.prefill_layer(d, **x)
    rows = np.array([0, 5, 23, 7], dtype=np.int32)
    o, l, ix = oracle_lib.prefill_layer(d, **x, rows=rows)
    np.testing.assert_array_equal(o, out[rows])
    np.testing.assert_array_equal(ix, idx[rows])
    sc = oracle_lib.index_scores(d, x["q_idx"], x["k_idx"], x["w_idx"], rows=rows)
    np.testing.assert_array_equal(oracle_lib.topk_select(d, sc, rows=rows), idx[rows])


def test_tie_stress_workload_selection_is_lexsort(oracle_lib):
    """Tie-stress recipe at a reduced size: integer scores, heavy ties."""
    d = make_dims(64, 448, 512, 2, 16, 8, 32, 128, 128)
    x = workloads.generate(d, 4, "ternary_ties", "ones")
    sc = oracle_lib.index_scores(d, x["q_idx"], x["k_idx"], x["w_idx"])
    idx = oracle_lib.topk_select(d, sc)
    n_tied = 0
    for i in range(d.n_q):
        t = d.q_pos0 + i
        assert np.array_equal(idx[i], _lexsort_select(sc[i], t, d.top_k))
        kth = np.sort(sc[i, : t + 1])[::-1][d.top_k - 1]
        n_tied += int((sc[i, : t + 1] == kth).sum())
    assert n_tied > 4 * d.n_q  # the recipe really produces ties at the boundary


# ------------------------------------------------ stored selection digests


def test_stored_selection_digests_match_the_oracle():
    """tests/golden/selection_hashes.json was written by an oracle-only
    script; recompute the tiny workload whole and a few 256-row blocks of the
    others here, so the stored digests stay tied to the oracle as it is."""
    import importlib.util

    here = os.path.join(os.path.dirname(__file__), "golden")
    spec = importlib.util.spec_from_file_location(
        "make_selection_hashes", os.path.join(here, "make_selection_hashes.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    with open(os.path.join(here, "selection_hashes.json")) as f:
        g = json.load(f)
    nb = g["block_rows"]
    assert set(g["cases"]) == {mod.case_key(*c) for c in mod.CASES}
    for key, c in sorted(g["cases"].items()):
        fp8 = c.get("variant", "") == "fp8"
        d, x = workloads.workload_inputs(c["workload"], c["w_mode"])
        assert mod.inputs_digest(x) == c["inputs_sha256"], key
        n_blocks = (d.n_q + nb - 1) // nb
        assert len(c["block_sha256"]) == n_blocks
        if d.n_q <= nb:
            whole, _ = mod.selection_digests(mod.oracle_selection(d, x, fp8=fp8))
            assert whole == c["selection_sha256"], key
            continue
        # first block always; the last one too where the oracle is quick
        blocks = [0] if d.ctx_len > 20000 else [0, n_blocks - 1]
        for b in blocks:
            rows = np.arange(b * nb, min(d.n_q, (b + 1) * nb), dtype=np.int32)
            if d.ctx_len > 20000:
                rows = rows[:nb]
            sel = mod.oracle_selection(d, x, rows=rows, fp8=fp8)
            _, digests = mod.selection_digests(sel)
            assert digests[0] == c["block_sha256"][b], (key, b)


# ------------------------------------------------ FP8 form of the indexer inputs


def test_fp8_hand_case(oracle_lib):
    with open(os.path.join(GOLDEN, "fp8_hand_case.json")) as f:
        g = json.load(f)
    x = _bf16([g["x"]])
    x8, scale, xhat = oracle_lib.quantize_fp8(x)
    assert float(scale[0]) == g["expected_scale"]
    assert x8[0].tolist() == g["expected_codes"]
    assert bf16_bits_to_f32(xhat)[0].tolist() == g["expected_xhat"]


def test_fp8_codes_match_torch_e4m3_conversion(oracle_lib):
    """e4m3 codes against torch's float8_e4m3fn conversion of x / scale (round
    to nearest even), on normal draws, small values (subnormal codes), zeros of
    both signs and an all-zero row; the scale is the smallest power of two that
    covers the row's maximum."""
    rng = np.random.default_rng(12)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    x[3] *= 1e-3
    x[4, :64] *= 1e-4                # subnormal e4m3 codes after scaling
    x[5] = 0.0
    x[6, ::3] = -0.0
    x[7] = np.round(x[7] * 8) / 8    # many ties
    xb = _bf16(x)
    x8, scale, xhat = oracle_lib.quantize_fp8(xb)
    xf = bf16_bits_to_f32(xb).astype(np.float64)
    amax = np.abs(xf).max(axis=1)
    s = scale.astype(np.float64)
    assert np.all(np.log2(s) == np.round(np.log2(s)))          # powers of two
    nz = amax > 0
    assert np.all(amax[nz] <= 448 * s[nz]) and np.all(amax[nz] > 224 * s[nz])
    assert np.all(s[~nz] == 1.0)
    ref = torch.from_numpy((xf / s[:, None]).astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(x8, ref.view(torch.uint8).numpy())
    deq = ref.to(torch.float64).numpy() * s[:, None]
    assert np.array_equal(bf16_bits_to_f32(xhat).astype(np.float64), deq)


def test_fp8_contract_scores_match_torch_on_dequantized_inputs(oracle_lib):
    d, x = _small_inputs(seed=13)
    sc = oracle_lib.index_scores_fp8(d, x["q_idx"], x["k_idx"], x["w_idx"])
    _, _, qh = oracle_lib.quantize_fp8(x["q_idx"])
    _, _, kh = oracle_lib.quantize_fp8(x["k_idx"])
    qi, ki = torch.from_numpy(_f64(qh)), torch.from_numpy(_f64(kh))
    w = torch.from_numpy(x["w_idx"].astype(np.float64))
    ref = torch.einsum("nj,njs->ns", w, torch.relu(torch.einsum("njc,sc->njs", qi, ki))).numpy()
    t = d.q_pos0 + np.arange(d.n_q)[:, None]
    causal = np.arange(d.ctx_len)[None, :] <= t
    np.testing.assert_allclose(sc[causal], ref[causal], rtol=1e-13, atol=1e-13)
    # the 8-bit form moves scores, but not far: within a few percent of the bf16 scores
    sb = oracle_lib.index_scores(d, x["q_idx"], x["k_idx"], x["w_idx"])
    assert np.abs(sc[causal] - sb[causal]).max() <= 0.1 * np.abs(sb[causal]).max()
