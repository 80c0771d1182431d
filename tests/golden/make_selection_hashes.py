"""Writes tests/golden/selection_hashes.json: SHA-256 digests of the float64
oracle's full top-k selection on every named workload.

The selections themselves are too large to store (up to 16,384 x 2,048 int32
per workload), so the file keeps, per workload and weight mode:
  * the digest of the whole [n_q, top_k] int32 selection (little-endian,
    row-major, -1 padded, ascending per row, as the oracle returns it);
  * one digest per block of BLOCK_ROWS consecutive query rows, so a mismatch
    can be narrowed to a block and the oracle re-run on that block alone;
  * the digest of the generated inputs, so a change to the input recipe shows
    up as a stale file instead of as a selection mismatch;
  * the digest of the oracle's source, for the record.

Only oracle/ and workloads/ are used: no value here comes from the CUDA path.
The selection rule follows the feedman.me post feedman.me/posts/wy2HU
("per-query top-2048", paragraph after the component table) with the tie
policy score descending, then key index ascending.

    python tests/golden/make_selection_hashes.py [--only NAME[:MODE]] [--threads N]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads  # noqa: E402

OUT = os.path.join(HERE, "selection_hashes.json")
BLOCK_ROWS = 256
# every named workload in its primary weight mode, plus the tie stress with
# non-integral weights
CASES = [(w.name, "ones" if w.kind == "ternary_ties" else "uniform") for w in workloads.WORKLOADS]
CASES.append(("ties_4k_ctx8k", "uniform"))
# the FP8 indexer variant's contract (the float64 scores of the dequantized
# e4m3 rows) on the 2K- and 8K-query chunks and the tie stress
CASES += [("chunk2k_ctx8k", "uniform", "fp8"), ("chunk8k_ctx17k", "uniform", "fp8"),
          ("ties_4k_ctx8k", "ones", "fp8")]


def inputs_digest(x: dict) -> str:
    h = hashlib.sha256()
    for key in ("q", "latent", "rope", "q_idx", "k_idx", "w_idx"):
        a = np.ascontiguousarray(x[key])
        h.update(key.encode())
        h.update(str(a.dtype).encode())
        h.update(str(a.shape).encode())
        h.update(a.tobytes())
    return h.hexdigest()


def selection_digests(idx: np.ndarray) -> tuple[str, list[str]]:
    idx = np.ascontiguousarray(idx, dtype="<i4")
    whole = hashlib.sha256(idx.tobytes()).hexdigest()
    blocks = [hashlib.sha256(idx[r:r + BLOCK_ROWS].tobytes()).hexdigest()
              for r in range(0, idx.shape[0], BLOCK_ROWS)]
    return whole, blocks


def oracle_selection(d, x, rows=None, threads=None, batch=None, fp8=False) -> np.ndarray:
    """The oracle's selection of the given rows (all rows by default), scored
    and selected in batches of rows to bound the float64 score memory; with
    fp8, under the FP8 indexer's contract (scores of the dequantized rows)."""
    if fp8:
        _, _, q_hat = oracle.quantize_fp8(x["q_idx"])
        _, _, k_hat = oracle.quantize_fp8(x["k_idx"])
        x = dict(x, q_idx=q_hat, k_idx=k_hat)
    if rows is None:
        rows = np.arange(d.n_q, dtype=np.int32)
    rows = np.asarray(rows, dtype=np.int32)
    if batch is None:
        batch = max(1, min(512, (1 << 28) // (8 * d.ctx_len)))
    out = np.empty((rows.size, d.top_k), dtype=np.int32)
    for b in range(0, rows.size, batch):
        r = rows[b:b + batch]
        sc = oracle.index_scores(d, x["q_idx"], x["k_idx"], x["w_idx"], rows=r, n_threads=threads)
        out[b:b + r.size] = oracle.topk_select(d, sc, rows=r, n_threads=threads)
    return out


def oracle_source_digest() -> str:
    with open(os.path.join(ROOT, "oracle", "dsa_oracle.cpp"), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def case_key(name: str, w_mode: str, variant: str = "") -> str:
    return f"{name}:{w_mode}" + (f":{variant}" if variant else "")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--only", action="append", default=[],
                    help="NAME:MODE[:VARIANT] to (re)compute; default: every case")
    ap.add_argument("--threads", type=int, default=0)
    args = ap.parse_args()
    oracle.build()
    data = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            data = json.load(f)
    data["about"] = ("SHA-256 digests of the float64 oracle's full top-k selection per workload "
                     "(int32 little-endian, [n_q, top_k], ascending rows, -1 padded), whole and per "
                     f"block of {BLOCK_ROWS} rows. Written by tests/golden/make_selection_hashes.py "
                     "from oracle/ and workloads/ only. Selection rule: feedman.me/posts/wy2HU, "
                     "'per-query top-2048' (paragraph after the component table); ties go to the "
                     "lower key index.")
    data["block_rows"] = BLOCK_ROWS
    data["oracle_source_sha256"] = oracle_source_digest()
    cases = data.setdefault("cases", {})
    todo = [c for c in CASES if not args.only or case_key(*c) in args.only]
    for case in todo:
        name, w_mode = case[0], case[1]
        variant = case[2] if len(case) > 2 else ""
        wl = workloads.BY_NAME[name]
        d, x = workloads.workload_inputs(name, w_mode)
        t0 = time.time()
        idx = oracle_selection(d, x, threads=args.threads or None, fp8=variant == "fp8")
        whole, blocks = selection_digests(idx)
        cases[case_key(*case)] = {
            "workload": name, "w_mode": w_mode, "variant": variant, "seed": wl.seed, "n_q": d.n_q,
            "ctx_len": d.ctx_len, "top_k": d.top_k, "inputs_sha256": inputs_digest(x),
            "selection_sha256": whole, "block_sha256": blocks,
        }
        print(f"{case_key(*case)}: {time.time() - t0:.0f} s", flush=True)
        with open(OUT + ".tmp", "w") as f:
            json.dump(data, f, indent=1, sort_keys=True)
            f.write("\n")
        os.replace(OUT + ".tmp", OUT)


if __name__ == "__main__":
    main()
