"""The checking build (libdsa_check.so: every dynamically indexed buffer access
bounds-checked, a bad index reported in the workspace status instead of being
made) runs the tiny workload and a reduced chunk of the tie stress with a
clean status and the same results as the oracle. It stands in for a memory
checker, and runs in a child process because the library variant is chosen
when the binding loads."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_CHILD = r"""
import json, sys
import numpy as np
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import torch
import sparse_attention_prefill_dsa_b200 as dsa
import oracle, workloads
from workloads import make_dims
from dsa_test_util import stage, run_layer, attn_errors
assert dsa.LIB_PATH.endswith("libdsa_check.so"), dsa.LIB_PATH
dsa.library()
res = []
cases = [workloads.workload_inputs("tiny_256q")]
d0 = workloads.BY_NAME["ties_4k_ctx8k"].dims
d = make_dims(149, d0.ctx_len - 149, d0.ctx_len, d0.n_heads, d0.d_latent, d0.d_rope,
              d0.n_idx_heads, d0.d_idx, d0.top_k, d0.softmax_scale)
cases.append((d, workloads.generate(d, 104, "ternary_ties", "ones")))
for d, x in cases:
    out, lse, idx = run_layer(dsa, d, stage(x))   # raises on a nonzero device status
    ref_out, ref_lse, ref_idx = oracle.prefill_layer(d, **x)
    res.append(dict(idx_equal=bool(np.array_equal(idx, ref_idx)),
                    err=attn_errors(out, ref_out)))
print(json.dumps(res))
"""


def test_checking_build_is_clean_on_tiny_and_tie_workloads():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_prefill_dsa_b200 import build

    build.build(variant="check")
    env = dict(os.environ, DSA_LIBRARY="check")
    code = _CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    for case in res:
        assert case["idx_equal"]
        max_abs, rel = case["err"]
        assert max_abs <= 2e-2 and rel <= 5e-3
