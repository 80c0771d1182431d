"""The C ABI on the CPU: the library loads, exports every function include/dsa.h
declares, sizes workspaces, and rejects bad arguments before touching a device.
No test here launches a kernel."""
import ctypes
import os
import re

import pytest

import workloads
from workloads import make_dims

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


@pytest.fixture(scope="module")
def dsa():
    from sparse_attention_prefill_dsa_b200 import build

    build.build()
    import sparse_attention_prefill_dsa_b200 as m

    m.library()
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("dsa_index_scores", "dsa_topk_select", "dsa_sparse_attn_prefill",
              "dsa_prefill_layer", "dsa_workspace_size", "dsa_status_string",
              "dsa_device_status"):
        assert n in names


def test_header_is_plain_c99(tmp_path):
    """The boundary is a C ABI: include/dsa.h compiles as strict C99."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_dsa.c"
    src.write_text('#include "dsa.h"\nint main(void) { dsa_dims d = {0}; (void)d; return 0; }\n')
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                        "-I", os.path.dirname(HEADER), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_library_exports_every_declared_symbol(dsa):
    lib = ctypes.CDLL(dsa.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in dsa.EXPORTED or name.startswith("dsa_"), name


def test_binding_has_a_function_per_symbol(dsa):
    for name in declared_functions():
        assert callable(getattr(dsa, name)), name


def test_dims_struct_layout_matches_header(dsa):
    assert ctypes.sizeof(dsa.dsa_dims) == 11 * 4
    text = open(HEADER).read()
    body = text[text.index("typedef struct dsa_dims"):text.index("} dsa_dims;")]
    fields = re.findall(r"\b(?:int32_t|uint32_t|float)\s+([a-z_0-9]+);", body)
    assert fields == [f for f, _ in dsa.dsa_dims._fields_]


def test_status_codes_and_strings(dsa):
    text = open(HEADER).read()
    for name, val in re.findall(r"#define (DSA_(?:OK|ERR_[A-Z_]+))\s+\(?(-?\d+)\)?", text):
        assert getattr(dsa, name) == int(val), name
        assert dsa.dsa_status_string(int(val))
    assert dsa.dsa_status_string(12345) == "unknown status"


def test_workspace_sizes(dsa):
    d = workloads.BY_NAME["chunk8k_ctx17k"].dims
    assert dsa.dsa_workspace_size(d, dsa.DSA_WS_TOPK) == 256
    ld = (d.ctx_len + 127) // 128 * 128
    assert dsa.dsa_workspace_size(d, dsa.DSA_WS_LAYER) == 256 + d.n_q * ld * 4 + d.n_q * d.top_k * 4
    assert dsa.dsa_workspace_size(d, 99) == 0
    # decode: the split attention's partials (n_split ranges of H x (Dc + 2) floats per query)
    d1 = workloads.make_dims(1, 49151, 49152, 32, 512, 64, 32, 128, 2048)
    part = 16 * 32 * 512 * 4 + (16 * 32 * 8 + 255) // 256 * 256  # 148 SMs: n_split = 16
    assert dsa.dsa_workspace_size(d1, dsa.DSA_WS_DECODE_ATTN) == 256 + part
    ld1 = 49152
    layer1 = 256 + ld1 * 4 + (2048 * 4 + 255) // 256 * 256
    assert dsa.dsa_workspace_size(d1, dsa.DSA_WS_DECODE_LAYER) == layer1 + part
    # rows past 49,152 keys: a top-k candidate buffer of ceil(R / 32768) segments
    for n_q, q_pos0, T, n_seg in ((1, 49151, 49152, 0), (1, 49152, 49153, 2),
                                  (1024, 130048, 131072, 4), (64, 65504, 70000, 3)):
        dl = workloads.make_dims(n_q, q_pos0, T, 32, 512, 64, 32, 128, 2048)
        cand = n_q * n_seg * 2048 * 4
        assert dsa.dsa_workspace_size(dl, dsa.DSA_WS_TOPK) == 256 + cand
        ldl = (T + 127) // 128 * 128
        assert dsa.dsa_workspace_size(dl, dsa.DSA_WS_LAYER) == \
            256 + n_q * ldl * 4 + n_q * 2048 * 4 + cand


def test_l2_scores_workspace_and_flag_rules(dsa):
    import dataclasses

    d = workloads.BY_NAME["chunk8k_ctx17k"].dims
    ld = (d.ctx_len + 127) // 128 * 128
    rows = (64 << 20) // (ld * 4) // 64 * 64  # 960 rows of 17,408 keys
    assert rows == 960
    dl2 = dataclasses.replace(d, flags=dsa.DSA_FLAG_L2_SCORES)
    assert dsa.dsa_workspace_size(dl2, dsa.DSA_WS_LAYER) == 256 + rows * ld * 4 + d.n_q * d.top_k * 4
    small = workloads.make_dims(40, 100, 140, 32, 512, 64, 32, 128, 64)  # fewer rows than a sub-block
    sl2 = dataclasses.replace(small, flags=dsa.DSA_FLAG_L2_SCORES)
    assert dsa.dsa_workspace_size(sl2, dsa.DSA_WS_LAYER) == dsa.dsa_workspace_size(small, dsa.DSA_WS_LAYER)
    # not with the FP8 indexer; the calls other than dsa_prefill_layer reject it
    both = dataclasses.replace(d, flags=dsa.DSA_FLAG_L2_SCORES | dsa.DSA_FLAG_FP8_INDEXER)
    assert _layer(dsa, both) == dsa.DSA_ERR_DIMS
    assert dsa.dsa_topk_select(dl2, FAKE, ld, None, None, None, FAKE, FAKE, 1 << 30, 0) == dsa.DSA_ERR_DIMS
    assert dsa.dsa_decode_layer(dl2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE,
                                1 << 40, stream=0) == dsa.DSA_ERR_DIMS


FAKE = 1 << 20  # an aligned, never dereferenced address


def _layer(dsa, d, **over):
    a = dict(q=FAKE, latent=FAKE, rope=FAKE, q_idx=FAKE, k_idx=FAKE, w_idx=FAKE, out=FAKE,
             lse=None, idx_out=None, workspace=FAKE)
    a.update(over)
    nbytes = over.pop("workspace_bytes", dsa.dsa_workspace_size(d, dsa.DSA_WS_LAYER))
    return dsa.dsa_prefill_layer(d, a["q"], a["latent"], a["rope"], a["q_idx"], a["k_idx"],
                                 a["w_idx"], a["out"], a["lse"], a["idx_out"], a["workspace"],
                                 workspace_bytes=nbytes, stream=0)


def test_host_validation_before_any_device_call(dsa):
    d = workloads.BY_NAME["chunk2k_ctx8k"].dims
    assert _layer(dsa, d, q=None) == dsa.DSA_ERR_NULL
    assert _layer(dsa, d, latent=FAKE + 8) == dsa.DSA_ERR_ALIGN
    assert _layer(dsa, d, workspace=None) == dsa.DSA_ERR_WORKSPACE
    assert _layer(dsa, d, workspace_bytes=100) == dsa.DSA_ERR_WORKSPACE
    bad = dsa.make_dims(d)
    bad.n_q = d.n_q + 1
    assert _layer(dsa, bad) == dsa.DSA_ERR_CAUSAL
    for field, val in (("top_k", 0), ("top_k", 2049), ("ctx_len", 131073), ("n_heads", 8),
                       ("d_latent", 256), ("n_idx_heads", 64), ("flags", 4), ("n_q", -1),
                       ("softmax_scale", 0.0)):
        bad = dsa.make_dims(d)
        setattr(bad, field, val)
        assert _layer(dsa, bad) in (dsa.DSA_ERR_DIMS, dsa.DSA_ERR_CAUSAL), field
    # top-k: indexer inputs all or none
    ws = dsa.dsa_workspace_size(d, dsa.DSA_WS_TOPK)
    assert dsa.dsa_topk_select(d, FAKE, d.ctx_len, FAKE, None, None, FAKE, FAKE, ws, 0) == \
        dsa.DSA_ERR_NULL
    assert dsa.dsa_topk_select(d, FAKE, d.ctx_len + 2, None, None, None, FAKE, FAKE, ws, 0) == \
        dsa.DSA_ERR_ALIGN
    assert dsa.dsa_index_scores(d, FAKE, FAKE, FAKE, FAKE, d.ctx_len - 4, FAKE, ws, 0) == \
        dsa.DSA_ERR_DIMS


def test_layout_selftest_validates_its_workspace_first(dsa):
    FAKE = 1 << 20
    st, counts, cycles = dsa.dsa_selftest_mma_layout(None, 0, 0)
    assert st == dsa.DSA_ERR_WORKSPACE
    assert dsa.dsa_selftest_mma_layout(FAKE, 287, 0)[0] == dsa.DSA_ERR_WORKSPACE  # header + 32
    assert dsa.dsa_selftest_mma_layout(FAKE + 8, 4096, 0)[0] == dsa.DSA_ERR_ALIGN


def test_valid_call_without_gpu_reports_device_error(dsa):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    d = make_dims(4, 0, 4, 4, 64, 16, 2, 32, 2)
    st = _layer(dsa, d)
    assert st in (dsa.DSA_ERR_CUDA, dsa.DSA_ERR_DEVICE)


def test_device_tensors_struct_matches_header(dsa):
    text = open(HEADER).read()
    body = text[text.index("typedef struct {\n  uint16_t* q;"):text.index("} dsa_device_tensors;")]
    fields = re.findall(r"\*\s*([a-z_0-9]+);", body)
    assert fields == [f for f, _ in dsa.dsa_device_tensors._fields_]
    assert ctypes.sizeof(dsa.dsa_device_tensors) == 9 * ctypes.sizeof(ctypes.c_void_p)


def _host(dsa, d, dev_over=None, events=(FAKE, FAKE), n_sub=4, **over):
    a = dict(q=FAKE, latent=FAKE, rope=FAKE, q_idx=FAKE, k_idx=FAKE, w_idx=FAKE, out=FAKE,
             lse=None, idx_out=None, workspace=FAKE)
    a.update(over)
    dev = {name: FAKE for name in ("q", "latent", "rope", "q_idx", "k_idx", "w_idx", "out")}
    dev.update(dev_over or {})
    return dsa.dsa_prefill_layer_host(d, a["q"], a["latent"], a["rope"], a["q_idx"], a["k_idx"],
                                      a["w_idx"], a["out"], a["lse"], a["idx_out"], dev,
                                      a["workspace"], (0, 0, 0), events, n_sub,
                                      workspace_bytes=dsa.dsa_workspace_size(d, dsa.DSA_WS_LAYER))


def test_host_entry_validation_before_any_device_call(dsa):
    d = workloads.BY_NAME["chunk2k_ctx8k"].dims
    assert _host(dsa, d, q=None) == dsa.DSA_ERR_NULL
    assert _host(dsa, d, dev_over={"out": None}) == dsa.DSA_ERR_NULL
    assert _host(dsa, d, lse=FAKE) == dsa.DSA_ERR_NULL          # host lse without a device lse
    assert _host(dsa, d, events=(FAKE, 0)) == dsa.DSA_ERR_NULL
    assert _host(dsa, d, dev_over={"q": FAKE + 8}) == dsa.DSA_ERR_ALIGN
    assert _host(dsa, d, n_sub=0) == dsa.DSA_ERR_DIMS
    assert _host(dsa, d, workspace=None) == dsa.DSA_ERR_WORKSPACE
