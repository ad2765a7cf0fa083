"""The C ABI on the host: the library builds for sm_100a, loads, exports every
entry point declared in include/sml.h, and rejects bad arguments before any
CUDA call (so these run without a GPU)."""
import ctypes

import pytest
import torch

from sparse_mla_attention_indexer_b200 import build as sml_build
from sparse_mla_attention_indexer_b200 import sml


@pytest.fixture(scope="module")
def L():
    sml_build.build()
    return sml.lib()


def test_every_declared_entry_point_is_exported(L):
    names = sml.declared_entry_points()
    assert {"sml_indexer_scores", "sml_topk", "sml_sparse_mla_decode", "sml_run_layer"} <= set(names)
    for name in names:
        assert hasattr(L, name), name
    assert sml.sml_version().startswith("sml ")


def _problem(**kw):
    base = dict(num_requests=2, num_tokens=3, num_heads=16, topk=2048, rope_dim=64, max_pages=4,
                max_ctx=256, ssmax=0, sm_scale=0.04, ssmax_s=0.4, ssmax_s_index=0.4,
                cu_q=0x1000, ctx_len=0x2000, block_table=0x3000)
    base.update(kw)
    return sml.Problem(**base)


def test_workspace_size_grows_with_stage_and_is_aligned(L):
    p = _problem()
    sizes = {s: sml.sml_workspace_size(p, s) for s in (1, 2, 3, 4)}
    assert all(v % 256 == 0 and v > 0 for v in sizes.values())
    assert sizes[4] >= sizes[2] and sizes[4] >= sizes[3]
    # the layer keeps its own score matrix: T * max_ctx floats
    assert sizes[4] >= 3 * 256 * 4


def test_invalid_problem_lists_every_reason(L):
    p = _problem(num_heads=24, topk=4096, rope_dim=32, sm_scale=float("nan"), cu_q=0)
    assert L.sml_workspace_size(ctypes.byref(p), 4) == 0
    msg = sml.sml_last_error()
    for part in ("num_heads", "topk", "rope_dim", "sm_scale", "cu_q is NULL"):
        assert part in msg, msg


def test_entry_points_reject_null_and_misaligned_without_cuda(L):
    p = _problem()
    ws_small = 256
    code = L.sml_indexer_scores(ctypes.byref(p), None, None, None, sml.Cache(None, 0), None,
                                0x100, ws_small, None)
    assert code == sml.SML_ERR_INVALID_ARG
    msg = sml.sml_last_error()
    assert "iq8" in msg and "index_cache.base" in msg and "scores" in msg
    code = L.sml_topk(ctypes.byref(p), 0x1000, 0x2000, 0x3000, 0x100, 8, None)
    assert code == sml.SML_ERR_WORKSPACE and "needs" in sml.sml_last_error()
    code = L.sml_sparse_mla_decode(ctypes.byref(p), 0x1001, sml.Cache(0x1000, 4), 0x10, 0x10,
                                   0x1000, 0x1000, 0x100, 1 << 30, None)
    assert code == sml.SML_ERR_INVALID_ARG and "q NULL or not 16-B aligned" in sml.sml_last_error()
    code = L.sml_run_layer(ctypes.byref(p), 0x1000, None, None, None, sml.Cache(0x1000, 4),
                           sml.Cache(None, 0), 0x1000, None, None, None, 0x1000, 0x1000, 0x100,
                           1 << 30, None)
    assert code == sml.SML_ERR_INVALID_ARG and "reuse_len" in sml.sml_last_error()


def test_unsupported_only_when_nothing_is_invalid(L):
    p = _problem(num_heads=8)
    assert L.sml_workspace_size(ctypes.byref(p), 1) == 0
    code = L.sml_topk(ctypes.byref(p), 0x1000, 0x2000, 0x3000, 0x100, 1 << 30, None)
    assert code == sml.SML_ERR_UNSUPPORTED
    assert sml.sml_status_string(code) == "unsupported shape or option"


def test_producers_reject_bad_arguments_without_cuda(L):
    code = L.sml_indexer_k_cache_write(0x1008, None, 4, sml.Cache(0x1001, 0), 0x80, None)
    assert code == sml.SML_ERR_INVALID_ARG
    msg = sml.sml_last_error()
    for part in ("k NULL or not 16-B aligned", "slot", "index_cache.base", "num_pages"):
        assert part in msg, msg
    code = L.sml_latent_cache_write(None, 0x1004, 0x2000, -1, sml.Cache(0x10000, 1 << 40), None, None)
    assert code == sml.SML_ERR_INVALID_ARG
    msg = sml.sml_last_error()
    for part in ("n < 0", "k_pe not 16-B aligned", "exceed int32"):
        assert part in msg, msg
    code = L.sml_indexer_q_quant(0x1000, 5, None, 0x2002, None)
    assert code == sml.SML_ERR_INVALID_ARG
    assert "iq8" in sml.sml_last_error() and "iq_scale" in sml.sml_last_error()
    # empty batches need no buffers
    assert L.sml_indexer_q_quant(None, 0, None, None, None) == sml.SML_OK


def test_cache_format_checks_without_cuda(L):
    p = _problem()
    lat = sml.Cache(0x10000, 4, 1, 0.0)          # plain E4M3 without a scale
    code = L.sml_sparse_mla_decode(ctypes.byref(p), 0x1000, lat, 0x2000, 0x3000, 0x4000, 0x5000, None, 0, None)
    assert code == sml.SML_ERR_INVALID_ARG and "latent.scale" in sml.sml_last_error()
    lat = sml.Cache(0x10000, 4, 7, 1.0)          # unknown format
    code = L.sml_sparse_mla_decode(ctypes.byref(p), 0x1000, lat, 0x2000, 0x3000, 0x4000, 0x5000, None, 0, None)
    assert "latent.format" in sml.sml_last_error()
    idx = sml.Cache(0x10000, 4, 1, 1.0)          # the indexer pool has one layout
    code = L.sml_indexer_scores(ctypes.byref(p), 0x1000, 0x2000, 0x3000, idx, 0x4000, None, 0, None)
    assert "index_cache.format" in sml.sml_last_error()


def test_cache_descriptors_of_every_latent_form():
    ds = torch.zeros(3 * sml.LATENT_PAGE_BYTES, dtype=torch.uint8)
    c = sml.latent_cache(ds)
    assert (c.num_pages, c.format) == (3, sml.SML_LATENT_FP8_DS_MLA)
    plain = torch.zeros(5 * sml.LATENT_E4M3_PAGE_BYTES, dtype=torch.uint8)
    c = sml.latent_cache(sml.E4M3Latent(plain, 0.25))
    assert (c.num_pages, c.format, c.scale) == (5, sml.SML_LATENT_E4M3, 0.25)
    bf = torch.zeros(2 * sml.LATENT_BF16_PAGE_BYTES, dtype=torch.uint8)
    c = sml.latent_cache(sml.Bf16Latent(bf))
    assert (c.num_pages, c.format) == (2, sml.SML_LATENT_BF16)
    c = sml.cache(None, sml.INDEX_PAGE_BYTES)
    assert (c.base, c.num_pages, c.format) == (None, 0, 0)


def _header_defines():
    """The integer #defines of include/sml.h, each evaluated from the ones before it."""
    import os
    import re
    path = os.path.join(os.path.dirname(__file__), "..", "include", "sml.h")
    vals = {}
    for line in open(path, encoding="utf-8"):
        m = re.match(r"#define\s+(SML_\w+)\s+(.+?)\s*(/\*.*)?$", line.strip())
        if not m or m.group(1) == "SML_H_":
            continue
        expr = m.group(2)
        if not re.fullmatch(r"[\sA-Z0-9_x()*+\-]+", expr):
            continue
        vals[m.group(1)] = eval(expr, {"__builtins__": {}}, dict(vals))
    return vals


def test_binding_constants_match_the_header():
    h = _header_defines()
    for name in ("SML_OK", "SML_ERR_INVALID_ARG", "SML_ERR_UNSUPPORTED", "SML_ERR_WORKSPACE", "SML_ERR_CUDA",
                 "SML_ERR_DEVICE_FAULT", "SML_ERR_TIMEOUT", "SML_FAULT_PAGE", "SML_FAULT_INDEX",
                 "SML_FAULT_LENGTHS", "SML_FAULT_TOPK_LEN", "SML_FAULT_TIMEOUT", "SML_STAGE_INDEXER",
                 "SML_STAGE_TOPK", "SML_STAGE_MLA", "SML_STAGE_LAYER", "SML_LATENT_FP8_DS_MLA",
                 "SML_LATENT_E4M3", "SML_LATENT_BF16", "SML_DCP_MAX_RANKS"):
        assert getattr(sml, name) == h[name], name
    assert sml.LATENT_PAGE_BYTES == h["SML_LATENT_PAGE_BYTES"] == 64 * 656
    assert sml.LATENT_E4M3_PAGE_BYTES == h["SML_LATENT_E4M3_PAGE_BYTES"] == 64 * 576
    assert sml.LATENT_BF16_PAGE_BYTES == h["SML_LATENT_BF16_PAGE_BYTES"] == 64 * 1152
    assert sml.INDEX_PAGE_BYTES == h["SML_INDEX_PAGE_BYTES"] == 64 * 132


def test_dcp_entry_points_reject_bad_arguments_without_cuda(L):
    rk = sml.DcpRanks()
    rk.num_ranks = 9
    rk.interleave = 0
    code = L.sml_dcp_merge_candidates(ctypes.byref(rk), 4, 2048, None, None, None, None, None)
    assert code in (sml.SML_ERR_INVALID_ARG, sml.SML_ERR_UNSUPPORTED)
    msg = sml.sml_last_error()
    for part in ("num_ranks", "interleave", "merged_scores"):
        assert part in msg, msg
    ptrs = (ctypes.c_void_p * 2)(None, None)
    code = L.sml_dcp_split_selection(2, 64, 3, 2048, 0x1000, 0x2000, 0x3000, ptrs, ptrs, None, None)
    assert code == sml.SML_ERR_INVALID_ARG and "local_idx[r]" in sml.sml_last_error()
    outs = (ctypes.c_void_p * 2)(0x1004, 0x2000)
    lses = (ctypes.c_void_p * 2)(0x3000, 0x4000)
    code = L.sml_lse_combine(2, 3, 16, outs, lses, 0x5000, 0x6000, None)
    assert code == sml.SML_ERR_INVALID_ARG and "16-B aligned" in sml.sml_last_error()
    assert L.sml_lse_combine(2, 0, 16, None, None, None, None, None) == sml.SML_OK
