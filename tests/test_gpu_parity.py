"""CUDA path vs the float64 oracle, through the C ABI, on seeded synthetic inputs.

Small ragged cases are compared element by element; the five benchmark
workloads at full size are compared on every top-k row and attention output
(oracle over the GPU's own selection) and on sampled indexer scores.
"""
import numpy as np
import pytest
import torch

from sparse_mla_attention_indexer_b200 import sml, synth
from sparse_mla_attention_indexer_b200.device import DeviceWorkload
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from sparse_mla_attention_indexer_b200 import build
    build.build()
    sml.lib()


def host(t):
    return t.cpu().numpy()


def run_stages(dw, i=0, reuse=None):
    """indexer -> top-k -> sparse MLA as three ABI calls; returns host arrays."""
    p = dw.problem(i)
    lay = dw.layers[i]
    ws = dw.workspace(sml.SML_STAGE_LAYER, i)
    idx, ln, out, lse = dw.outputs()
    scores = None
    if reuse is None:
        scores = dw.scores()
        sml.sml_indexer_scores(p, lay.iq8, lay.iq_scale, lay.iw, dw.index_cache, scores, ws)
        sml.sml_topk(p, scores, idx, ln, ws)
        use_idx, use_len = idx, ln
    else:
        use_idx, use_len = reuse
    sml.sml_sparse_mla_decode(p, lay.q, dw.latent, use_idx, use_len, out, lse, ws)
    code, bits = sml.sml_read_device_status(ws)
    assert code == sml.SML_OK, f"device status {code} bits {bits:#x}"
    return dict(scores=None if scores is None else host(scores), idx=host(use_idx),
                len=host(use_len), out=host(out), lse=host(lse), d_idx=use_idx, d_len=use_len)


def run_layer(dw, i=0, reuse=None):
    p = dw.problem(i)
    lay = dw.layers[i]
    ws = dw.workspace(sml.SML_STAGE_LAYER, i)
    idx, ln, out, lse = dw.outputs()
    if reuse is None:
        sml.sml_run_layer(p, lay.q, lay.iq8, lay.iq_scale, lay.iw, dw.latent, dw.index_cache,
                          None, None, idx, ln, out, lse, ws)
    else:
        sml.sml_run_layer(p, lay.q, None, None, None, dw.latent, None, reuse[0], reuse[1],
                          None, None, out, lse, ws)
    code, bits = sml.sml_read_device_status(ws)
    assert code == sml.SML_OK, f"device status {code} bits {bits:#x}"
    return dict(idx=host(idx) if reuse is None else host(reuse[0]),
                len=host(ln) if reuse is None else host(reuse[1]), out=host(out), lse=host(lse))


# --- small ragged cases: every element --------------------------------------------

SMALL = [
    # (ctx lengths, query counts, heads, topk, rope_dim, ssmax, permuted)
    ([1, 63, 64, 65, 300, 2049], [1, 1, 2, 3, 1, 4], 16, 2048, 64, False, True),
    ([4097, 777, 128], [1, 2, 1], 32, 64, 64, True, True),
    ([5000, 2100], [3, 1], 64, 7, 0, True, False),
    ([3000], [2], 128, 1, 64, False, True),
    ([2500, 129, 2048], [2, 1, 1], 128, 2048, 0, True, True),
]


@pytest.mark.parametrize("case", range(len(SMALL)))
def test_small_ragged_every_element(case):
    L, Q, H, K, rope, ssmax, perm = SMALL[case]
    wl = synth.make_workload(f"small{case}", L, Q, H, topk=K, permuted=perm, ssmax=ssmax,
                             layers=(("l0", rope, True, None),), extra_pages=3)
    dw = DeviceWorkload(wl)
    r = run_stages(dw)
    parity.check_scores(wl, 0, r["scores"])
    parity.check_topk(wl, r["scores"], r["idx"], r["len"])
    parity.check_attention(wl, 0, r["idx"], r["len"], r["out"], r["lse"])
    # the one-call layer gives the same bits as the three stages
    r2 = run_layer(dw)
    assert np.array_equal(r2["idx"], r["idx"]) and np.array_equal(r2["len"], r["len"])
    assert np.array_equal(r2["out"], r["out"]) and np.array_equal(r2["lse"], r["lse"], equal_nan=True)


def test_tiny_decode_workload_every_element():
    wl = synth.tiny_decode()
    dw = DeviceWorkload(wl)
    r = run_stages(dw)
    parity.check_scores(wl, 0, r["scores"])
    parity.check_topk(wl, r["scores"], r["idx"], r["len"])
    parity.check_attention(wl, 0, r["idx"], r["len"], r["out"], r["lse"])


# --- top-k on crafted scores: ties, signed zeros, NaN, -inf, two-level rows --------

def _topk_case(rows, K):
    """Run sml_topk on explicit score rows (one request per row, 1 query each)."""
    T = len(rows)
    n = [len(x) for x in rows]
    max_ctx = max(n)
    scores = np.full((T, max_ctx), np.nan, dtype=np.float32)
    for t, x in enumerate(rows):
        scores[t, :len(x)] = x
    cu_q = torch.arange(T + 1, dtype=torch.int32, device="cuda")
    ctx = torch.tensor(n, dtype=torch.int32, device="cuda")
    bt = torch.zeros(T, (max_ctx + 63) // 64, dtype=torch.int32, device="cuda")
    p = sml.make_problem(num_heads=16, topk=K, rope_dim=64, cu_q=cu_q, ctx_len=ctx, block_table=bt,
                         max_ctx=max_ctx, sm_scale=0.04, num_tokens=T)
    ws = torch.empty(sml.sml_workspace_size(p, sml.SML_STAGE_TOPK), dtype=torch.uint8, device="cuda")
    sml.sml_workspace_init(ws)
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    ln = torch.empty(T, dtype=torch.int32, device="cuda")
    d_scores = torch.from_numpy(scores).cuda()
    for _ in range(2):  # twice: the arrival counters must be back at zero
        sml.sml_topk(p, d_scores, idx, ln, ws)
        code, bits = sml.sml_read_device_status(ws)
        assert code == sml.SML_OK, bits
        idx_h, ln_h = host(idx), host(ln)
        for t, x in enumerate(rows):
            want = parity.dsa.topk_row(np.asarray(x, dtype=np.float32), K)
            assert ln_h[t] == min(K, len(x))
            assert np.array_equal(idx_h[t, :ln_h[t]], want), f"row {t}"
            assert np.all(idx_h[t, ln_h[t]:] == -1)


def test_topk_ties_signed_zero_nan_inf():
    rng = np.random.default_rng(1)
    vals = np.array([-1.5, -0.0, 0.0, 0.25, 2.0, np.inf, -np.inf, np.nan], dtype=np.float32)
    rows = [rng.choice(vals, size=n) for n in (1, 5, 40, 2047, 2048, 2049, 5000)]
    rows.append(np.zeros(3000, dtype=np.float32))               # all tied: first K positions
    rows.append(np.full(3000, -0.0, dtype=np.float32))
    rows.append(np.where(rng.random(4000) < 0.5, 0.0, -0.0).astype(np.float32))
    rows.append(rng.standard_normal(30000).astype(np.float32))
    _topk_case(rows, 2048)
    _topk_case(rows, 7)
    _topk_case(rows, 1)


def test_topk_cluster_heavy_ties():
    """Rows of one cluster (at most 8 chunks) whose threshold bucket holds more
    than 4,096 keys, so the cluster runs its radix select over that bucket:
    exact zeros below fewer than K positive scores (the floor falls to the
    zeros' bin, every key is a candidate), an all-zero row, and signed zeros
    with a few larger keys; each with K = 2048 and K = 7."""
    rng = np.random.default_rng(4)
    zeros_below = np.zeros(31_000, dtype=np.float32)
    zeros_below[rng.choice(31_000, 1000, replace=False)] = rng.random(1000).astype(np.float32) + 0.5
    all_zero = np.zeros(60_000, dtype=np.float32)
    signed = np.where(rng.random(45_000) < 0.5, 0.0, -0.0).astype(np.float32)
    signed[rng.choice(45_000, 3, replace=False)] = 2.0
    signed[rng.choice(45_000, 5000, replace=False)] = -1.0
    rows = [zeros_below, all_zero, signed]
    _topk_case(rows, 2048)
    _topk_case(rows, 7)


def test_topk_cluster_misjudged_floor_and_unaligned_rows():
    """Rows of one cluster: a row whose large keys sit only at the strided
    sample's positions, so fewer than K keys pass the sampled floor and every
    CTA reselects over its chunk reloaded from global memory; and a row
    stride (max_ctx = 30,001) that leaves rows 1..3 off a 16-B boundary, so
    their chunks arrive by plain loads instead of the bulk copy."""
    rng = np.random.default_rng(5)
    n = 20_000
    misjudged = np.zeros(n, dtype=np.float32)
    pos = (np.arange(1024, dtype=np.int64) * n) // 1024          # the kernel's strided sample
    misjudged[pos] = 10.0 + np.arange(1024, dtype=np.float32) * 1e-3
    rows = [rng.standard_normal(30_001).astype(np.float32), misjudged,
            rng.standard_normal(29_999).astype(np.float32),
            np.round(rng.standard_normal(25_003) * 3).astype(np.float32)]
    _topk_case(rows, 2048)
    _topk_case(rows, 7)


def test_topk_two_level_rows_with_ties_across_chunks():
    rng = np.random.default_rng(2)
    big = rng.standard_normal(100_000).astype(np.float32)
    big[rng.choice(100_000, 5000, replace=False)] = 3.0          # 5000 ties above the rest
    coarse = np.round(rng.standard_normal(70_000) * 4).astype(np.float32)   # heavy ties
    exact = rng.standard_normal(32_769).astype(np.float32)     # one past a chunk
    _topk_case([big, coarse, exact, rng.standard_normal(300_000).astype(np.float32)], 2048)
    _topk_case([coarse, exact], 100)


def test_topk_long_rows_floor_paths():
    """Rows over eight chunks: a sampled floor cuts each chunk's candidates.
    Cover the floor's three outcomes: keys above it spread thinly (floor
    segments), one chunk holding more than K of them (that chunk falls back to
    its own top K), and a sample that misjudges (only the sampled positions are
    large, so fewer than K candidates exist and the whole row is selected)."""
    rng = np.random.default_rng(3)
    n = 300_000
    misjudged = np.zeros(n, dtype=np.float32)
    pos = (np.arange(1024, dtype=np.int64) * n) // 1024          # the kernel's strided sample
    misjudged[pos] = 10.0 + np.arange(1024, dtype=np.float32) * 1e-3
    crowded = rng.standard_normal(200_000).astype(np.float32)
    crowded[49152:65536] += 10.0                                 # one chunk holds every large key
    ties = rng.standard_normal(500_000).astype(np.float32)
    ties[rng.choice(500_000, 1000, replace=False)] = 4.0         # ties near the threshold
    spread = rng.standard_normal(1_048_576).astype(np.float32)
    _topk_case([misjudged, crowded, ties, spread], 2048)
    _topk_case([misjudged, crowded, ties], 7)


# --- the benchmark workloads at full size -----------------------------------------

def test_batched_decode_full():
    wl = synth.batched_decode()
    dw = DeviceWorkload(wl)
    r = run_stages(dw)
    parity.check_scores(wl, 0, r["scores"], tokens=range(0, wl.T, 4))
    parity.check_scores(wl, 0, r["scores"], tokens=range(1, wl.T, 4), sample=4000)
    parity.check_topk(wl, r["scores"], r["idx"], r["len"])
    parity.check_attention(wl, 0, r["idx"], r["len"], r["out"], r["lse"])
    r2 = run_layer(dw)   # the call bench.py times
    assert np.array_equal(r2["idx"], r["idx"]) and np.array_equal(r2["out"], r["out"])


def test_spec_verify_full():
    wl = synth.spec_verify()
    dw = DeviceWorkload(wl)
    r = run_stages(dw)
    parity.check_scores(wl, 0, r["scores"], sample=3000)
    parity.check_topk(wl, r["scores"], r["idx"], r["len"])
    parity.check_attention(wl, 0, r["idx"], r["len"], r["out"], r["lse"])


def test_long_context_three_layers():
    wl = synth.long_context()
    dw = DeviceWorkload(wl)
    rope = run_stages(dw, 0)
    parity.check_scores(wl, 0, rope["scores"], sample=20000)
    parity.check_topk(wl, rope["scores"], rope["idx"], rope["len"])
    parity.check_attention(wl, 0, rope["idx"], rope["len"], rope["out"], rope["lse"])
    nope = run_stages(dw, 1)
    parity.check_scores(wl, 1, nope["scores"], sample=20000)
    parity.check_topk(wl, nope["scores"], nope["idx"], nope["len"])
    parity.check_attention(wl, 1, nope["idx"], nope["len"], nope["out"], nope["lse"])
    shared = run_stages(dw, 2, reuse=(nope["d_idx"], nope["d_len"]))
    assert np.array_equal(shared["idx"], nope["idx"])
    parity.check_attention(wl, 2, shared["idx"], shared["len"], shared["out"], shared["lse"])
    lay = run_layer(dw, 2, reuse=(nope["d_idx"], nope["d_len"]))
    assert np.array_equal(lay["out"], shared["out"])


def test_prefill_chunk_sampled():
    wl = synth.prefill_chunk()
    dw = DeviceWorkload(wl)
    r = run_stages(dw)
    toks = list(range(0, 8)) + list(range(8, wl.T, 97)) + [wl.T - 1]
    parity.check_scores(wl, 0, r["scores"], tokens=toks, sample=1500)
    parity.check_topk(wl, r["scores"], r["idx"], r["len"], tokens=toks)
    parity.check_attention(wl, 0, r["idx"], r["len"], r["out"], r["lse"], tokens=toks)


# --- device-side checks: bad data sets status bits, never traps --------------------

def test_device_checks_set_status_bits():
    wl = synth.make_workload("faults", [500, 300], [1, 2], 16, topk=64)
    dw = DeviceWorkload(wl)
    p = dw.problem(0)
    lay = dw.layers[0]
    ws = dw.workspace()
    idx, ln, out, lse = dw.outputs()
    # a block-table entry past the pool
    bad_bt = dw.block_table.clone()
    bad_bt[0, 2] = wl.num_pages + 5
    pb = sml.make_problem(num_heads=16, topk=64, rope_dim=64, cu_q=dw.cu_q, ctx_len=dw.ctx_len,
                          block_table=bad_bt, max_ctx=wl.max_ctx, sm_scale=wl.sm_scale, num_tokens=wl.T)
    sml.sml_run_layer(pb, lay.q, lay.iq8, lay.iq_scale, lay.iw, dw.latent, dw.index_cache, None, None,
                      idx, ln, out, lse, ws)
    code, bits = sml.sml_read_device_status(ws, clear=True)
    assert code == sml.SML_ERR_DEVICE_FAULT and bits & sml.SML_FAULT_PAGE
    # a selected position outside the visible context, and a length past topk
    sml.sml_run_layer(p, lay.q, lay.iq8, lay.iq_scale, lay.iw, dw.latent, dw.index_cache, None, None,
                      idx, ln, out, lse, ws)
    assert sml.sml_read_device_status(ws)[0] == sml.SML_OK
    bad_idx = idx.clone()
    bad_idx[1, 3] = 10_000
    sml.sml_sparse_mla_decode(p, lay.q, dw.latent, bad_idx, ln, out, lse, ws)
    code, bits = sml.sml_read_device_status(ws)
    assert code == sml.SML_ERR_DEVICE_FAULT and bits & sml.SML_FAULT_INDEX
    bad_len = ln.clone()
    bad_len[0] = 65
    sml.sml_sparse_mla_decode(p, lay.q, dw.latent, idx, bad_len, out, lse, ws)
    code, bits = sml.sml_read_device_status(ws)
    assert code == sml.SML_ERR_DEVICE_FAULT and bits & sml.SML_FAULT_TOPK_LEN
    # context length inconsistent with the query count
    bad_ctx = dw.ctx_len.clone()
    bad_ctx[1] = 1
    pc = sml.make_problem(num_heads=16, topk=64, rope_dim=64, cu_q=dw.cu_q, ctx_len=bad_ctx,
                          block_table=dw.block_table, max_ctx=wl.max_ctx, sm_scale=wl.sm_scale,
                          num_tokens=wl.T)
    sml.sml_run_layer(pc, lay.q, lay.iq8, lay.iq_scale, lay.iw, dw.latent, dw.index_cache, None, None,
                      idx, ln, out, lse, ws)
    code, bits = sml.sml_read_device_status(ws)
    assert code == sml.SML_ERR_DEVICE_FAULT and bits & sml.SML_FAULT_LENGTHS
    # the context is still usable
    sml.sml_run_layer(p, lay.q, lay.iq8, lay.iq_scale, lay.iw, dw.latent, dw.index_cache, None, None,
                      idx, ln, out, lse, ws)
    assert sml.sml_read_device_status(ws)[0] == sml.SML_OK
    torch.cuda.synchronize()


# --- the plain per-tensor E4M3 latent pool (576-B rows) ------------------------------

@pytest.mark.parametrize("case", [0, 1, 2, 4])
def test_plain_e4m3_latent_small_every_element(case):
    L, Q, H, K, rope, ssmax, perm = SMALL[case]
    wl = synth.make_workload(f"plain{case}", L, Q, H, topk=K, permuted=perm, ssmax=ssmax,
                             layers=(("l0", rope, True, None),), extra_pages=3, latent_format="e4m3")
    dw = DeviceWorkload(wl)
    r = run_stages(dw)
    parity.check_topk(wl, r["scores"], r["idx"], r["len"])
    parity.check_attention(wl, 0, r["idx"], r["len"], r["out"], r["lse"])
    r2 = run_layer(dw)
    assert np.array_equal(r2["out"], r["out"]) and np.array_equal(r2["lse"], r["lse"], equal_nan=True)


def test_plain_e4m3_latent_batched_decode_full():
    base = synth.batched_decode()
    wl = synth.make_workload("batched_decode_e4m3", base.ctx_len, np.ones(base.B, np.int32), 16,
                             latent_format="e4m3")
    dw = DeviceWorkload(wl)
    r = run_stages(dw)
    parity.check_topk(wl, r["scores"], r["idx"], r["len"])
    parity.check_attention(wl, 0, r["idx"], r["len"], r["out"], r["lse"])


# --- the bf16 latent pool (1,152-B rows) ---------------------------------------------

@pytest.mark.parametrize("case", [0, 1, 2, 4])
def test_bf16_latent_small_every_element(case):
    L, Q, H, K, rope, ssmax, perm = SMALL[case]
    wl = synth.make_workload(f"bf16_{case}", L, Q, H, topk=K, permuted=perm, ssmax=ssmax,
                             layers=(("l0", rope, True, None),), extra_pages=3, latent_format="bf16")
    dw = DeviceWorkload(wl)
    r = run_stages(dw)
    parity.check_topk(wl, r["scores"], r["idx"], r["len"])
    parity.check_attention(wl, 0, r["idx"], r["len"], r["out"], r["lse"])
    r2 = run_layer(dw)
    assert np.array_equal(r2["out"], r["out"]) and np.array_equal(r2["lse"], r["lse"], equal_nan=True)


def test_bf16_latent_batched_decode_full():
    base = synth.batched_decode()
    wl = synth.make_workload("batched_decode_bf16", base.ctx_len, np.ones(base.B, np.int32), 16,
                             latent_format="bf16")
    dw = DeviceWorkload(wl)
    r = run_stages(dw)
    parity.check_topk(wl, r["scores"], r["idx"], r["len"])
    parity.check_attention(wl, 0, r["idx"], r["len"], r["out"], r["lse"])


def test_plain_e4m3_rejects_a_bad_scale():
    wl = synth.make_workload("plain_bad", [300], [1], 16, topk=64, latent_format="e4m3")
    dw = DeviceWorkload(wl)
    p = dw.problem(0)
    idx, ln, out, lse = dw.outputs()
    bad = sml.E4M3Latent(dw.latent.pool, 0.0)
    with pytest.raises(sml.SmlError) as e:
        sml.sml_sparse_mla_decode(p, dw.layers[0].q, bad, idx, ln, out, lse, dw.workspace())
    assert "latent.scale" in str(e.value)
