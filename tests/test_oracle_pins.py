"""Pins of the float64 oracle to things other than itself.

Each test checks the oracle against what the pages print (tests/golden), the
FP8 / bf16 format definitions and PyTorch's casts, a library routine
(scaled_dot_product_attention, torch.topk), closed forms, invariants that the
method implies, or brute force on tiny inputs written a different way.
"""
import math
import struct

import numpy as np
import pytest
import torch

from oracle import dsa, formats as F, mla
from sparse_mla_attention_indexer_b200 import synth

GOLDEN = __file__.rsplit("/", 1)[0] + "/golden/kv_bytes.txt"


def golden():
    vals = {}
    for line in open(GOLDEN, encoding="utf-8"):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split()
            vals[k] = float(v)
    return vals


# --- formats ------------------------------------------------------------------

def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = F.decode_e4m3(codes)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(ref[ok]))


def test_e4m3_landmarks_of_the_format():
    v = F.decode_e4m3(np.array([0x7E, 0x01, 0x07, 0x08, 0x38, 0x80, 0xFE], dtype=np.uint8))
    assert list(v) == [448.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, -0.0, -448.0]
    assert np.isnan(F.decode_e4m3(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def test_bf16_decode_matches_torch():
    bits = np.random.default_rng(1).integers(0, 1 << 16, size=4096, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    ours = F.decode_bf16(bits)
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok]) and np.array_equal(np.isnan(ours), ~ok)


def test_byte_accounting_printed_on_the_pages():
    g = golden()
    assert F.LATENT_ROW_BYTES == g["latent_row_fp8_ds_mla"]
    assert F.PLAIN_E4M3_ROW_BYTES == g["latent_row_plain_e4m3"]
    assert F.BF16_ROW_BYTES == g["latent_row_bf16"]
    assert F.INDEXER_ROW_BYTES == g["indexer_row"]
    layers, idx_layers = int(g["cache_owning_layers"]), 44
    assert F.LATENT_ROW_BYTES * layers == g["latent_bytes_per_token"]
    assert F.INDEXER_ROW_BYTES * idx_layers == g["indexer_bytes_per_token"]
    assert F.LATENT_ROW_BYTES * layers + F.INDEXER_ROW_BYTES * idx_layers == g["kv_bytes_per_token"]
    plain = F.PLAIN_E4M3_ROW_BYTES * layers + F.INDEXER_ROW_BYTES * idx_layers
    bf16 = F.BF16_ROW_BYTES * layers + F.INDEXER_ROW_BYTES * idx_layers
    assert plain == g["plain_e4m3_bytes_per_token"] and bf16 == g["bf16_bytes_per_token"]
    assert round(bf16 / plain, 2) == g["e4m3_vs_bf16_capacity"]
    assert round(g["dcp8_capacity_fp8_mtok"] / g["tp8_capacity_fp8_mtok"], 1) == g["dcp8_capacity_gain"]
    assert F.LATENT_PAGE_BYTES == 64 * 656 and F.INDEXER_PAGE_BYTES == 64 * 132


def _pack_latent_row(codes, scales, pe_bits):
    return bytes(codes) + struct.pack("<4f", *scales) + struct.pack("<64H", *pe_bits)


def test_latent_row_layout_from_independent_packing():
    rng = np.random.default_rng(7)
    pool = bytearray(3 * 64 * 656)
    want = {}
    for page, row in [(2, 0), (0, 63), (1, 17)]:
        codes = rng.integers(0, 0x7E, size=512).astype(np.uint8)
        scales = [0.5, 0.25, 2.0, 0.125]
        pe = rng.integers(0, 0x3F80, size=64).astype(np.uint16)
        off = page * 64 * 656 + row * 656
        pool[off:off + 656] = _pack_latent_row(codes, scales, pe)
        want[(page, row)] = (codes, scales, pe)
    pool = np.frombuffer(bytes(pool), dtype=np.uint8)
    keys = list(want)
    c_hat, k_pe = F.latent_rows(pool, [k[0] for k in keys], [k[1] for k in keys])
    for i, k in enumerate(keys):
        codes, scales, pe = want[k]
        for d in (0, 127, 128, 300, 511):
            assert c_hat[i, d] == F.e4m3_value(int(codes[d])) * scales[d // 128]
        for d in (0, 63):
            assert k_pe[i, d] == struct.unpack("<f", struct.pack("<I", int(pe[d]) << 16))[0]


def test_indexer_page_layout_from_independent_packing():
    pool = bytearray(2 * 64 * 132)
    page, row = 1, 9
    codes = bytes((0x10 + i) % 0x7E for i in range(128))   # no NaN code
    off = page * 64 * 132
    pool[off + row * 128: off + row * 128 + 128] = codes
    pool[off + 64 * 128 + row * 4: off + 64 * 128 + row * 4 + 4] = struct.pack("<f", 0.75)
    k = F.indexer_keys(np.frombuffer(bytes(pool), dtype=np.uint8), [page], [row])
    assert k.shape == (1, 128)
    assert all(k[0, d] == F.e4m3_value(codes[d]) * 0.75 for d in range(128))


def test_generator_quantisation_within_half_spacing():
    x = synth.stream(3, "q").standard_normal((64, 512), dtype=np.float32)
    codes, scale = synth.quantise_rows(x, 128)
    back = F.decode_e4m3(codes).reshape(64, 4, 128) * scale[:, :, None]
    xb = x.reshape(64, 4, 128).astype(np.float64)
    # E4M3 has 3 mantissa bits: rounding error <= 2^-4 relative (normal range)
    # or half a subnormal step 2^-10 (in units of the scale).
    err = np.abs(back - xb)
    bound = np.maximum(np.abs(xb) * 2.0 ** -4, 2.0 ** -10 * scale[:, :, None]) * (1 + 1e-6)
    assert np.all(err <= bound)
    assert np.allclose(np.abs(back).max(axis=2), np.abs(xb).max(axis=2), rtol=1e-6)


# --- small workloads -----------------------------------------------------------

@pytest.fixture(scope="module")
def small():
    # two requests: 300 tokens / 1 query, 77 tokens / 3 queries; ragged last pages
    return synth.make_workload("pins_small", [300, 77], [1, 3], 4, topk=64, ssmax=True,
                               layers=(("rope", 64, True, None), ("nope", 0, True, None)))


def test_visible_lengths_causal_within_request(small):
    n = dsa.visible_lengths(small.cu_q, small.ctx_len)
    assert list(n) == [300, 75, 76, 77]


def _brute_score(wl, t, s):
    """Indexer score by scalar loops over raw bytes (independent of oracle.formats)."""
    req = 0 if t < wl.cu_q[1] else 1
    page = int(wl.block_table[req, s // 64])
    row = s % 64
    base = page * 64 * 132
    kcodes = wl.index_cache[base + row * 128: base + row * 128 + 128]
    sk = struct.unpack("<f", bytes(wl.index_cache[base + 8192 + row * 4: base + 8192 + row * 4 + 4]))[0]
    lay = wl.layers[0]
    sq = float(lay.iq_scale[t])
    total = 0.0
    for h in range(64):
        dot = 0.0
        for d in range(128):
            dot += F.e4m3_value(int(lay.iq8[t, h, d])) * F.e4m3_value(int(kcodes[d]))
        total += float(lay.iw[t, h]) * max(dot * sq * sk, 0.0)
    n = int(dsa.visible_lengths(wl.cu_q, wl.ctx_len)[t])
    return total * (wl.ssmax_s_index * math.log(n) if wl.ssmax else 1.0)


def test_indexer_brute_force_scalar_loops(small):
    rows = dsa.indexer_scores(small.view(0), small.layers[0].iq8, small.layers[0].iq_scale,
                              small.layers[0].iw, small.index_cache)
    for t, s in [(0, 0), (0, 299), (0, 130), (1, 74), (3, 76), (2, 5)]:
        assert rows[t][s] == pytest.approx(_brute_score(small, t, s), rel=1e-12, abs=1e-12)
    assert [len(r) for r in rows] == [300, 75, 76, 77]


def test_indexer_closed_forms(small):
    v = small.view(0)
    lay = small.layers[0]
    q8 = lay.iq8[0]
    n = 300
    keys = F.indexer_keys(small.index_cache, *F.physical(small.block_table[0], np.arange(n)))
    q = F.decode_e4m3(q8) * float(lay.iq_scale[0])
    # one head, weight 1: the plain (ReLU-ed) scaled dot product
    w = np.zeros(64)
    w[5] = 1.0
    row = dsa.indexer_scores_row(q8, lay.iq_scale[0], w, small.index_cache, small.block_table[0], n, 1.0)
    assert np.allclose(row, np.maximum(keys @ q[5], 0.0), rtol=1e-13, atol=0)
    # a head whose query is negated contributes ReLU(-dot): the two add up to |dot|
    q8_neg = q8.copy()
    q8_neg[6] = q8[5] ^ 0x80
    w2 = np.zeros(64)
    w2[5] = w2[6] = 1.0
    row2 = dsa.indexer_scores_row(q8_neg, lay.iq_scale[0], w2, small.index_cache, small.block_table[0], n, 1.0)
    assert np.allclose(row2, np.abs(keys @ q[5]), rtol=1e-13)
    # linear in the head weights and in the SSMax factor
    wa, wb = lay.iw[0].astype(np.float64), np.linspace(-1, 1, 64)
    ra = dsa.indexer_scores_row(q8, lay.iq_scale[0], wa, small.index_cache, small.block_table[0], n, 1.0)
    rb = dsa.indexer_scores_row(q8, lay.iq_scale[0], wb, small.index_cache, small.block_table[0], n, 1.0)
    rab = dsa.indexer_scores_row(q8, lay.iq_scale[0], wa + 2 * wb, small.index_cache, small.block_table[0], n, 3.0)
    assert np.allclose(rab, 3.0 * (ra + 2 * rb), rtol=1e-10, atol=1e-12)


# --- top-k -----------------------------------------------------------------------

def _brute_topk(scores, k):
    """Repeated argmax: take the largest remaining score, lowest index first."""
    left = list(range(len(scores)))
    picked = []
    while left and len(picked) < k:
        def better(a, b):
            sa, sb = scores[a], scores[b]
            if math.isnan(sb) and not math.isnan(sa):
                return True
            if math.isnan(sa):
                return False
            return sa > sb or (sa == sb and a < b)
        best = left[0]
        for i in left[1:]:
            if better(i, best):
                best = i
        picked.append(best)
        left.remove(best)
    return sorted(picked)


def test_topk_brute_force_with_ties_nan_and_signed_zero():
    rng = np.random.default_rng(11)
    for trial in range(60):
        n = int(rng.integers(1, 40))
        vals = rng.choice([-1.5, -0.0, 0.0, 0.25, 2.0, np.inf, -np.inf, np.nan], size=n)
        for k in (1, 3, 7, n, n + 5):
            assert list(dsa.topk_row(vals, k)) == _brute_topk(list(vals), k)


def test_topk_special_cases_and_torch_topk():
    assert list(dsa.topk_row(np.zeros(50), 7)) == list(range(7))
    assert list(dsa.topk_row(np.array([-0.0, 0.0, -0.0]), 2)) == [0, 1]
    assert list(dsa.topk_row(np.arange(5.0), 10)) == [0, 1, 2, 3, 4]
    x = np.random.default_rng(2).standard_normal(5000)
    ref = torch.topk(torch.from_numpy(x), 2048).indices.numpy()
    assert np.array_equal(dsa.topk_row(x, 2048), np.sort(ref))


# --- attention -----------------------------------------------------------------------

def test_attention_equals_sdpa_library_routine(small):
    v = small.view(0)
    t = 2
    pos = np.array([0, 3, 17, 40, 63, 64, 70])
    out, lse = mla.token_attention(v, small.latent, t, pos)
    c_hat, k_pe = F.latent_rows(small.latent, *F.physical(small.block_table[1], pos))
    q = torch.from_numpy(F.decode_bf16(small.layers[0].q[t]))                 # [H, 576]
    k = torch.from_numpy(np.concatenate([c_hat, k_pe], axis=1))              # [m, 576]
    n = int(dsa.visible_lengths(small.cu_q, small.ctx_len)[t])
    scale = small.sm_scale * 0.4 * math.log(n)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[None, :, None, :], k[None, None].expand(1, 4, -1, -1),
        torch.from_numpy(c_hat)[None, None].expand(1, 4, -1, -1), scale=scale)[0, :, 0, :]
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
    z = scale * (q.numpy() @ k.numpy().T)
    assert np.allclose(lse, np.log(np.exp(z).sum(axis=1)), rtol=1e-12)


def test_attention_closed_forms(small):
    rng = np.random.default_rng(5)
    c_hat = rng.standard_normal((9, 512))
    k_pe = rng.standard_normal((9, 64))
    out, lse = mla.attend(np.zeros((3, 576)), c_hat, k_pe, 64, 0.1)
    assert np.allclose(out, c_hat.mean(axis=0)) and np.allclose(lse, math.log(9))
    q = rng.standard_normal((3, 576))
    out1, lse1 = mla.attend(q, c_hat[4:5], k_pe[4:5], 64, 0.3)
    assert np.allclose(out1, c_hat[4]) and np.allclose(lse1, 0.3 * (q @ np.concatenate([c_hat[4], k_pe[4]])))
    out0, lse0 = mla.attend(q, c_hat[:0], k_pe[:0], 64, 0.3)
    assert np.all(out0 == 0) and np.all(lse0 == -np.inf)
    # the logit scale multiplies q . k: (4q, scale/4) gives the same result
    out_a, lse_a = mla.attend(q, c_hat, k_pe, 64, 0.2)
    out_b, lse_b = mla.attend(4.0 * q, c_hat, k_pe, 64, 0.05)
    assert np.allclose(out_a, out_b, rtol=1e-12) and np.allclose(lse_a, lse_b, rtol=1e-12)
    # a key whose k_pe part is raised gains weight only through the RoPE term
    k_pe2 = k_pe.copy()
    k_pe2[2] += q[0, 512:] * 10.0
    out_c, _ = mla.attend(q[:1], c_hat, k_pe2, 64, 0.2)
    out_d, _ = mla.attend(q[:1, :512], c_hat, k_pe2, 0, 0.2)
    assert np.linalg.norm(out_c[0] - c_hat[2]) < np.linalg.norm(out_d[0] - c_hat[2])


def _brute_attention(q, c_hat, k_pe, rope_dim, scale):
    H, m = q.shape[0], c_hat.shape[0]
    out = np.zeros((H, 512))
    lse = np.zeros(H)
    for h in range(H):
        z = []
        for i in range(m):
            s = sum(q[h, d] * c_hat[i, d] for d in range(512))
            if rope_dim:
                s += sum(q[h, 512 + d] * k_pe[i, d] for d in range(rope_dim))
            z.append(scale * s)
        mx = max(z)
        e = [math.exp(x - mx) for x in z]
        tot = sum(e)
        for i in range(m):
            for d in range(512):
                out[h, d] += e[i] / tot * c_hat[i, d]
        lse[h] = mx + math.log(tot)
    return out, lse


def test_attention_brute_force_scalar_loops(small):
    rng = np.random.default_rng(9)
    c_hat = rng.standard_normal((5, 512))
    k_pe = rng.standard_normal((5, 64))
    q = rng.standard_normal((2, 576))
    for rope in (64, 0):
        qq = q if rope else q[:, :512]
        o, l = mla.attend(qq, c_hat, k_pe, rope, 0.37)
        bo, bl = _brute_attention(qq, c_hat, k_pe, rope, 0.37)
        assert np.allclose(o, bo, rtol=1e-11, atol=1e-12) and np.allclose(l, bl, rtol=1e-12)


def test_nope_equals_rope_path_with_zero_rope_query(small):
    v_nope = small.view(1)
    t = 1
    pos = np.arange(0, 75, 4)
    out0, lse0 = mla.token_attention(v_nope, small.latent, t, pos)
    v_rope = small.view(1)
    q_pad = np.zeros(v_nope.q.shape[:2] + (576,), dtype=np.uint16)
    q_pad[:, :, :512] = v_nope.q
    v_rope.q, v_rope.rope_dim = q_pad, 64
    out1, lse1 = mla.token_attention(v_rope, small.latent, t, pos)
    assert np.allclose(out0, out1, rtol=1e-13) and np.allclose(lse0, lse1, rtol=1e-13)


def test_sparse_equals_dense_when_context_fits_topk(small):
    wl = synth.make_workload("pins_dense", [200, 64, 1], [1, 2, 1], 4, topk=256)
    v = wl.view(0)
    idx, out, lse = mla.run_layer(v, wl.latent, wl.index_cache)
    dout, dlse = mla.dense_mla(v, wl.latent)
    assert np.allclose(out, dout, rtol=1e-13, atol=1e-14) and np.allclose(lse, dlse, rtol=1e-13)
    assert [len(i) for i in idx] == [200, 63, 64, 1]


def test_split_then_lse_merge_equals_unsplit(small):
    v = small.view(0)
    pos = np.arange(300)
    whole_o, whole_l = mla.token_attention(v, small.latent, 0, pos)
    rng = np.random.default_rng(4)
    for S in (1, 2, 5, 16):
        cuts = np.sort(rng.choice(np.arange(1, 300), size=S - 1, replace=False)) if S > 1 else []
        parts = np.split(pos, cuts)
        parts.append(np.array([], dtype=np.int64))          # an empty split drops out
        po, pl = zip(*[mla.token_attention(v, small.latent, 0, p) for p in parts])
        o, l = mla.lse_merge(np.stack(po), np.stack(pl))
        assert np.allclose(o, whole_o, rtol=1e-12, atol=1e-13) and np.allclose(l, whole_l, rtol=1e-13)


def test_block_table_permutation_invariance():
    ident = synth.make_workload("pins_perm", [150, 190], [2, 1], 2, topk=32, permuted=False)
    perm = np.random.default_rng(8).permutation(ident.num_pages)       # logical page p -> perm[p]
    lat = np.empty_like(ident.latent).reshape(ident.num_pages, -1)
    idc = np.empty_like(ident.index_cache).reshape(ident.num_pages, -1)
    lat[perm] = ident.latent.reshape(ident.num_pages, -1)
    idc[perm] = ident.index_cache.reshape(ident.num_pages, -1)
    v0 = ident.view(0)
    v1 = ident.view(0)
    v1.block_table = perm[ident.block_table].astype(np.int32)
    a = mla.run_layer(v0, ident.latent, ident.index_cache)
    b = mla.run_layer(v1, lat.reshape(-1), idc.reshape(-1))
    assert all(np.array_equal(x, y) for x, y in zip(a[0], b[0]))
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])


def test_shared_indexer_layer_reuses_owner_indices(small):
    owner = small.view(1)
    idx_owner, _, _ = mla.run_layer(owner, small.latent, small.index_cache)
    shared = small.view(0)
    idx_shared, out_s, _ = mla.run_layer(shared, small.latent, None, reuse_idx=idx_owner)
    assert all(np.array_equal(a, b) for a, b in zip(idx_owner, idx_shared))
    ref_o, _ = mla.sparse_mla(shared, small.latent, idx_owner, [len(i) for i in idx_owner])
    assert np.array_equal(out_s, ref_o)


def test_ssmax_factor_one_is_ssmax_off(small):
    v_on = small.view(0)
    n = 300
    v_on.ssmax_s = v_on.ssmax_s_index = 1.0 / math.log(n)
    v_off = small.view(0)
    v_off.ssmax = False
    a = mla.run_layer(v_on, small.latent, small.index_cache, tokens=[0])
    b = mla.run_layer(v_off, small.latent, small.index_cache, tokens=[0])
    assert np.array_equal(a[0][0], b[0][0]) and np.allclose(a[1], b[1], rtol=1e-12)


# --- producers: FP8 quantisation and cache writes ---------------------------------

from oracle import producers as PR  # noqa: E402


def _torch_e4m3(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = F.decode_e4m3(codes).astype(np.float32)
    assert np.array_equal(PR.e4m3_encode(vals), codes)


def test_e4m3_encode_ties_go_to_the_even_code():
    # midpoint between every pair of neighbouring finite magnitudes
    mags = F.decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    mids = ((mags[:-1] + mags[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (mags[:-1] + mags[1:]) / 2)   # exact in fp32
    got = PR.e4m3_encode(mids).astype(int)
    lo = np.arange(0x7E)
    want = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(got, want)
    assert np.array_equal(PR.e4m3_encode(-mids).astype(int), want | 0x80)


def test_e4m3_encode_matches_torch_cast_and_brute_force_nearest():
    rng = synth.stream(5, "e4m3_encode")
    x = (rng.standard_normal(20000) * np.exp2(rng.uniform(-14, 9, 20000))).astype(np.float32)
    x = x[np.abs(x) < 464]                        # torch's cast has no saturation past 464
    got = PR.e4m3_encode(x)
    assert np.array_equal(got, _torch_e4m3(x))
    # brute force over every finite code: the chosen value is a nearest one
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = F.decode_e4m3(finite)
    sub = x[:2000].astype(np.float64)
    best = np.abs(vals[None, :] - sub[:, None]).min(axis=1)
    assert np.array_equal(np.abs(F.decode_e4m3(got[:2000]) - sub), best)


def test_e4m3_encode_saturates_and_keeps_signed_zero():
    x = np.array([448.0, 463.9, 464.0, 1e4, 3e38, -500.0, 0.0, -0.0], dtype=np.float32)
    assert PR.e4m3_encode(x).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x80]


def test_quantise_block_invariants():
    rng = synth.stream(6, "quant_block")
    for scale_exp in (-30, -3, 0, 5, 30):
        x = (rng.standard_normal(128) * 2.0 ** scale_exp).astype(np.float32)
        codes, s = PR.quantise_block(x)
        assert s.dtype == np.float32 and s > 0
        # the block's largest magnitude lands on the largest finite code
        assert codes[np.argmax(np.abs(x))] & 0x7F == 0x7E
        back = F.decode_e4m3(codes) * float(s)
        bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * float(s)) * (1 + 1e-6)
        assert np.all(np.abs(back - x) <= bound)
    codes, s = PR.quantise_block(np.zeros(128, dtype=np.float32))
    assert s == 1.0 and not codes.any()
    codes, s = PR.quantise_block(np.array([-0.0, 0.0], dtype=np.float32))
    assert s == 1.0 and codes.tolist() == [0x80, 0x00]


def test_quantiser_agrees_with_the_torch_based_generator():
    # synth.quantise_rows quantises with PyTorch's cast: an independent implementation
    x = synth.stream(7, "gen_vs_oracle").standard_normal((32, 512), dtype=np.float32)
    gcodes, gscale = synth.quantise_rows(x, 128)
    for i in range(32):
        for b in range(4):
            codes, s = PR.quantise_block(x[i, b * 128:(b + 1) * 128])
            assert s == gscale[i, b]
            assert np.array_equal(codes, gcodes[i, b * 128:(b + 1) * 128])


def test_cache_writes_read_back_through_the_layout_readers():
    rng = synth.stream(8, "writes")
    n, pages = 40, 3
    slot = rng.permutation(pages * 64)[:n].astype(np.int32)
    slot[5] = -1
    c = synth.to_bf16_bits(rng.standard_normal((n, 512)).astype(np.float32))
    kpe = synth.to_bf16_bits(rng.standard_normal((n, 64)).astype(np.float32))
    k = synth.to_bf16_bits(rng.standard_normal((n, 128)).astype(np.float32))
    lat0 = rng.integers(0, 256, pages * F.LATENT_PAGE_BYTES, dtype=np.uint8)
    idx0 = rng.integers(0, 256, pages * F.INDEXER_PAGE_BYTES, dtype=np.uint8)
    lat, bad1 = PR.write_latent(lat0, c, kpe, slot)
    idx, bad2 = PR.write_indexer_k(idx0, k, slot)
    assert not bad1 and not bad2
    w = slot >= 0
    c_hat, pe = F.latent_rows(lat, slot[w] // 64, slot[w] % 64)
    cx = F.decode_bf16(c[w])
    assert np.array_equal(pe, F.decode_bf16(kpe[w]))
    bound = np.maximum(np.abs(cx) * 2.0 ** -4, 2.0 ** -10 * np.abs(cx).reshape(-1, 4, 128).max(2).repeat(128, 1) / 448)
    assert np.all(np.abs(c_hat - cx) <= bound * (1 + 1e-6))
    kh = F.indexer_keys(idx, slot[w] // 64, slot[w] % 64)
    kx = F.decode_bf16(k[w])
    kb = np.maximum(np.abs(kx) * 2.0 ** -4, 2.0 ** -10 * np.abs(kx).max(1, keepdims=True) / 448)
    assert np.all(np.abs(kh - kx) <= kb * (1 + 1e-6))
    # rows of other slots are untouched; the skipped token wrote nothing
    lat_rows = np.zeros(pages * 64, bool)
    lat_rows[slot[w]] = True
    lr = lat.reshape(pages * 64, F.LATENT_ROW_BYTES)
    assert np.array_equal(lr[~lat_rows], lat0.reshape(pages * 64, -1)[~lat_rows])
    keys = idx.reshape(pages, -1)[:, :F.INDEXER_KEYS_BYTES].reshape(pages * 64, 128)
    keys0 = idx0.reshape(pages, -1)[:, :F.INDEXER_KEYS_BYTES].reshape(pages * 64, 128)
    assert np.array_equal(keys[~lat_rows], keys0[~lat_rows])
    # a NoPE row stores a zero RoPE key; an out-of-range slot is reported, not written
    lat2, bad = PR.write_latent(lat0, c[:2], None, np.array([7, pages * 64], dtype=np.int32))
    assert bad
    _, pe2 = F.latent_rows(lat2, [0], [7])
    assert not pe2.any()
    assert np.array_equal(lat2[F.LATENT_ROW_BYTES * 8:], lat0[F.LATENT_ROW_BYTES * 8:])


def test_indexer_q_quantisation_is_one_block_per_token():
    rng = synth.stream(9, "iq")
    iq = synth.to_bf16_bits((rng.standard_normal((3, 64, 128)) * np.array([1e-3, 1.0, 50.0])[:, None, None])
                            .astype(np.float32))
    codes, scales = PR.quantise_indexer_q(iq)
    x = F.decode_bf16(iq)
    for t in range(3):
        assert scales[t] == np.float32(np.float32(np.abs(x[t]).max()) / np.float32(448))
        assert (codes[t] & 0x7F).max() == 0x7E
        back = F.decode_e4m3(codes[t]) * float(scales[t])
        assert np.all(np.abs(back - x[t]) <= np.maximum(np.abs(x[t]) * 2.0 ** -4, 2.0 ** -10 * float(scales[t])) * (1 + 1e-6))


# --- the plain per-tensor E4M3 latent format (576 B per token) --------------------

def test_plain_e4m3_row_layout_from_independent_packing():
    g = golden()
    assert F.PLAIN_E4M3_ROW_BYTES == g["latent_row_plain_e4m3"] == 576
    pool = bytearray(2 * 64 * 576)
    page, row = 1, 21
    codes = bytes((0x08 + 3 * i) % 0x7E for i in range(576))
    off = page * 64 * 576 + row * 576
    pool[off: off + 576] = codes
    c, pe = F.plain_e4m3_rows(F.PlainE4M3Pool(np.frombuffer(bytes(pool), dtype=np.uint8), 0.375), [page], [row])
    assert c.shape == (1, 512) and pe.shape == (1, 64)
    assert all(c[0, d] == F.e4m3_value(codes[d]) * 0.375 for d in range(512))
    assert all(pe[0, d] == F.e4m3_value(codes[512 + d]) * 0.375 for d in range(64))


def test_plain_pool_gives_the_attention_of_an_equal_fp8_ds_mla_pool(small):
    """Values that both formats hold exactly (every block scale equal to the
    power-of-two pool scale, RoPE keys that are E4M3 values times it) give
    identical rows and identical attention through the two readers."""
    wl = small
    s = 2.0 ** -5
    rng = synth.stream(10, "plain_vs_ds")
    n_rows = wl.num_pages * 64
    codes = rng.integers(0, 0x7F, size=(n_rows, 576), dtype=np.uint8) | (rng.integers(0, 2, (n_rows, 576)) << 7).astype(np.uint8)
    plain = F.PlainE4M3Pool(codes.reshape(-1), s)
    ds = np.zeros((n_rows, F.LATENT_ROW_BYTES), dtype=np.uint8)
    ds[:, :512] = codes[:, :512]
    ds[:, 512:528] = np.full((n_rows, 4), s, dtype="<f4").view(np.uint8)
    pe = (F.decode_e4m3(codes[:, 512:]) * s).astype(np.float32)
    ds[:, 528:] = synth.to_bf16_bits(pe).astype("<u2").view(np.uint8).reshape(n_rows, 128)
    assert np.array_equal(F.decode_bf16(synth.to_bf16_bits(pe)), pe.astype(np.float64))   # exact in bf16
    ds = ds.reshape(-1)
    pages = np.arange(wl.num_pages).repeat(64)
    rows = np.tile(np.arange(64), wl.num_pages)
    c1, p1 = F.latent_rows(plain, pages, rows)
    c2, p2 = F.latent_rows(ds, pages, rows)
    assert np.array_equal(c1, c2) and np.array_equal(p1, p2)
    v = wl.view(0)
    T = wl.T
    idx = np.tile(np.arange(64), (T, 1))
    ln = np.minimum(64, dsa.visible_lengths(wl.cu_q, wl.ctx_len))
    o1, l1 = mla.sparse_mla(v, plain, idx, ln)
    o2, l2 = mla.sparse_mla(v, ds, idx, ln)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_plain_e4m3_writer_round_trip_and_untouched_rows():
    rng = synth.stream(11, "plain_writer")
    pages, n = 2, 30
    slot = synth.producer_slots(11, "plain_writer/slot", n, pages, 7)
    c = synth.to_bf16_bits(rng.standard_normal((n, 512)).astype(np.float32))
    kpe = synth.to_bf16_bits(rng.standard_normal((n, 64)).astype(np.float32))
    s = 6.0 / 448.0
    pool0 = F.PlainE4M3Pool(rng.integers(0, 256, pages * F.PLAIN_E4M3_PAGE_BYTES, dtype=np.uint8), s)
    pool, bad = PR.write_latent_plain_e4m3(pool0, c, kpe, slot)
    assert not bad and pool.scale == np.float32(s)
    w = slot >= 0
    ch, ph = F.plain_e4m3_rows(pool, slot[w] // 64, slot[w] % 64)
    for got, want in ((ch, F.decode_bf16(c[w])), (ph, F.decode_bf16(kpe[w]))):
        inside = np.abs(want) <= 448 * np.float32(s)
        bound = np.maximum(np.abs(want) * 2.0 ** -4, 2.0 ** -10 * float(np.float32(s))) * (1 + 1e-6)
        assert np.all(np.abs(got - want)[inside] <= bound[inside])
        # outside the range the code saturates at +-448 s
        assert np.all(np.abs(got[~inside]) == 448 * float(np.float32(s)))
    touched = np.zeros(pages * 64, bool)
    touched[slot[w]] = True
    a = pool.data.reshape(pages * 64, 576)
    b = pool0.data.reshape(pages * 64, 576)
    assert np.array_equal(a[~touched], b[~touched])
    nope, _ = PR.write_latent_plain_e4m3(pool0, c[:1], None, np.array([3], dtype=np.int32))
    assert not nope.data[3 * 576 + 512: 4 * 576].any()


# --- decode context parallelism: the cache sharded by token over ranks ----------------

from oracle import dcp  # noqa: E402


def _dcp_rows():
    rng = np.random.default_rng(12)
    vals = np.array([-1.5, -0.0, 0.0, 0.25, 2.0, np.inf, -np.inf, np.nan], dtype=np.float32)
    rows = [rng.choice(vals, size=n).astype(np.float32) for n in (1, 9, 300, 5000)]
    rows.append(np.zeros(3000, dtype=np.float32))                              # ties across every rank
    rows.append(np.round(rng.standard_normal(7000) * 3).astype(np.float32))    # heavy ties
    rows.append(rng.standard_normal(20000).astype(np.float32))
    return rows


@pytest.mark.parametrize("R,I", [(1, 1), (2, 1), (3, 1), (8, 1), (2, 64), (8, 64), (5, 100)])
def test_dcp_selection_is_the_unsharded_topk(R, I):
    for row in _dcp_rows():
        for k in (1, 7, 64, 2048):
            got = dcp.select(row, R, I, k)
            assert np.array_equal(got, dsa.topk_row(row, k)), (R, I, k, len(row))


def test_dcp_candidates_hold_the_global_topk_and_at_most_k_each():
    row = np.round(np.random.default_rng(13).standard_normal(9000) * 2).astype(np.float32)
    k = 700
    want = set(dsa.topk_row(row, k).tolist())
    union = set()
    for r in range(4):
        s, p = dcp.rank_candidates(row, r, 4, 1, k)
        assert len(p) <= k and np.all(dcp.owner(p, 4, 1) == r)
        assert np.array_equal(s, row[p])
        union |= set(p.tolist())
    assert want <= union


def test_dcp_attention_is_the_unsharded_sparse_mla(small):
    wl = small
    v = wl.view(0)
    scores = dsa.indexer_scores(v, v.iq8, v.iq_scale, v.iw, wl.index_cache)
    for R, I in ((2, 1), (3, 64), (8, 64)):
        for t in range(wl.T):
            sel = dcp.select(scores[t], R, I, wl.topk)
            assert np.array_equal(sel, dsa.topk_row(scores[t], wl.topk))
            out, lse, per_rank = dcp.attention(v, wl.latent, t, sel, R, I)
            ref_o, ref_l = mla.token_attention(v, wl.latent, t, sel)
            assert np.allclose(out, ref_o, rtol=1e-12, atol=1e-12)
            assert np.allclose(lse, ref_l, rtol=1e-12, atol=1e-12)
            # a rank holding none of the selected tokens has an empty row
            holders = set(dcp.owner(sel, R, I).tolist())
            for r in range(R):
                assert (r in holders) == bool(np.all(np.isfinite(per_rank[r])))


# --- the bf16 latent pool (1,152 B per token) ----------------------------------------

def test_bf16_row_layout_from_independent_packing():
    assert F.BF16_ROW_BYTES == 1152
    vals = [((i * 37) % 255 - 127) / 16.0 for i in range(576)]   # at most 7 significant bits: exact in bf16
    raw = b"".join(struct.pack("<f", v)[2:] for v in vals)      # bf16 = top half of the fp32
    pool = bytearray(2 * 64 * 1152)
    page, row = 1, 5
    off = page * 64 * 1152 + row * 1152
    pool[off: off + 1152] = raw
    c, pe = F.bf16_rows(F.Bf16Pool(np.frombuffer(bytes(pool), dtype=np.uint8)), [page], [row])
    assert np.array_equal(c[0], np.array(vals[:512])) and np.array_equal(pe[0], np.array(vals[512:]))


def test_bf16_pool_gives_the_attention_of_an_equal_fp8_ds_mla_pool(small):
    """E4M3 codes times a power-of-two block scale are bf16 values, so a bf16
    pool can hold exactly the rows of an fp8_ds_mla pool: same rows, same
    attention."""
    wl = small
    n_rows = wl.num_pages * 64
    pages = np.arange(wl.num_pages).repeat(64)
    rows = np.tile(np.arange(64), wl.num_pages)
    rng = synth.stream(14, "bf16_vs_ds")
    codes = (rng.integers(0, 0x7F, size=(n_rows, 512)) | (rng.integers(0, 2, (n_rows, 512)) << 7)).astype(np.uint8)
    scale = np.float32(2.0 ** -6)
    ds = np.zeros((n_rows, F.LATENT_ROW_BYTES), dtype=np.uint8)
    ds[:, :512] = codes
    ds[:, 512:528] = np.full((n_rows, 4), scale, dtype="<f4").view(np.uint8)
    pe_bits = synth.to_bf16_bits(rng.standard_normal((n_rows, 64)).astype(np.float32))
    ds[:, 528:] = pe_bits.astype("<u2").view(np.uint8).reshape(n_rows, 128)
    c_vals = (F.decode_e4m3(codes) * float(scale)).astype(np.float32)
    c_bits = synth.to_bf16_bits(c_vals)
    assert np.array_equal(F.decode_bf16(c_bits), c_vals.astype(np.float64))      # exact in bf16
    b16, bad = PR.write_latent_bf16(F.Bf16Pool(np.zeros(wl.num_pages * F.BF16_PAGE_BYTES, np.uint8)),
                                    c_bits, pe_bits, np.arange(n_rows, dtype=np.int32))
    assert not bad
    c1, p1 = F.latent_rows(b16, pages, rows)
    c2, p2 = F.latent_rows(ds.reshape(-1), pages, rows)
    assert np.array_equal(c1, c2) and np.array_equal(p1, p2)
    v = wl.view(0)
    idx = np.tile(np.arange(64), (wl.T, 1))
    ln = np.minimum(64, dsa.visible_lengths(wl.cu_q, wl.ctx_len))
    o1, l1 = mla.sparse_mla(v, b16, idx, ln)
    o2, l2 = mla.sparse_mla(v, ds.reshape(-1), idx, ln)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
