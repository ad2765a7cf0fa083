"""Comparison of the CUDA path with the float64 oracle, under the agreement rules:

* indexer scores: |gpu - oracle| <= 1e-4 * A + 1e-30, A = c_t * sum_h |w_h| *
  ReLU(q_h . k_s) (the size of the summed terms: a relative rule on each score
  would be meaningless where the weighted sum cancels to ~0);
* top-k: the GPU's positions equal, bit for bit, the oracle's selection applied
  to the GPU's own score row (ties to the lower position), len = min(K, n_t),
  padding -1;
* attention: max |gpu - oracle| <= 2e-3 * RMS(oracle) over the whole output of
  the case, computed by the oracle over the GPU's own selected positions; lse
  within 2e-3 absolute (a relative error of 2e-3 on the softmax sum).
"""
from __future__ import annotations

import numpy as np

from oracle import dsa, formats, mla

SCORE_REL = 1e-4
OUT_RMS_REL = 2e-3
LSE_ABS = 2e-3


def oracle_latent(wl):
    """The workload's latent pool as the oracle reads it."""
    if wl.latent_format == "e4m3":
        return formats.PlainE4M3Pool(wl.latent, wl.latent_scale)
    if wl.latent_format == "bf16":
        return formats.Bf16Pool(wl.latent)
    return wl.latent


def check_scores(wl, layer_i, scores_gpu, tokens=None, sample=None, seed=0):
    """Compare GPU score rows with the oracle; ``sample`` = positions per row (None: all)."""
    v = wl.view(layer_i)
    req = dsa.request_of_tokens(wl.cu_q)
    n_all = dsa.visible_lengths(wl.cu_q, wl.ctx_len)
    tokens = range(wl.T) if tokens is None else tokens
    rng = np.random.default_rng(seed)
    worst = 0.0
    for t in tokens:
        n = int(n_all[t])
        if sample is None or sample >= n:
            pos = np.arange(n)
        else:  # both ends of the row, page edges and random interior positions
            edge = np.array([0, 1, 63, 64, 127, 128, n - 129, n - 65, n - 64, n - 2, n - 1])
            pos = np.unique(np.concatenate([edge[(edge >= 0) & (edge < n)], rng.integers(0, n, sample)]))
        c = dsa.ssmax_factor(v.ssmax, v.ssmax_s_index, n)
        ref, mag = dsa.indexer_scores_row(v.iq8[t], v.iq_scale[t], v.iw[t], wl.index_cache,
                                          wl.block_table[req[t]], n, c, positions=pos,
                                          with_magnitude=True)
        got = scores_gpu[t, pos].astype(np.float64)
        err = np.abs(got - ref)
        bad = err > SCORE_REL * mag + 1e-30
        assert not bad.any(), (f"token {t}: {bad.sum()} scores off, e.g. pos {pos[bad][:5]} "
                               f"got {got[bad][:3]} want {ref[bad][:3]} mag {mag[bad][:3]}")
        worst = max(worst, float((err / np.maximum(mag, 1e-30)).max()))
    return worst


def check_topk(wl, scores_gpu, idx_gpu, len_gpu, tokens=None):
    n_all = dsa.visible_lengths(wl.cu_q, wl.ctx_len)
    tokens = range(wl.T) if tokens is None else tokens
    K = wl.topk
    for t in tokens:
        n = int(n_all[t])
        want = dsa.topk_row(scores_gpu[t, :n], K)
        ln = int(len_gpu[t])
        assert ln == min(K, n), f"token {t}: len {ln} != {min(K, n)}"
        got = idx_gpu[t, :ln].astype(np.int64)
        assert np.array_equal(got, want), f"token {t}: top-k differs at {np.nonzero(got != want)[0][:5]}"
        assert np.all(idx_gpu[t, ln:] == -1), f"token {t}: padding not -1"


def check_attention(wl, layer_i, idx_gpu, len_gpu, out_gpu, lse_gpu, tokens=None):
    v = wl.view(layer_i)
    tokens = list(range(wl.T)) if tokens is None else list(tokens)
    ref_o, ref_l = mla.sparse_mla(v, oracle_latent(wl), idx_gpu, len_gpu, tokens=tokens)
    got_o = out_gpu[tokens].astype(np.float64)
    got_l = lse_gpu[tokens].astype(np.float64)
    rms = float(np.sqrt(np.mean(ref_o ** 2)))
    err = float(np.abs(got_o - ref_o).max())
    assert err <= OUT_RMS_REL * rms, f"attention max-abs error {err:.3e} > {OUT_RMS_REL} * RMS {rms:.3e}"
    fin = np.isfinite(ref_l)
    assert np.array_equal(fin, np.isfinite(got_l)), "lse finiteness differs"
    lerr = float(np.abs(got_l[fin] - ref_l[fin]).max()) if fin.any() else 0.0
    assert lerr <= LSE_ABS, f"lse error {lerr:.3e}"
    return err / rms, lerr
