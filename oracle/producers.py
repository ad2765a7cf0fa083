"""The producers just before the decode step: FP8 quantisation of new tokens'
indexer keys, latent rows and indexer queries, and the writes into the paged
caches that the step then reads.

TEST INFRASTRUCTURE ONLY.  This module belongs to the CPU oracle: it may be
imported by ``tests/``, by ``__graft_entry__.smoke()`` and by the CPU-baseline
leg of ``bench.py``, and by nothing else.  It shares no code with the CUDA
library.

Sources (web pages on vLLM's Mistral Large 4 support):

* vLLM blog, "vLLM 首日支持 Mistral Large 4：1T 参数 MoE 多模态模型", paragraph
  "可断开的 CUDA 图和融合" (breakable CUDA graphs and fusions): the first round
  of hand-written fusions covers the indexer Q path and the indexer K path;
  the decode round writes the indexer K straight into the FP8 cache;
* same blog, section "实现细节 / 模型架构", paragraph "稀疏 MLA + DSA indexer":
  the latent cache is ``fp8_ds_mla`` and the indexer cache is FP8;
* same blog, section "ROCm 实现细节", paragraph "AITER 上的 DSA 索引器": one
  FP8 scale per indexer key, 132 B per token.

Readings (the pages print no quantiser):

* a block of values x is stored as E4M3 codes of q = x / s with
  s = amax|x| / 448 (s = 1 when amax is 0); 448 is the largest finite E4M3
  value, so the block's largest magnitude lands on it;
* the blocks are: 128 latent values (four per fp8_ds_mla row), one 128-value
  indexer key, and one query token's 64 x 128 indexer values;
* every code is the E4M3 value nearest to q, ties to the even code, and
  magnitudes beyond 448 clamp to 448 (no NaN from finite inputs);
* s and q are computed in float32 (bf16 inputs widen exactly): here floating
  point decides an integer code, so the oracle takes that decision in the
  precision the kernels use; the E4M3 rounding itself is exact arithmetic on
  those float32 values;
* a new token goes to slot = physical page * 64 + row; slot -1 skips the
  token; any other slot outside [0, pages * 64) is skipped and reported;
* the RoPE key of a latent row is stored as given (bf16 bits); a NoPE layer
  passes none and its 128 B are zero.

Byte layouts: those of ``formats`` (fp8_ds_mla row [512 x e4m3][4 x fp32]
[64 x bf16]; plain E4M3 row [576 x e4m3] under one pool scale that the caller
gives; bf16 row [576 x bf16]; indexer page [64 x 128 B keys][64 x fp32
scales]).
"""
from __future__ import annotations

import numpy as np

from . import formats as F

E4M3_MAX = 448.0

# The 127 finite non-negative E4M3 magnitudes in code order (0x00 .. 0x7E);
# codes and magnitudes increase together.
_MAGS = np.array([F.e4m3_value(c) for c in range(0x7F)], dtype=np.float64)


def e4m3_encode(q: np.ndarray) -> np.ndarray:
    """E4M3 codes (uint8) of finite float32 values: nearest value, ties to the
    even code, magnitudes past 448 clamped to 448, sign kept (-0 -> 0x80)."""
    q = np.asarray(q, dtype=np.float32)
    a = np.abs(q.astype(np.float64)).ravel()
    hi = np.clip(np.searchsorted(_MAGS, a, side="left"), 1, len(_MAGS) - 1)
    lo = hi - 1
    d_lo = a - _MAGS[lo]
    d_hi = _MAGS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= E4M3_MAX, 0x7E, code)
    code = np.where(a == 0.0, 0, code)
    sign = np.signbit(q).ravel().astype(np.int64) << 7
    return (code | sign).astype(np.uint8).reshape(q.shape)


def quantise_block(x: np.ndarray):
    """One block (any shape) of float32 values -> (codes like x, float32 scale)."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.abs(x).max()) if x.size else np.float32(0)
    scale = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
    q = (x / scale).astype(np.float32)
    return e4m3_encode(q), scale


def _slots(slot: np.ndarray, num_pages: int):
    """Split slots into (token ids to write, pages, rows, any slot out of range)."""
    slot = np.asarray(slot, dtype=np.int64)
    ok = (slot >= 0) & (slot < num_pages * F.PAGE_TOKENS)
    bad = bool(((slot != -1) & ~ok).any())
    ids = np.nonzero(ok)[0]
    return ids, slot[ids] // F.PAGE_TOKENS, slot[ids] % F.PAGE_TOKENS, bad


def write_indexer_k(cache: np.ndarray, k_bits: np.ndarray, slot: np.ndarray):
    """Quantise indexer keys (bf16 bits [n, 128]) into a copy of an indexer
    pool.  Returns (new pool bytes, any slot out of range)."""
    out = np.array(cache, dtype=np.uint8, copy=True)
    num_pages = out.size // F.INDEXER_PAGE_BYTES
    ids, pages, rows, bad = _slots(slot, num_pages)
    k = F.decode_bf16(k_bits).astype(np.float32)
    for i, p, r in zip(ids, pages, rows):
        codes, s = quantise_block(k[i])
        base = p * F.INDEXER_PAGE_BYTES
        out[base + r * F.INDEXER_DIM: base + (r + 1) * F.INDEXER_DIM] = codes
        so = base + F.INDEXER_KEYS_BYTES + r * 4
        out[so: so + 4] = np.frombuffer(np.float32(s).astype("<f4").tobytes(), dtype=np.uint8)
    return out, bad


def write_latent(cache: np.ndarray, c_bits: np.ndarray, kpe_bits, slot: np.ndarray):
    """Quantise latent rows (bf16 bits [n, 512]) with their RoPE keys (bf16
    bits [n, 64], or None for a NoPE layer) into a copy of an fp8_ds_mla pool.
    Returns (new pool bytes, any slot out of range)."""
    out = np.array(cache, dtype=np.uint8, copy=True)
    num_pages = out.size // F.LATENT_PAGE_BYTES
    ids, pages, rows, bad = _slots(slot, num_pages)
    c = F.decode_bf16(c_bits).astype(np.float32)
    for i, p, r in zip(ids, pages, rows):
        row = np.zeros(F.LATENT_ROW_BYTES, dtype=np.uint8)
        scales = np.zeros(F.N_SCALE, dtype="<f4")
        for b in range(F.N_SCALE):
            blk = slice(b * F.SCALE_BLOCK, (b + 1) * F.SCALE_BLOCK)
            row[blk], scales[b] = quantise_block(c[i, blk])
        row[F.LATENT_DIM: F.LATENT_DIM + 4 * F.N_SCALE] = scales.view(np.uint8)
        if kpe_bits is not None:
            pe = np.ascontiguousarray(np.asarray(kpe_bits[i], dtype="<u2"))
            row[F.LATENT_DIM + 4 * F.N_SCALE:] = pe.view(np.uint8)
        start = p * F.LATENT_PAGE_BYTES + r * F.LATENT_ROW_BYTES
        out[start: start + F.LATENT_ROW_BYTES] = row
    return out, bad


def quantise_indexer_q(iq_bits: np.ndarray):
    """Indexer queries (bf16 bits [T, 64, 128]) -> (E4M3 codes [T, 64, 128],
    float32 scales [T]), one block per query token."""
    iq = F.decode_bf16(iq_bits).astype(np.float32)
    codes = np.empty(iq.shape, dtype=np.uint8)
    scales = np.empty(iq.shape[0], dtype=np.float32)
    for t in range(iq.shape[0]):
        codes[t], scales[t] = quantise_block(iq[t])
    return codes, scales


def write_latent_plain_e4m3(pool: F.PlainE4M3Pool, c_bits: np.ndarray, kpe_bits, slot: np.ndarray):
    """Latent rows (bf16 bits [n, 512]) and RoPE keys (bf16 bits [n, 64], or
    None: zero codes) into a copy of a plain E4M3 pool: every value's code is
    that of fp32(x) / scale, with the pool's given per-tensor scale (blog,
    section "ROCm 实现细节", paragraph "FP8 潜在缓存").  Returns (new pool, any
    slot out of range)."""
    out = np.array(pool.data, dtype=np.uint8, copy=True)
    num_pages = out.size // F.PLAIN_E4M3_PAGE_BYTES
    ids, pages, rows, bad = _slots(slot, num_pages)
    s = np.float32(pool.scale)
    c = F.decode_bf16(c_bits).astype(np.float32)
    pe = F.decode_bf16(kpe_bits).astype(np.float32) if kpe_bits is not None else None
    for i, p, r in zip(ids, pages, rows):
        row = np.zeros(F.PLAIN_E4M3_ROW_BYTES, dtype=np.uint8)
        row[:F.LATENT_DIM] = e4m3_encode((c[i] / s).astype(np.float32))
        if pe is not None:
            row[F.LATENT_DIM:] = e4m3_encode((pe[i] / s).astype(np.float32))
        start = p * F.PLAIN_E4M3_PAGE_BYTES + r * F.PLAIN_E4M3_ROW_BYTES
        out[start: start + F.PLAIN_E4M3_ROW_BYTES] = row
    return F.PlainE4M3Pool(out, float(s)), bad


def write_latent_bf16(pool: F.Bf16Pool, c_bits: np.ndarray, kpe_bits, slot: np.ndarray):
    """Latent rows (bf16 bits [n, 512]) and RoPE keys (bf16 bits [n, 64], or
    None: zeros) into a copy of a bf16 pool, stored as given.  Returns (new
    pool, any slot out of range)."""
    out = np.array(pool.data, dtype=np.uint8, copy=True)
    num_pages = out.size // F.BF16_PAGE_BYTES
    ids, pages, rows, bad = _slots(slot, num_pages)
    for i, p, r in zip(ids, pages, rows):
        row = np.zeros(F.LATENT_DIM + F.ROPE_DIM, dtype="<u2")
        row[:F.LATENT_DIM] = np.asarray(c_bits[i], dtype=np.uint16)
        if kpe_bits is not None:
            row[F.LATENT_DIM:] = np.asarray(kpe_bits[i], dtype=np.uint16)
        start = p * F.BF16_PAGE_BYTES + r * F.BF16_ROW_BYTES
        out[start: start + F.BF16_ROW_BYTES] = row.view(np.uint8)
    return F.Bf16Pool(out), bad
