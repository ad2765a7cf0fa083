"""Byte formats that the sparse-MLA decode step reads, decoded in float64.

TEST INFRASTRUCTURE ONLY.  This module belongs to the CPU oracle: it may be
imported by ``tests/``, by ``__graft_entry__.smoke()`` and by the CPU-baseline
leg of ``bench.py``, and by nothing else.  It shares no code with the CUDA
library.

Sources (web pages on vLLM's Mistral Large 4 support):

* vLLM blog, "vLLM 首日支持 Mistral Large 4：1T 参数 MoE 多模态模型"
  (day-0 support for Mistral Large 4), section "实现细节 / 模型架构"
  (implementation details / model architecture), paragraph "稀疏 MLA + DSA
  indexer": the default latent cache is ``fp8_ds_mla``; a token costs 47,136 B
  of KV cache, 41,328 B of MLA latent and 5,808 B of indexer keys.
* same blog, section "ROCm 实现细节" (ROCm implementation details), paragraphs
  "AITER 上的 DSA 索引器" and "FP8 潜在缓存": an indexer key is quantised to
  FP8 with a single scale and costs 132 B per token per indexer layer;
  ``fp8_ds_mla`` costs 656 B per token per layer, against 576 B for a plain
  per-tensor E4M3 cache and 1,152 B for bf16; 63 layers own a cache.
* the model architecture paragraph (highlights list): KV LoRA rank 512,
  RoPE dim 64; top 2048 keys per query.

Readings where the pages print only byte totals (the pages give no layout):

* latent row, 656 B = [512 x e4m3 latent][4 x fp32 scale, one per 128-element
  block][64 x bf16 RoPE key]; a page holds 64 such rows back to back;
* indexer page = [64 rows x 128 B e4m3 key][64 x fp32 per-token scale],
  i.e. 132 B per token;
* all multi-byte values little-endian.

FP8 E4M3 here is the OCP 8-bit floating point "E4M3" encoding (the one
PyTorch calls ``float8_e4m3fn``): 1 sign bit, 4 exponent bits with bias 7,
3 mantissa bits, subnormals when the exponent field is 0, no infinities, and
NaN only for exponent and mantissa fields all ones.
"""
from __future__ import annotations

from typing import NamedTuple

import numpy as np

# --- sizes fixed by the pages -------------------------------------------------
PAGE_TOKENS = 64            # 64-token cache blocks (blog, DSpark / DCP paragraphs)
LATENT_DIM = 512            # KV LoRA rank
ROPE_DIM = 64               # RoPE dim of the MLA key
SCALE_BLOCK = 128           # one fp32 scale per 128 latent elements
N_SCALE = LATENT_DIM // SCALE_BLOCK
INDEXER_HEADS = 64
INDEXER_DIM = 128

# --- derived byte layout (reading above) --------------------------------------
LATENT_ROW_BYTES = LATENT_DIM * 1 + N_SCALE * 4 + ROPE_DIM * 2      # 656
LATENT_PAGE_BYTES = PAGE_TOKENS * LATENT_ROW_BYTES                  # 41,984
INDEXER_ROW_BYTES = INDEXER_DIM * 1 + 4                             # 132
INDEXER_KEYS_BYTES = PAGE_TOKENS * INDEXER_DIM                      # 8,192
INDEXER_PAGE_BYTES = PAGE_TOKENS * INDEXER_ROW_BYTES                # 8,448
PLAIN_E4M3_ROW_BYTES = (LATENT_DIM + ROPE_DIM) * 1                  # 576
BF16_ROW_BYTES = (LATENT_DIM + ROPE_DIM) * 2                        # 1,152


def e4m3_value(code: int) -> float:
    """Value of one OCP E4M3 code, from the format definition."""
    sign = -1.0 if code & 0x80 else 1.0
    exp_field = (code >> 3) & 0xF
    mant = code & 0x7
    if exp_field == 0xF and mant == 0x7:
        return float("nan")
    if exp_field == 0:
        return sign * (mant / 8.0) * 2.0 ** (1 - 7)
    return sign * (1.0 + mant / 8.0) * 2.0 ** (exp_field - 7)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """float64 values of an array of E4M3 codes (uint8)."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """float64 values of bfloat16 bit patterns (uint16): the top half of a float32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):          # NaN patterns stay NaN
        return b.view(np.float32).astype(np.float64)


def _le_f32(raw: np.ndarray) -> np.ndarray:
    """float64 values of little-endian fp32 numbers stored as [..., 4*k] bytes."""
    raw = np.ascontiguousarray(raw, dtype=np.uint8)
    return raw.view("<f4").astype(np.float64)


def latent_rows(cache, pages: np.ndarray, rows: np.ndarray):
    """Read latent rows (physical page, row in page) from an fp8_ds_mla pool
    (uint8 bytes), a ``PlainE4M3Pool`` or a ``Bf16Pool``.

    Returns (c_hat [n, 512] = e4m3 * block scale, k_pe [n, 64]) in float64.
    """
    if isinstance(cache, PlainE4M3Pool):
        return plain_e4m3_rows(cache, pages, rows)
    if isinstance(cache, Bf16Pool):
        return bf16_rows(cache, pages, rows)
    pages = np.asarray(pages, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    start = pages * LATENT_PAGE_BYTES + rows * LATENT_ROW_BYTES
    raw = cache[start[:, None] + np.arange(LATENT_ROW_BYTES)[None, :]]
    nope = decode_e4m3(raw[:, :LATENT_DIM])
    scales = _le_f32(raw[:, LATENT_DIM:LATENT_DIM + 4 * N_SCALE])          # [n, 4]
    c_hat = nope * np.repeat(scales, SCALE_BLOCK, axis=1)
    pe_raw = np.ascontiguousarray(raw[:, LATENT_DIM + 4 * N_SCALE:])
    k_pe = decode_bf16(pe_raw.view("<u2"))
    return c_hat, k_pe


def indexer_keys(cache: np.ndarray, pages: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """Read dequantised indexer keys k = e4m3 * per-token scale, [n, 128] float64."""
    pages = np.asarray(pages, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    kstart = pages * INDEXER_PAGE_BYTES + rows * INDEXER_DIM
    codes = cache[kstart[:, None] + np.arange(INDEXER_DIM)[None, :]]
    sstart = pages * INDEXER_PAGE_BYTES + INDEXER_KEYS_BYTES + rows * 4
    scale = _le_f32(cache[sstart[:, None] + np.arange(4)[None, :]])[:, 0]
    return decode_e4m3(codes) * scale[:, None]


PLAIN_E4M3_PAGE_BYTES = PAGE_TOKENS * PLAIN_E4M3_ROW_BYTES          # 36,864


class PlainE4M3Pool(NamedTuple):
    """A latent pool in the plain per-tensor E4M3 format (blog, section "ROCm
    实现细节", paragraph "FP8 潜在缓存": all 576 latent dims stored as FP8 with
    one per-tensor scale, 576 B per token).  Reading: a row is [512 x e4m3
    latent][64 x e4m3 RoPE key], a page 64 rows back to back, and ``scale``
    the pool's fp32 scale."""
    data: np.ndarray
    scale: float


BF16_PAGE_BYTES = PAGE_TOKENS * BF16_ROW_BYTES                       # 73,728


class Bf16Pool(NamedTuple):
    """A latent pool in bf16 (blog, section "ROCm 实现细节", paragraph "FP8 潜在
    缓存": 1,152 B per token per layer in bf16).  Reading: a row is [512 x bf16
    latent][64 x bf16 RoPE key], little-endian, a page 64 rows back to back."""
    data: np.ndarray


def bf16_rows(pool: Bf16Pool, pages: np.ndarray, rows: np.ndarray):
    """Read latent rows from a bf16 pool: (c_hat [n, 512], k_pe [n, 64]) in float64."""
    pages = np.asarray(pages, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    start = pages * BF16_PAGE_BYTES + rows * BF16_ROW_BYTES
    raw = pool.data[start[:, None] + np.arange(BF16_ROW_BYTES)[None, :]]
    v = decode_bf16(np.ascontiguousarray(raw).view("<u2"))
    return v[:, :LATENT_DIM], v[:, LATENT_DIM:]


def plain_e4m3_rows(pool: PlainE4M3Pool, pages: np.ndarray, rows: np.ndarray):
    """Read latent rows from a plain E4M3 pool: (c_hat [n, 512], k_pe [n, 64]),
    every code times the pool scale, in float64."""
    pages = np.asarray(pages, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    start = pages * PLAIN_E4M3_PAGE_BYTES + rows * PLAIN_E4M3_ROW_BYTES
    raw = pool.data[start[:, None] + np.arange(PLAIN_E4M3_ROW_BYTES)[None, :]]
    v = decode_e4m3(raw) * float(np.float32(pool.scale))
    return v[:, :LATENT_DIM], v[:, LATENT_DIM:]


def physical(block_table_row: np.ndarray, positions: np.ndarray):
    """Logical token positions of one request -> (physical page, row in page)."""
    positions = np.asarray(positions, dtype=np.int64)
    return block_table_row[positions // PAGE_TOKENS].astype(np.int64), positions % PAGE_TOKENS
