"""Seeded synthetic workloads for the sparse-MLA decode step.

This module only draws random numbers and packs them into the cache byte
layouts that the library reads (see ``include/sml.h``); it holds none of the
step's arithmetic.  Tests, ``bench.py`` and the CPU oracle all take their
inputs from here.

Value distributions (one per tensor, each from its own named PCG64 stream):

* MLA query, bf16 N(0, 1), [T, H, 512 + rope_dim];
* latent rows: 512 values N(0, 1) quantised to FP8 E4M3 with one fp32 scale
  per 128-element block (scale = amax / 448), RoPE key bf16 N(0, 1);
* indexer keys N(0, 1), FP8 E4M3 with one fp32 scale per token (amax / 448);
* indexer queries N(0, 1), FP8 E4M3 with one fp32 scale per query token
  (amax over its 64 x 128 values / 448); head weights N(0, 1) / 8;
* block tables: identity, or a random permutation of a shared page pool;
* rows of a request's last page past its length hold random bytes, which no
  correct reader ever looks at.

FP8 rounding (round to nearest even, saturating at 448) and bf16 rounding use
PyTorch's CPU casts.
"""
from __future__ import annotations

import math
import os
import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from types import SimpleNamespace

import numpy as np
import torch

PAGE = 64
LATENT_ROW = 656
LATENT_PAGE = PAGE * LATENT_ROW
PLAIN_ROW = 576                      # plain per-tensor E4M3 latent row
PLAIN_PAGE = PAGE * PLAIN_ROW
BF16_ROW = 1152                      # bf16 latent row: 512 latent + 64 RoPE values
BF16_PAGE = PAGE * BF16_ROW
PLAIN_SCALE = 8.0 / 448.0            # pool scale of plain E4M3 latents: N(0, 1) values within +-8
INDEX_PAGE = PAGE * 132
E4M3_MAX = 448.0


def stream(seed: int, name: str) -> np.random.Generator:
    """Independent PCG64 stream for (seed, name)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, zlib.crc32(name.encode())])))


def to_e4m3(x: np.ndarray) -> np.ndarray:
    """Round float32 values (|x| <= 448 after clamping) to E4M3 codes (uint8)."""
    t = torch.from_numpy(np.clip(x, -E4M3_MAX, E4M3_MAX).astype(np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def quantise_rows(x: np.ndarray, block: int):
    """Per-block E4M3 quantisation of [n, d] float32: returns (codes, scales [n, d/block])."""
    n, d = x.shape
    xb = x.reshape(n, d // block, block)
    amax = np.abs(xb).max(axis=2)
    scale = np.where(amax > 0, amax / E4M3_MAX, 1.0).astype(np.float32)
    codes = to_e4m3((xb / scale[:, :, None]).reshape(n, d))
    return codes, scale


@dataclass
class Layer:
    """Per-layer query inputs.  ``reuse_from`` names the layer whose top-k a
    shared-indexer layer reuses (its indexer inputs are then None)."""
    rope_dim: int
    q: np.ndarray                       # uint16 bf16 bits [T, H, 512 + rope_dim]
    iq8: np.ndarray | None = None       # uint8 E4M3 [T, 64, 128]
    iq_scale: np.ndarray | None = None  # float32 [T]
    iw: np.ndarray | None = None        # float32 [T, 64]
    reuse_from: int | None = None
    name: str = ""                      # the layer's tag in its workload ("rope", "nope", ...)


@dataclass
class Workload:
    name: str
    num_heads: int
    topk: int
    cu_q: np.ndarray          # int32 [B + 1]
    ctx_len: np.ndarray       # int32 [B]
    block_table: np.ndarray   # int32 [B, max_pages]
    num_pages: int
    latent: np.ndarray        # uint8 [num_pages * 41,984]
    index_cache: np.ndarray   # uint8 [num_pages * 8,448]
    layers: list = field(default_factory=list)
    ssmax: bool = False
    ssmax_s: float = 0.4
    ssmax_s_index: float = 0.4
    sm_scale: float = 1.0 / math.sqrt(576.0)
    latent_format: str = "fp8_ds_mla"   # or "e4m3": 576-B rows under one pool scale; or "bf16": 1,152-B rows
    latent_scale: float = 0.0

    @property
    def B(self):
        return len(self.ctx_len)

    @property
    def T(self):
        return int(self.cu_q[-1])

    @property
    def max_pages(self):
        return self.block_table.shape[1]

    @property
    def max_ctx(self):
        return int(self.ctx_len.max())

    def view(self, i: int = 0) -> SimpleNamespace:
        """Flat namespace of the batch plus layer i (what the oracle reads)."""
        lay = self.layers[i]
        return SimpleNamespace(
            cu_q=self.cu_q, ctx_len=self.ctx_len, block_table=self.block_table,
            num_heads=self.num_heads, topk=self.topk, ssmax=self.ssmax,
            ssmax_s=self.ssmax_s, ssmax_s_index=self.ssmax_s_index,
            sm_scale=self.sm_scale, rope_dim=lay.rope_dim, q=lay.q,
            iq8=lay.iq8, iq_scale=lay.iq_scale, iw=lay.iw)


def _chunked(num_pages: int, chunk_pages: int, fill):
    """Run fill(chunk_no, p0, p1) over page chunks on a thread pool.  Each chunk
    draws from its own named stream, so the bytes do not depend on the threads."""
    starts = range(0, num_pages, chunk_pages)
    jobs = [(i, p0, min(num_pages, p0 + chunk_pages)) for i, p0 in enumerate(starts)]
    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(lambda j: fill(*j), jobs))


def _fill_latent(seed: int, name: str, num_pages: int, chunk_pages: int = 512) -> np.ndarray:
    out = np.empty(num_pages * LATENT_PAGE, dtype=np.uint8)
    rows_all = out.reshape(num_pages * PAGE, LATENT_ROW)

    def fill(i, p0, p1):
        rng = stream(seed, f"{name}/latent/{i}")
        n = (p1 - p0) * PAGE
        x = rng.standard_normal((n, 512), dtype=np.float32)
        codes, scale = quantise_rows(x, 128)
        pe = to_bf16_bits(rng.standard_normal((n, 64), dtype=np.float32))
        rows = rows_all[p0 * PAGE:p1 * PAGE]
        rows[:, :512] = codes
        rows[:, 512:528] = scale.astype("<f4").view(np.uint8).reshape(n, 16)
        rows[:, 528:] = pe.astype("<u2").view(np.uint8).reshape(n, 128)

    _chunked(num_pages, chunk_pages, fill)
    return out


def _fill_index(seed: int, name: str, num_pages: int, chunk_pages: int = 2048) -> np.ndarray:
    out = np.empty(num_pages * INDEX_PAGE, dtype=np.uint8)
    pages = out.reshape(num_pages, INDEX_PAGE)

    def fill(i, p0, p1):
        rng = stream(seed, f"{name}/index_k/{i}")
        n = (p1 - p0) * PAGE
        x = rng.standard_normal((n, 128), dtype=np.float32)
        codes, scale = quantise_rows(x, 128)
        pg = pages[p0:p1]
        pg[:, :PAGE * 128] = codes.reshape(p1 - p0, PAGE * 128)
        pg[:, PAGE * 128:] = scale.astype("<f4").view(np.uint8).reshape(p1 - p0, PAGE * 4)

    _chunked(num_pages, chunk_pages, fill)
    return out


def _scribble_tails(wl: Workload, rng: np.random.Generator):
    """Random bytes in the unused rows of each request's last page."""
    row = {"e4m3": PLAIN_ROW, "bf16": BF16_ROW}.get(wl.latent_format, LATENT_ROW)
    lat = wl.latent.reshape(wl.num_pages, PAGE, row)
    idx = wl.index_cache.reshape(wl.num_pages, INDEX_PAGE)
    for r in range(wl.B):
        L = int(wl.ctx_len[r])
        if L % PAGE == 0:
            continue
        p = int(wl.block_table[r, (L - 1) // PAGE])
        used = L % PAGE
        lat[p, used:] = rng.integers(0, 256, size=lat[p, used:].shape, dtype=np.uint8)
        idx[p, used * 128:PAGE * 128] = rng.integers(0, 256, size=(PAGE - used) * 128, dtype=np.uint8)
        idx[p, PAGE * 128 + used * 4:] = rng.integers(0, 256, size=(PAGE - used) * 4, dtype=np.uint8)


def make_layer(seed: int, tag: str, T: int, H: int, rope_dim: int, with_indexer: bool = True,
               reuse_from: int | None = None) -> Layer:
    q = to_bf16_bits(stream(seed, tag + "/q").standard_normal((T, H, 512 + rope_dim), dtype=np.float32))
    lay = Layer(rope_dim=rope_dim, q=q, reuse_from=reuse_from)
    if with_indexer:
        x = stream(seed, tag + "/iq").standard_normal((T, 64 * 128), dtype=np.float32)
        codes, scale = quantise_rows(x, 64 * 128)
        lay.iq8 = codes.reshape(T, 64, 128)
        lay.iq_scale = scale[:, 0].astype(np.float32)
        lay.iw = (stream(seed, tag + "/iw").standard_normal((T, 64), dtype=np.float32) / 8).astype(np.float32)
    return lay


def plain_pool(seed: int, name: str, num_pages: int, chunk_pages: int = 512) -> np.ndarray:
    """Plain E4M3 latent pool: 576 values N(0, 1) per row (512 latent, 64 RoPE),
    codes of x / PLAIN_SCALE."""
    out = np.empty((num_pages, PLAIN_PAGE), dtype=np.uint8)

    def fill(i, p0, p1):
        x = stream(seed, f"{name}/plain/{i}").standard_normal(((p1 - p0) * PAGE, PLAIN_ROW), dtype=np.float32)
        out[p0:p1] = to_e4m3(x / np.float32(PLAIN_SCALE)).reshape(p1 - p0, PLAIN_PAGE)

    _chunked(num_pages, chunk_pages, fill)
    return out.reshape(-1)


def bf16_pool(seed: int, name: str, num_pages: int, chunk_pages: int = 512) -> np.ndarray:
    """bf16 latent pool: 576 values N(0, 1) per row (512 latent, 64 RoPE), as
    bf16 bits (float32 rounded to nearest even), little-endian."""
    out = np.empty((num_pages, BF16_PAGE), dtype=np.uint8)

    def fill(i, p0, p1):
        x = stream(seed, f"{name}/bf16/{i}").standard_normal(((p1 - p0) * PAGE, PLAIN_ROW), dtype=np.float32)
        b = x.view(np.uint32)
        h = ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype("<u2")
        out[p0:p1] = h.view(np.uint8).reshape(p1 - p0, BF16_PAGE)

    _chunked(num_pages, chunk_pages, fill)
    return out.reshape(-1)


def make_workload(name: str, ctx_len, q_count, num_heads: int, topk: int = 2048,
                  layers=(("rope", 64, True, None),), permuted: bool = True, ssmax: bool = False,
                  seed: int = 0, extra_pages: int = 0, latent_format: str = "fp8_ds_mla") -> Workload:
    """Build a batch of requests with the given context lengths and query counts.

    ``layers``: tuples (tag, rope_dim, with_indexer, reuse_from).
    ``extra_pages``: unused pages appended to the pool (random bytes).
    ``latent_format``: "fp8_ds_mla" (656-B rows), "e4m3" (576-B rows, one
    pool scale PLAIN_SCALE) or "bf16" (1,152-B rows).
    """
    ctx_len = np.asarray(ctx_len, dtype=np.int32)
    q_count = np.asarray(q_count, dtype=np.int32)
    assert ctx_len.shape == q_count.shape and np.all(q_count >= 1) and np.all(ctx_len >= q_count)
    B = len(ctx_len)
    cu_q = np.zeros(B + 1, dtype=np.int32)
    cu_q[1:] = np.cumsum(q_count)
    pages_per = (ctx_len + PAGE - 1) // PAGE
    used_pages = int(pages_per.sum())
    num_pages = used_pages + extra_pages
    max_pages = int(pages_per.max())
    rng_bt = stream(seed, name + "/block_table")
    phys = rng_bt.permutation(num_pages)[:used_pages] if permuted else np.arange(used_pages)
    block_table = np.zeros((B, max_pages), dtype=np.int32)
    off = 0
    for r in range(B):
        block_table[r, :pages_per[r]] = phys[off:off + pages_per[r]]
        off += pages_per[r]
    plain = latent_format == "e4m3"
    assert latent_format in ("fp8_ds_mla", "e4m3", "bf16")
    latent = (plain_pool(seed, name, num_pages) if plain else
              bf16_pool(seed, name, num_pages) if latent_format == "bf16" else _fill_latent(seed, name, num_pages))
    wl = Workload(name=name, num_heads=num_heads, topk=topk, cu_q=cu_q, ctx_len=ctx_len,
                  block_table=block_table, num_pages=num_pages,
                  latent=latent,
                  index_cache=_fill_index(seed, name, num_pages),
                  ssmax=ssmax, latent_format=latent_format, latent_scale=PLAIN_SCALE if plain else 0.0)
    _scribble_tails(wl, stream(seed, name + "/tails"))
    T = int(cu_q[-1])
    for tag, rope_dim, with_idx, reuse in layers:
        wl.layers.append(make_layer(seed, name + "/" + tag, T, num_heads, rope_dim, with_idx, reuse))
        wl.layers[-1].name = tag
    return wl


# --- the five workloads of the benchmark suite ---------------------------------

def tiny_decode(seed: int = 0) -> Workload:
    """1 request x 1 query token, context 4,096, 16 heads, identity block table."""
    return make_workload("tiny_decode", [4096], [1], 16, permuted=False, seed=seed)


def batched_decode(seed: int = 0) -> Workload:
    """32 requests x 1 query token, contexts uniform in [8,192, 65,536], 16 heads,
    permuted block table over a shared pool, SSMax off (one TP8 rank of decode)."""
    L = stream(seed, "batched_decode/ctx_len").integers(8192, 65536, size=32, endpoint=True)
    return make_workload("batched_decode", L, np.ones(32, np.int32), 16, seed=seed)


def spec_verify(seed: int = 0) -> Workload:
    """8 requests x 4 causal query tokens (1 target + 3 draft) at 60,000 context,
    128 heads, SSMax on (s = 0.4)."""
    return make_workload("spec_verify", [60000] * 8, [4] * 8, 128, ssmax=True, seed=seed)


def long_context(seed: int = 0) -> Workload:
    """1 request x 4 query tokens over 1,048,576 cached tokens, 128 heads, three
    layers over the same caches: RoPE, NoPE (RoPE dim 0, own indexer), and a
    shared-indexer RoPE layer reusing the NoPE layer's top-k."""
    return make_workload("long_context", [1 << 20], [4], 128, seed=seed,
                         layers=(("rope", 64, True, None), ("nope", 0, True, None),
                                 ("shared", 64, False, 1)))


def prefill_chunk(seed: int = 0) -> Workload:
    """2,048 causal query tokens after a 30,720-token prefix (32,768 total),
    16 heads, SSMax on."""
    return make_workload("prefill_chunk", [32768], [2048], 16, ssmax=True, seed=seed)


SUITE = {
    "tiny_decode": tiny_decode,
    "batched_decode": batched_decode,
    "spec_verify": spec_verify,
    "long_context": long_context,
    "prefill_chunk": prefill_chunk,
}


# --- inputs of the producers (new tokens before they enter the caches) ---------

def producer_rows(seed: int, name: str, n: int, dim: int, spread: bool = True) -> np.ndarray:
    """bf16 bits [n, dim] of new tokens' values, N(0, 1) per element.

    ``spread``: each row is also multiplied by 2^U(-24, 24), and the first rows
    are the special cases a quantiser meets: all zeros, all negative zeros, one
    non-zero element, values near bf16's largest and smallest normal magnitudes,
    and a row with a single element far above the rest."""
    rng = stream(seed, name)
    x = rng.standard_normal((n, dim), dtype=np.float32)
    if spread:
        x *= np.exp2(rng.uniform(-24, 24, size=(n, 1))).astype(np.float32)
        special = [np.zeros(dim, np.float32), -np.zeros(dim, np.float32),
                   np.eye(1, dim, dim // 3, dtype=np.float32)[0] * -3.0,
                   x[0] / np.abs(x[0]).max() * np.float32(3.0e38),
                   x[0] / np.abs(x[0]).max() * np.float32(2.0e-38),
                   np.where(np.arange(dim) == 7, np.float32(1e4), x[0] / np.abs(x[0]).max())]
        for i, row in enumerate(special[:n]):
            x[i] = row
    return to_bf16_bits(x)


def producer_slots(seed: int, name: str, n: int, num_pages: int, skip_every: int = 0) -> np.ndarray:
    """n distinct slots (page * 64 + row) of a num_pages pool, in random order;
    every skip_every-th one is -1 (a padding token)."""
    slot = stream(seed, name).permutation(num_pages * PAGE)[:n].astype(np.int32)
    if skip_every:
        slot[::skip_every] = -1
    return slot
