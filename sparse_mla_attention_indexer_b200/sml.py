"""ctypes binding of libsml.so (declared in ``include/sml.h``).

Argument marshalling only: every entry point takes torch tensors (device
memory) or plain ints, passes their addresses and sizes to the C ABI and raises
``SmlError`` on a non-zero status.  Every step of the computation runs in the
library's CUDA kernels; if ``libsml.so`` is missing the first call raises.

One decode layer, every tensor on the GPU in the layout ``include/sml.h``
gives (cu_q [B + 1], ctx_len [B] and block_table [B, max_pages] int32; q
[T, H, 576] bf16; iq [T, 64, 128] bf16; iw [T, 64] fp32; the two page pools
uint8)::

    from sparse_mla_attention_indexer_b200 import sml
    p = sml.make_problem(num_heads=16, topk=2048, rope_dim=64, cu_q=cu_q, ctx_len=ctx_len,
                         block_table=block_table, max_ctx=max_ctx, num_tokens=T,
                         sm_scale=576 ** -0.5)
    ws = torch.empty(sml.sml_workspace_size(p, sml.SML_STAGE_LAYER), dtype=torch.uint8,
                     device="cuda")
    sml.sml_workspace_init(ws)                                   # once per workspace
    sml.sml_indexer_k_cache_write(k_new, slot, index_pool, ws)   # the new tokens ...
    sml.sml_latent_cache_write(c_new, k_pe_new, slot, latent_pool, ws)   # ... into the caches
    sml.sml_indexer_q_quant(iq, iq8, iq_scale)
    sml.sml_run_layer(p, q, iq8, iq_scale, iw, latent_pool, index_pool, None, None,
                      idx, idx_len, out, lse, ws)                # indexer, top-k, sparse MLA
    code, bits = sml.sml_read_device_status(ws)                  # synchronises the stream

``max_ctx`` and ``num_tokens`` given explicitly keep ``make_problem`` from
reading the device arrays.  A shared-indexer layer passes the owner layer's
idx / idx_len as reuse_idx / reuse_len; the stages run one by one through
``sml_indexer_scores``, ``sml_topk`` and ``sml_sparse_mla_decode``.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import NamedTuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsml.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "sml.h")

SML_OK = 0
SML_ERR_INVALID_ARG = -1
SML_ERR_UNSUPPORTED = -2
SML_ERR_WORKSPACE = -3
SML_ERR_CUDA = -4
SML_ERR_DEVICE_FAULT = -5
SML_ERR_TIMEOUT = -6

SML_FAULT_PAGE = 0x1
SML_FAULT_INDEX = 0x2
SML_FAULT_LENGTHS = 0x4
SML_FAULT_TOPK_LEN = 0x8
SML_FAULT_TIMEOUT = 0x10

SML_STAGE_INDEXER = 1
SML_STAGE_TOPK = 2
SML_STAGE_MLA = 3
SML_STAGE_LAYER = 4

PAGE_TOKENS = 64
LATENT_PAGE_BYTES = 64 * 656
LATENT_E4M3_PAGE_BYTES = 64 * 576
LATENT_BF16_PAGE_BYTES = 64 * 1152
INDEX_PAGE_BYTES = 64 * 132
SML_LATENT_FP8_DS_MLA = 0
SML_LATENT_E4M3 = 1
SML_LATENT_BF16 = 2


class SmlError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


class Problem(ctypes.Structure):
    _fields_ = [
        ("num_requests", ctypes.c_int32),
        ("num_tokens", ctypes.c_int32),
        ("num_heads", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("rope_dim", ctypes.c_int32),
        ("max_pages", ctypes.c_int32),
        ("max_ctx", ctypes.c_int32),
        ("ssmax", ctypes.c_int32),
        ("sm_scale", ctypes.c_float),
        ("ssmax_s", ctypes.c_float),
        ("ssmax_s_index", ctypes.c_float),
        ("cu_q", ctypes.c_void_p),
        ("ctx_len", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("vis_len", ctypes.c_void_p),
        ("ssmax_len", ctypes.c_void_p),
    ]


class Cache(ctypes.Structure):
    _fields_ = [("base", ctypes.c_void_p), ("num_pages", ctypes.c_int64), ("format", ctypes.c_int32),
                ("scale", ctypes.c_float)]


SML_DCP_MAX_RANKS = 8


class DcpRanks(ctypes.Structure):
    _fields_ = [("num_ranks", ctypes.c_int32), ("interleave", ctypes.c_int32),
                ("scores", ctypes.c_void_p * SML_DCP_MAX_RANKS),
                ("score_stride", ctypes.c_int64 * SML_DCP_MAX_RANKS),
                ("idx", ctypes.c_void_p * SML_DCP_MAX_RANKS),
                ("idx_len", ctypes.c_void_p * SML_DCP_MAX_RANKS),
                ("packed", ctypes.c_int32)]


class Bf16Latent(NamedTuple):
    """A latent pool in bf16 (1,152-B rows: 512 latent then 64 RoPE values)."""
    pool: torch.Tensor


class E4M3Latent(NamedTuple):
    """A latent pool in the plain per-tensor E4M3 format (576-B rows) and its scale;
    a bare uint8 tensor is an fp8_ds_mla pool."""
    pool: torch.Tensor
    scale: float


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libsml.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libsml.so is not built ({LIB_PATH}); run "
                               "`python -m sparse_mla_attention_indexer_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        pp = ctypes.POINTER(Problem)
        L.sml_workspace_size.argtypes = [pp, i32]
        L.sml_workspace_size.restype = sz
        L.sml_workspace_init.argtypes = [vp, sz, vp]
        L.sml_indexer_scores.argtypes = [pp, vp, vp, vp, Cache, vp, vp, sz, vp]
        L.sml_topk.argtypes = [pp, vp, vp, vp, vp, sz, vp]
        L.sml_sparse_mla_decode.argtypes = [pp, vp, Cache, vp, vp, vp, vp, vp, sz, vp]
        L.sml_sparse_mla_decode_noalloc.argtypes = [pp, vp, Cache, vp, vp, vp, vp, vp]
        L.sml_run_layer.argtypes = [pp, vp, vp, vp, vp, Cache, Cache, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sml_read_device_status.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_int32), vp]
        L.sml_noalloc_read_status.argtypes = [i32, ctypes.POINTER(ctypes.c_int32), vp]
        L.sml_indexer_k_cache_write.argtypes = [vp, vp, ctypes.c_int32, Cache, vp, vp]
        L.sml_latent_cache_write.argtypes = [vp, vp, vp, ctypes.c_int32, Cache, vp, vp]
        L.sml_indexer_q_quant.argtypes = [vp, ctypes.c_int32, vp, vp, vp]
        i32p = ctypes.c_int32
        L.sml_dcp_merge_candidates.argtypes = [ctypes.POINTER(DcpRanks), i32p, i32p, vp, vp, vp, vp, vp]
        L.sml_dcp_pack_candidates.argtypes = [i32p, i32p, vp, ctypes.c_int64, vp, vp, vp, vp, vp]
        L.sml_dcp_split_selection.argtypes = [i32p, i32p, i32p, i32p, vp, vp, vp, ctypes.POINTER(vp),
                                              ctypes.POINTER(vp), vp, vp]
        L.sml_lse_combine.argtypes = [i32p, i32p, i32p, ctypes.POINTER(vp), ctypes.POINTER(vp), vp, vp, vp]
        L.sml_status_string.argtypes = [i32]
        for name in ("sml_status_string", "sml_last_error", "sml_version"):
            getattr(L, name).restype = ctypes.c_char_p
        for name in ("sml_workspace_init", "sml_indexer_scores", "sml_topk", "sml_sparse_mla_decode",
                     "sml_sparse_mla_decode_noalloc", "sml_run_layer", "sml_read_device_status",
                     "sml_noalloc_read_status",
                     "sml_indexer_k_cache_write", "sml_latent_cache_write", "sml_indexer_q_quant",
                     "sml_dcp_merge_candidates", "sml_dcp_split_selection", "sml_lse_combine",
                     "sml_dcp_pack_candidates"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def declared_entry_points(header: str = HEADER):
    """Names of the functions declared in include/sml.h."""
    text = open(header, encoding="utf-8").read()
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(sml_\w+)\s*\(", text, flags=re.M)))


def _p(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _s(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _numel(x) -> int:
    return 0 if x is None else int(x.numel())


def _check(code: int):
    if code != SML_OK:
        raise SmlError(code, lib().sml_last_error().decode())


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def make_problem(*, num_heads, topk, rope_dim, cu_q, ctx_len, block_table, max_ctx=None,
                 ssmax=False, sm_scale, ssmax_s=0.4, ssmax_s_index=0.4, num_tokens=None,
                 vis_len=None, ssmax_len=None) -> Problem:
    """Problem struct for device tensors cu_q [B+1], ctx_len [B], block_table [B, max_pages]
    (int32), and optionally vis_len [T] / ssmax_len [T] (int32 overrides of n_t and of the
    SSMax n)."""
    B = ctx_len.numel()
    return Problem(num_requests=B,
                   num_tokens=int(num_tokens) if num_tokens is not None else int(cu_q[-1]),
                   num_heads=num_heads, topk=topk, rope_dim=rope_dim,
                   max_pages=block_table.shape[1],
                   max_ctx=int(max_ctx) if max_ctx is not None else int(ctx_len.max()),
                   ssmax=int(bool(ssmax)), sm_scale=sm_scale, ssmax_s=ssmax_s,
                   ssmax_s_index=ssmax_s_index, cu_q=_p(cu_q), ctx_len=_p(ctx_len),
                   block_table=_p(block_table), vis_len=_p(vis_len), ssmax_len=_p(ssmax_len))


def cache(pool, page_bytes: int) -> Cache:
    """Cache descriptor of a uint8 pool tensor (or None for an absent cache)."""
    if pool is None:
        return Cache(None, 0, 0, 0.0)
    return Cache(_p(pool), _nbytes(pool) // page_bytes, 0, 0.0)


def latent_cache(latent) -> Cache:
    """Descriptor of a latent pool: a uint8 tensor (fp8_ds_mla), an E4M3Latent or a Bf16Latent."""
    if isinstance(latent, Bf16Latent):
        return Cache(_p(latent.pool), _nbytes(latent.pool) // LATENT_BF16_PAGE_BYTES, SML_LATENT_BF16, 0.0)
    if isinstance(latent, E4M3Latent):
        return Cache(_p(latent.pool), _nbytes(latent.pool) // LATENT_E4M3_PAGE_BYTES, SML_LATENT_E4M3,
                     float(latent.scale))
    return cache(latent, LATENT_PAGE_BYTES)


def sml_workspace_size(problem: Problem, stage: int) -> int:
    n = lib().sml_workspace_size(ctypes.byref(problem), stage)
    if n == 0:
        raise SmlError(SML_ERR_INVALID_ARG, lib().sml_last_error().decode())
    return n


def sml_workspace_init(workspace, stream=None):
    _check(lib().sml_workspace_init(_p(workspace), _nbytes(workspace), _s(stream)))


def sml_indexer_scores(problem, iq8, iq_scale, iw, index_cache, scores, workspace, stream=None):
    _check(lib().sml_indexer_scores(ctypes.byref(problem), _p(iq8), _p(iq_scale), _p(iw),
                                    cache(index_cache, INDEX_PAGE_BYTES), _p(scores), _p(workspace),
                                    _nbytes(workspace), _s(stream)))


def sml_topk(problem, scores, idx, idx_len, workspace, stream=None):
    _check(lib().sml_topk(ctypes.byref(problem), _p(scores), _p(idx), _p(idx_len), _p(workspace),
                          _nbytes(workspace), _s(stream)))


def sml_sparse_mla_decode(problem, q, latent, idx, idx_len, out, lse, workspace, stream=None):
    _check(lib().sml_sparse_mla_decode(ctypes.byref(problem), _p(q), latent_cache(latent),
                                       _p(idx), _p(idx_len), _p(out), _p(lse), _p(workspace),
                                       _nbytes(workspace), _s(stream)))


def sml_sparse_mla_decode_noalloc(problem, q, latent, idx, idx_len, out, lse, stream=None):
    """Sparse MLA decode without a workspace (scratch built into the library)."""
    _check(lib().sml_sparse_mla_decode_noalloc(ctypes.byref(problem), _p(q),
                                               latent_cache(latent), _p(idx),
                                               _p(idx_len), _p(out), _p(lse), _s(stream)))


def sml_noalloc_read_status(clear: bool = False, stream=None):
    """(status code, SML_FAULT_* bits) of the no-allocation entry point's own
    status word on the current device; synchronises the stream."""
    bits = ctypes.c_int32(0)
    code = lib().sml_noalloc_read_status(int(clear), ctypes.byref(bits), _s(stream))
    if code == SML_ERR_CUDA:
        _check(code)
    return code, bits.value


def sml_run_layer(problem, q, iq8, iq_scale, iw, latent, index_cache, reuse_idx, reuse_len,
                  idx_out, len_out, out, lse, workspace, stream=None):
    _check(lib().sml_run_layer(ctypes.byref(problem), _p(q), _p(iq8), _p(iq_scale), _p(iw),
                               latent_cache(latent), cache(index_cache, INDEX_PAGE_BYTES),
                               _p(reuse_idx), _p(reuse_len), _p(idx_out), _p(len_out), _p(out),
                               _p(lse), _p(workspace), _nbytes(workspace), _s(stream)))


def sml_indexer_k_cache_write(k, slot, index_cache, workspace=None, stream=None):
    """Quantise new indexer keys k [n, 128] bf16 into the indexer cache at slot [n] int32."""
    _check(lib().sml_indexer_k_cache_write(_p(k), _p(slot), _numel(slot), cache(index_cache, INDEX_PAGE_BYTES),
                                           _p(workspace), _s(stream)))


def sml_latent_cache_write(c, k_pe, slot, latent, workspace=None, stream=None):
    """Quantise new latent rows c [n, 512] bf16 (+ k_pe [n, 64] bf16, or None) into the
    fp8_ds_mla cache at slot [n] int32."""
    _check(lib().sml_latent_cache_write(_p(c), _p(k_pe), _p(slot), _numel(slot), latent_cache(latent),
                                        _p(workspace), _s(stream)))


def sml_indexer_q_quant(iq, iq8, iq_scale, stream=None):
    """Indexer queries iq [T, 64, 128] bf16 -> iq8 (e4m3 codes, uint8) and iq_scale [T] fp32."""
    _check(lib().sml_indexer_q_quant(_p(iq), _numel(iq_scale), _p(iq8), _p(iq_scale), _s(stream)))


def _ptrs(tensors):
    arr = (ctypes.c_void_p * max(1, len(tensors)))()
    for i, t in enumerate(tensors):
        arr[i] = _p(t)
    return arr


def sml_dcp_pack_candidates(scores, idx, idx_len, cand_scores, workspace=None, stream=None):
    """One rank's candidates for the exchange: cand_scores [T, topk] = scores at idx (NaN padding)."""
    T, K = idx.shape
    _check(lib().sml_dcp_pack_candidates(T, K, _p(scores), scores.shape[1], _p(idx), _p(idx_len),
                                         _p(cand_scores), _p(workspace), _s(stream)))


def sml_dcp_merge_candidates(scores, idx, idx_len, interleave, topk, merged_scores, merged_pos, merged_len,
                             workspace=None, stream=None, packed=False):
    """Ranks' top-k results (lists of per-rank tensors: scores [T, stride_r] -- or, packed,
    [T, topk] from sml_dcp_pack_candidates -- idx [T, topk], idx_len [T]) -> candidates in
    global position order."""
    rk = DcpRanks()
    rk.num_ranks = len(scores)
    rk.interleave = interleave
    rk.packed = int(bool(packed))
    for r, (sc, ix, ln) in enumerate(zip(scores, idx, idx_len)):
        rk.scores[r] = _p(sc)
        rk.score_stride[r] = sc.shape[1]
        rk.idx[r] = _p(ix)
        rk.idx_len[r] = _p(ln)
    _check(lib().sml_dcp_merge_candidates(ctypes.byref(rk), _numel(merged_len), topk, _p(merged_scores),
                                          _p(merged_pos), _p(merged_len), _p(workspace), _s(stream)))


def sml_dcp_split_selection(interleave, topk, sel, sel_len, merged_pos, local_idx, local_len, workspace=None,
                            stream=None):
    """Global selection (indices into the merged rows) -> each rank's compacted local list."""
    _check(lib().sml_dcp_split_selection(len(local_idx), interleave, _numel(sel_len), topk, _p(sel), _p(sel_len),
                                         _p(merged_pos), _ptrs(local_idx), _ptrs(local_len), _p(workspace),
                                         _s(stream)))


def sml_lse_combine(part_out, part_lse, out, lse, stream=None):
    """LSE combine of per-rank partial attentions (lists of tensors [T, H, 512] / [T, H])."""
    T, H = lse.shape
    _check(lib().sml_lse_combine(len(part_out), T, H, _ptrs(part_out), _ptrs(part_lse), _p(out), _p(lse),
                                 _s(stream)))


def sml_read_device_status(workspace, clear: bool = True, stream=None):
    """(status code, SML_FAULT_* bits); synchronises the stream."""
    bits = ctypes.c_int32(0)
    code = lib().sml_read_device_status(_p(workspace), int(clear), ctypes.byref(bits), _s(stream))
    if code in (SML_ERR_INVALID_ARG, SML_ERR_WORKSPACE, SML_ERR_CUDA):
        _check(code)
    return code, bits.value


def sml_status_string(code: int) -> str:
    return lib().sml_status_string(code).decode()


def sml_last_error() -> str:
    return lib().sml_last_error().decode()


def sml_version() -> str:
    return lib().sml_version().decode()
