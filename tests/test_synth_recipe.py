"""The seeded synthetic workloads keep the shapes, sizes and structure of their
stated recipe: request and query counts, context lengths and their range,
heads, top-k, SSMax, the layers of the long-context step, and a block table
that gives every request its own ceil(ctx / 64) distinct pages of the pool.
The cache fills are replaced by zero pools here (their bytes are not under
test), so the whole suite builds in seconds."""
import numpy as np
import pytest

from sparse_mla_attention_indexer_b200 import synth


@pytest.fixture
def cheap_pools(monkeypatch):
    monkeypatch.setattr(synth, "_fill_latent",
                        lambda seed, name, num_pages: np.zeros(num_pages * synth.LATENT_PAGE, np.uint8))
    monkeypatch.setattr(synth, "_fill_index",
                        lambda seed, name, num_pages: np.zeros(num_pages * synth.INDEX_PAGE, np.uint8))


def _check_block_table(wl, permuted):
    pages = -(-wl.ctx_len // 64)
    assert wl.block_table.shape == (wl.B, int(pages.max()))
    used = np.concatenate([wl.block_table[r, :pages[r]] for r in range(wl.B)])
    assert len(np.unique(used)) == len(used) == int(pages.sum())
    assert used.min() >= 0 and used.max() < wl.num_pages
    if not permuted:
        assert np.array_equal(used, np.arange(len(used)))


def _check_layer(lay, T, H, rope_dim, indexer, reuse=None):
    assert lay.rope_dim == rope_dim and lay.q.shape == (T, H, 512 + rope_dim) and lay.q.dtype == np.uint16
    assert lay.reuse_from == reuse
    if indexer:
        assert lay.iq8.shape == (T, 64, 128) and lay.iq_scale.shape == (T,) and lay.iw.shape == (T, 64)
    else:
        assert lay.iq8 is None and lay.iw is None


def test_decode_workloads(cheap_pools):
    wl = synth.tiny_decode()
    assert (wl.B, wl.T, wl.num_heads, wl.topk, wl.ssmax) == (1, 1, 16, 2048, False)
    assert list(wl.ctx_len) == [4096]
    _check_block_table(wl, permuted=False)
    _check_layer(wl.layers[0], 1, 16, 64, True)

    wl = synth.batched_decode()
    assert (wl.B, wl.T, wl.num_heads, wl.topk, wl.ssmax) == (32, 32, 16, 2048, False)
    assert np.array_equal(wl.cu_q, np.arange(33))
    assert wl.ctx_len.min() >= 8192 and wl.ctx_len.max() <= 65536 and len(np.unique(wl.ctx_len)) > 16
    _check_block_table(wl, permuted=True)
    _check_layer(wl.layers[0], 32, 16, 64, True)

    wl = synth.spec_verify()
    assert (wl.B, wl.T, wl.num_heads, wl.topk, wl.ssmax, wl.ssmax_s) == (8, 32, 128, 2048, True, 0.4)
    assert np.array_equal(wl.cu_q, np.arange(0, 33, 4)) and np.all(wl.ctx_len == 60000)
    _check_block_table(wl, permuted=True)


def test_long_context_and_prefill(cheap_pools):
    wl = synth.long_context()
    assert (wl.B, wl.T, wl.num_heads, wl.topk, wl.ssmax) == (1, 4, 128, 2048, False)
    assert list(wl.ctx_len) == [1 << 20] and wl.num_pages == (1 << 20) // 64
    assert [lay.name for lay in wl.layers] == ["rope", "nope", "shared"]
    _check_layer(wl.layers[0], 4, 128, 64, True)
    _check_layer(wl.layers[1], 4, 128, 0, True)
    _check_layer(wl.layers[2], 4, 128, 64, False, reuse=1)

    wl = synth.prefill_chunk()
    assert (wl.B, wl.T, wl.num_heads, wl.topk, wl.ssmax) == (1, 2048, 16, 2048, True)
    assert list(wl.ctx_len) == [32768]
    _check_block_table(wl, permuted=True)


def test_same_seed_same_workload_other_seed_other(cheap_pools):
    a, b, c = synth.batched_decode(0), synth.batched_decode(0), synth.batched_decode(1)
    assert np.array_equal(a.ctx_len, b.ctx_len) and np.array_equal(a.block_table, b.block_table)
    assert np.array_equal(a.layers[0].q, b.layers[0].q)
    assert not np.array_equal(a.ctx_len, c.ctx_len)
