"""The producers (FP8 quantisation and cache writes) on the GPU against the
oracle, byte for byte: every code, scale and RoPE key, and every byte of the
pool that no slot names stays as it was."""
import numpy as np
import pytest
import torch

from oracle import producers as PR
from sparse_mla_attention_indexer_b200 import sml, synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from sparse_mla_attention_indexer_b200 import build
    build.build()
    sml.lib()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def bf16_dev(bits):
    return dev(bits.view(np.int16)).view(torch.bfloat16)


def status_ws():
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    sml.sml_workspace_init(ws)
    return ws


# 10,003 new tokens: more than one grid-stride sweep of 8 warps x 8 CTAs per SM
@pytest.mark.parametrize("n,pages,skip", [(10003, 200, 97), (37, 3, 0), (1, 1, 0)])
def test_indexer_k_cache_write_bit_exact(n, pages, skip):
    k = synth.producer_rows(1, f"k/{n}", n, 128)
    slot = synth.producer_slots(1, f"slot/{n}", n, pages, skip)
    pool0 = synth.stream(1, f"pool/{n}").integers(0, 256, pages * synth.INDEX_PAGE, dtype=np.uint8)
    want, bad = PR.write_indexer_k(pool0, k, slot)
    assert not bad
    pool = dev(pool0)
    ws = status_ws()
    sml.sml_indexer_k_cache_write(bf16_dev(k), dev(slot), pool, ws)
    assert sml.sml_read_device_status(ws)[0] == sml.SML_OK
    got = pool.cpu().numpy()
    diff = np.nonzero(got != want)[0]
    assert diff.size == 0, f"{diff.size} bytes differ, first at {diff[:8]}"


@pytest.mark.parametrize("n,pages,skip,rope", [(10003, 160, 101, True), (300, 6, 7, False), (2, 1, 0, True)])
def test_latent_cache_write_bit_exact(n, pages, skip, rope):
    c = synth.producer_rows(2, f"c/{n}", n, 512)
    kpe = synth.producer_rows(2, f"kpe/{n}", n, 64, spread=False) if rope else None
    slot = synth.producer_slots(2, f"slot/{n}", n, pages, skip)
    pool0 = synth.stream(2, f"pool/{n}").integers(0, 256, pages * synth.LATENT_PAGE, dtype=np.uint8)
    want, bad = PR.write_latent(pool0, c, kpe, slot)
    assert not bad
    pool = dev(pool0)
    sml.sml_latent_cache_write(bf16_dev(c), None if kpe is None else bf16_dev(kpe), dev(slot), pool, status_ws())
    got = pool.cpu().numpy()
    diff = np.nonzero(got != want)[0]
    assert diff.size == 0, f"{diff.size} bytes differ, first at {diff[:8]}"


@pytest.mark.parametrize("T", [1207, 3, 1])
def test_indexer_q_quant_bit_exact(T):
    iq = synth.producer_rows(3, f"iq/{T}", T, 64 * 128).reshape(T, 64, 128)
    want_codes, want_scale = PR.quantise_indexer_q(iq)
    iq8 = torch.full((T, 64, 128), 0xAB, dtype=torch.uint8, device=DEV)
    scale = torch.full((T,), -1.0, dtype=torch.float32, device=DEV)
    sml.sml_indexer_q_quant(bf16_dev(iq), iq8, scale)
    got_scale = scale.cpu().numpy()
    assert np.array_equal(got_scale.view(np.uint32), want_scale.view(np.uint32))
    got = iq8.cpu().numpy()
    bad = np.nonzero((got != want_codes).reshape(T, -1).any(axis=1))[0]
    assert bad.size == 0, f"tokens {bad[:8]} differ"


def test_bad_slots_are_skipped_and_reported():
    n, pages = 50, 2
    k = synth.producer_rows(4, "k/bad", n, 128)
    c = synth.producer_rows(4, "c/bad", n, 512)
    slot = synth.producer_slots(4, "slot/bad", n, pages, 0)
    slot[3] = pages * 64          # one past the pool
    slot[9] = -7                  # negative, not the skip marker
    slot[11] = -1                 # skip marker: no report
    for write, size, args in ((PR.write_indexer_k, synth.INDEX_PAGE, (k,)),
                              (PR.write_latent, synth.LATENT_PAGE, (c, None))):
        pool0 = synth.stream(4, f"pool/bad/{size}").integers(0, 256, pages * size, dtype=np.uint8)
        want, bad = write(pool0, *args, slot)
        assert bad
        pool = dev(pool0)
        ws = status_ws()
        if write is PR.write_indexer_k:
            sml.sml_indexer_k_cache_write(bf16_dev(k), dev(slot), pool, ws)
        else:
            sml.sml_latent_cache_write(bf16_dev(c), None, dev(slot), pool, ws)
        code, bits = sml.sml_read_device_status(ws)
        assert code == sml.SML_ERR_DEVICE_FAULT and bits == sml.SML_FAULT_PAGE
        assert np.array_equal(pool.cpu().numpy(), want)
    # only the skip marker: no report
    slot_ok = synth.producer_slots(4, "slot/ok", n, pages, 5)
    ws = status_ws()
    pool = torch.zeros(pages * synth.INDEX_PAGE, dtype=torch.uint8, device=DEV)
    sml.sml_indexer_k_cache_write(bf16_dev(k), dev(slot_ok), pool, ws)
    assert sml.sml_read_device_status(ws)[0] == sml.SML_OK


def test_empty_batches_are_no_ops():
    pool = torch.zeros(synth.INDEX_PAGE, dtype=torch.uint8, device=DEV)
    lat = torch.zeros(synth.LATENT_PAGE, dtype=torch.uint8, device=DEV)
    empty_slot = torch.empty(0, dtype=torch.int32, device=DEV)
    sml.sml_indexer_k_cache_write(None, empty_slot, pool)
    sml.sml_latent_cache_write(None, None, empty_slot, lat)
    sml.sml_indexer_q_quant(None, None, torch.empty(0, dtype=torch.float32, device=DEV))
    torch.cuda.synchronize()
    assert not pool.any() and not lat.any()


def test_whole_pools_of_a_workload_match_the_oracle():
    """Both pools of a small workload, every slot written in order into zeroed
    pools from unspread bf16 rows, equal the oracle's pools byte for byte."""
    wl = synth.make_workload("producers_step", [700, 150], [1, 2], 16, topk=64)
    n_slots = wl.num_pages * 64
    slot = np.arange(n_slots, dtype=np.int32)
    c = synth.producer_rows(5, "step/c", n_slots, 512, spread=False)
    kpe = synth.producer_rows(5, "step/kpe", n_slots, 64, spread=False)
    k = synth.producer_rows(5, "step/k", n_slots, 128, spread=False)
    lat_want, _ = PR.write_latent(np.zeros_like(wl.latent), c, kpe, slot)
    idx_want, _ = PR.write_indexer_k(np.zeros_like(wl.index_cache), k, slot)
    lat = torch.zeros(wl.latent.size, dtype=torch.uint8, device=DEV)
    idx = torch.zeros(wl.index_cache.size, dtype=torch.uint8, device=DEV)
    sml.sml_latent_cache_write(bf16_dev(c), bf16_dev(kpe), dev(slot), lat)
    sml.sml_indexer_k_cache_write(bf16_dev(k), dev(slot), idx)
    assert np.array_equal(lat.cpu().numpy(), lat_want)
    assert np.array_equal(idx.cpu().numpy(), idx_want)


@pytest.mark.parametrize("n,pages,skip,rope", [(10003, 160, 101, True), (300, 6, 7, False)])
def test_plain_e4m3_latent_write_bit_exact(n, pages, skip, rope):
    from oracle import formats as F
    c = synth.producer_rows(6, f"pc/{n}", n, 512, spread=False)
    kpe = synth.producer_rows(6, f"pkpe/{n}", n, 64, spread=False) if rope else None
    slot = synth.producer_slots(6, f"pslot/{n}", n, pages, skip)
    scale = 5.0 / 448.0      # some values saturate at +-448 codes
    pool0 = synth.stream(6, f"ppool/{n}").integers(0, 256, pages * synth.PLAIN_PAGE, dtype=np.uint8)
    want, bad = PR.write_latent_plain_e4m3(F.PlainE4M3Pool(pool0, scale), c, kpe, slot)
    assert not bad
    pool = dev(pool0)
    sml.sml_latent_cache_write(bf16_dev(c), None if kpe is None else bf16_dev(kpe), dev(slot),
                               sml.E4M3Latent(pool, want.scale), status_ws())
    got = pool.cpu().numpy()
    diff = np.nonzero(got != want.data)[0]
    assert diff.size == 0, f"{diff.size} bytes differ, first at {diff[:8]}"


@pytest.mark.parametrize("n,pages,skip,rope", [(10003, 160, 101, True), (300, 6, 7, False)])
def test_bf16_latent_write_bit_exact(n, pages, skip, rope):
    """The bf16 latent writer stores every row exactly as the oracle's writer
    does (values as given, zeros for a NoPE row's RoPE key), skip markers and
    untouched rows included."""
    from oracle import formats as F
    c = synth.producer_rows(7, f"bc/{n}", n, 512, spread=False)
    kpe = synth.producer_rows(7, f"bkpe/{n}", n, 64, spread=False) if rope else None
    slot = synth.producer_slots(7, f"bslot/{n}", n, pages, skip)
    pool0 = synth.stream(7, f"bpool/{n}").integers(0, 256, pages * synth.BF16_PAGE, dtype=np.uint8)
    want, bad = PR.write_latent_bf16(F.Bf16Pool(pool0), c, kpe, slot)
    assert not bad
    pool = dev(pool0)
    ws = status_ws()
    sml.sml_latent_cache_write(bf16_dev(c), None if kpe is None else bf16_dev(kpe), dev(slot),
                               sml.Bf16Latent(pool), ws)
    assert sml.sml_read_device_status(ws)[0] == sml.SML_OK
    got = pool.cpu().numpy()
    diff = np.nonzero(got != want.data)[0]
    assert diff.size == 0, f"{diff.size} bytes differ, first at {diff[:8]}"
