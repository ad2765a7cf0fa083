"""sml_sparse_mla_decode_noalloc against sml_sparse_mla_decode and the oracle.

The no-allocation entry point serves callers that cannot give the library a
workspace (their device memory is all spoken for, or they may not call
cudaMalloc).  It keeps its split partials in scratch built into libsml.so, so
two calls in a row must both match the workspace entry point and the float64
oracle over the same selection; the second call also shows that the scratch
left behind by the first does no harm.  Its device checks report through a
status word of its own, read with sml_noalloc_read_status.  This file is
collected last on purpose.
"""
import numpy as np
import pytest
import torch

from sparse_mla_attention_indexer_b200 import sml, synth
from sparse_mla_attention_indexer_b200.device import DeviceWorkload
from tests import parity


@pytest.fixture(scope="module")
def lib():
    from sparse_mla_attention_indexer_b200 import build
    build.build()
    return sml.lib()


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice(lib):
    wl = synth.make_workload("noalloc", [9000, 3000, 700, 20000], [1, 2, 1, 3], 32, topk=2048,
                             ssmax=True)
    dw = DeviceWorkload(wl)
    p = dw.problem(0)
    lay = dw.layers[0]
    ws = dw.workspace()
    idx, ln, ref_out, ref_lse = dw.outputs()
    sml.sml_run_layer(p, lay.q, lay.iq8, lay.iq_scale, lay.iw, dw.latent, dw.index_cache, None, None,
                      idx, ln, ref_out, ref_lse, ws)
    assert sml.sml_read_device_status(ws)[0] == sml.SML_OK
    ref_o = ref_out.cpu().numpy().astype(np.float64)
    ref_l = ref_lse.cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(ref_o ** 2)))
    idx_h, ln_h = idx.cpu().numpy(), ln.cpu().numpy()
    assert sml.sml_noalloc_read_status(clear=True) == (sml.SML_OK, 0)
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        sml.sml_sparse_mla_decode_noalloc(p, lay.q, dw.latent, idx, ln, out, lse)
        torch.cuda.synchronize()
        o = out.cpu().numpy()
        lo = lse.cpu().numpy()
        # the workspace entry point
        assert np.abs(o - ref_o).max() <= parity.OUT_RMS_REL * rms, f"call {call}"
        assert np.abs(lo - ref_l).max() <= parity.LSE_ABS, f"call {call}"
        # the float64 oracle over the same selection
        parity.check_attention(wl, 0, idx_h, ln_h, o, lo)
        assert sml.sml_noalloc_read_status() == (sml.SML_OK, 0), f"call {call}"


@pytest.mark.gpu
def test_noalloc_reports_device_faults_in_its_own_status_word(lib):
    wl = synth.make_workload("noalloc_fault", [900, 300], [1, 2], 16, topk=64)
    dw = DeviceWorkload(wl)
    p = dw.problem(0)
    lay = dw.layers[0]
    ws = dw.workspace()
    idx, ln, out, lse = dw.outputs()
    sml.sml_run_layer(p, lay.q, lay.iq8, lay.iq_scale, lay.iw, dw.latent, dw.index_cache, None, None,
                      idx, ln, out, lse, ws)
    assert sml.sml_read_device_status(ws)[0] == sml.SML_OK
    sml.sml_noalloc_read_status(clear=True)
    bad = idx.clone()
    bad[1, 3] = 10_000                      # past the visible context: masked and reported
    sml.sml_sparse_mla_decode_noalloc(p, lay.q, dw.latent, bad, ln, out, lse)
    code, bits = sml.sml_noalloc_read_status(clear=True)
    assert code == sml.SML_ERR_DEVICE_FAULT and bits & sml.SML_FAULT_INDEX
    # cleared: the next good call reports nothing
    sml.sml_sparse_mla_decode_noalloc(p, lay.q, dw.latent, idx, ln, out, lse)
    assert sml.sml_noalloc_read_status() == (sml.SML_OK, 0)


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    # 4,096 tokens x 128 heads of split partials cannot fit in 16 MiB; rejected
    # on the host before any device work.
    p = sml.Problem(num_requests=1, num_tokens=4096, num_heads=128, topk=2048, rope_dim=64,
                    max_pages=128, max_ctx=8192, ssmax=0, sm_scale=0.04, ssmax_s=0.4,
                    ssmax_s_index=0.4, cu_q=0x1000, ctx_len=0x2000, block_table=0x3000)
    code = lib.sml_sparse_mla_decode_noalloc(p, 0x1000, sml.Cache(0x1000, 4), 0x10, 0x10, 0x1000,
                                             0x1000, None)
    assert code == sml.SML_ERR_UNSUPPORTED
    assert "scratch" in sml.sml_last_error()
