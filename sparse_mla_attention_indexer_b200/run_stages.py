"""Run the three stages of one synthetic workload a few times (for profilers).

    python -m sparse_mla_attention_indexer_b200.run_stages [workload] [repetitions]
    python -m sparse_mla_attention_indexer_b200.run_stages producers [repetitions]

Each repetition flushes L2 with a 256 MiB write, then calls sml_indexer_scores,
sml_topk and sml_sparse_mla_decode on layer 0 of the workload; the device
status word is checked at the end.  ``producers`` instead calls, per
repetition, the indexer K and latent cache writes for 16,384 new tokens at
distinct random slots of 1,024-page pools and the indexer Q quantisation of
2,048 tokens.
"""
from __future__ import annotations

import sys

import torch

from . import sml, synth
from .device import DeviceWorkload


def producers(reps: int) -> int:
    n, nq, pages = 16384, 2048, 1024

    def bf16(bits):
        return torch.from_numpy(bits.view("int16")).cuda().view(torch.bfloat16)

    k = bf16(synth.producer_rows(11, "profile/k", n, 128, spread=False))
    c = bf16(synth.producer_rows(11, "profile/c", n, 512, spread=False))
    kpe = bf16(synth.producer_rows(11, "profile/kpe", n, 64, spread=False))
    iq = bf16(synth.producer_rows(11, "profile/iq", nq, 64 * 128, spread=False))
    slot = torch.from_numpy(synth.producer_slots(11, "profile/slot", n, pages)).cuda()
    lat = torch.zeros(pages * synth.LATENT_PAGE, dtype=torch.uint8, device="cuda")
    idx = torch.zeros(pages * synth.INDEX_PAGE, dtype=torch.uint8, device="cuda")
    iq8 = torch.empty(nq * 64 * 128, dtype=torch.uint8, device="cuda")
    iqs = torch.empty(nq, dtype=torch.float32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    sml.sml_workspace_init(ws)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(reps):
        flush.fill_(1)
        sml.sml_indexer_k_cache_write(k, slot, idx, ws)
        sml.sml_latent_cache_write(c, kpe, slot, lat, ws)
        sml.sml_indexer_q_quant(iq, iq8, iqs)
    torch.cuda.synchronize()
    code, bits = sml.sml_read_device_status(ws)
    print("device status", code, hex(bits))
    return 0 if code == sml.SML_OK else 1


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    name = argv[0] if argv else "batched_decode"
    reps = int(argv[1]) if len(argv) > 1 else 3
    if name == "producers":
        return producers(reps)
    wl = synth.SUITE[name]()
    dw = DeviceWorkload(wl)
    p = dw.problem(0)
    lay = dw.layers[0]
    ws = dw.workspace()
    idx, ln, out, lse = dw.outputs()
    scores = dw.scores()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(reps):
        flush.fill_(1)
        sml.sml_indexer_scores(p, lay.iq8, lay.iq_scale, lay.iw, dw.index_cache, scores, ws)
        sml.sml_topk(p, scores, idx, ln, ws)
        sml.sml_sparse_mla_decode(p, lay.q, dw.latent, idx, ln, out, lse, ws)
    torch.cuda.synchronize()
    code, bits = sml.sml_read_device_status(ws)
    print("device status", code, hex(bits))
    return 0 if code == sml.SML_OK else 1


if __name__ == "__main__":
    sys.exit(main())
