"""Run the three stages of one synthetic workload a few times (for profilers).

    python -m sparse_mla_attention_indexer_b200.run_stages [workload] [repetitions]

Each repetition flushes L2 with a 256 MiB write, then calls sml_indexer_scores,
sml_topk and sml_sparse_mla_decode on layer 0 of the workload; the device
status word is checked at the end.
"""
from __future__ import annotations

import sys

import torch

from . import sml, synth
from .device import DeviceWorkload


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    name = argv[0] if argv else "batched_decode"
    reps = int(argv[1]) if len(argv) > 1 else 3
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
