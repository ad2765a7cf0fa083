"""Device-resident copy of a synthetic workload, laid out as include/sml.h expects.

Marshalling only: tensors are copied to the GPU as raw bytes (caches), bf16
(queries), e4m3 codes (indexer queries) and int32 metadata.
"""
from __future__ import annotations

import numpy as np
import torch

from . import sml


class DeviceLayer:
    def __init__(self, lay, device):
        self.rope_dim = lay.rope_dim
        self.reuse_from = lay.reuse_from
        self.q = torch.from_numpy(np.ascontiguousarray(lay.q).view(np.int16)).to(device).view(torch.bfloat16)
        if lay.iq8 is not None:
            self.iq8 = torch.from_numpy(np.ascontiguousarray(lay.iq8)).to(device)
            self.iq_scale = torch.from_numpy(np.ascontiguousarray(lay.iq_scale)).to(device)
            self.iw = torch.from_numpy(np.ascontiguousarray(lay.iw)).to(device)
        else:
            self.iq8 = self.iq_scale = self.iw = None


class DeviceWorkload:
    """A ``synth.Workload`` on the GPU, with one Problem struct per layer."""

    def __init__(self, wl, device: str = "cuda"):
        self.wl = wl
        self.device = device
        self.cu_q = torch.from_numpy(wl.cu_q).to(device)
        self.ctx_len = torch.from_numpy(wl.ctx_len).to(device)
        self.block_table = torch.from_numpy(np.ascontiguousarray(wl.block_table)).to(device)
        self.latent = torch.from_numpy(wl.latent).to(device)
        if wl.latent_format == "e4m3":
            self.latent = sml.E4M3Latent(self.latent, wl.latent_scale)
        elif wl.latent_format == "bf16":
            self.latent = sml.Bf16Latent(self.latent)
        self.index_cache = torch.from_numpy(wl.index_cache).to(device)
        self.layers = [DeviceLayer(lay, device) for lay in wl.layers]
        self.T, self.H, self.K = wl.T, wl.num_heads, wl.topk

    def problem(self, i: int = 0) -> sml.Problem:
        wl = self.wl
        return sml.make_problem(num_heads=wl.num_heads, topk=wl.topk,
                                rope_dim=wl.layers[i].rope_dim, cu_q=self.cu_q,
                                ctx_len=self.ctx_len, block_table=self.block_table,
                                max_ctx=wl.max_ctx, ssmax=wl.ssmax, sm_scale=wl.sm_scale,
                                ssmax_s=wl.ssmax_s, ssmax_s_index=wl.ssmax_s_index,
                                num_tokens=wl.T)

    def workspace(self, stage: int = sml.SML_STAGE_LAYER, i: int = 0) -> torch.Tensor:
        n = sml.sml_workspace_size(self.problem(i), stage)
        ws = torch.empty(n, dtype=torch.uint8, device=self.device)
        sml.sml_workspace_init(ws)
        return ws

    def outputs(self):
        """(idx, idx_len, out, lse) buffers for one layer."""
        d = self.device
        return (torch.empty(self.T, self.K, dtype=torch.int32, device=d),
                torch.empty(self.T, dtype=torch.int32, device=d),
                torch.empty(self.T, self.H, 512, dtype=torch.float32, device=d),
                torch.empty(self.T, self.H, dtype=torch.float32, device=d))

    def scores(self) -> torch.Tensor:
        return torch.empty(self.T, self.wl.max_ctx, dtype=torch.float32, device=self.device)
