"""Convenience layer over the C ABI for callers that hold torch tensors.

``FrontEnd`` keeps the embedding table and RMSNorm weight on the device and runs
``dmel_forward`` on batches of clips; with ``prepare=True`` it computes the table's Gram matrix
once (``dmel_table_prepare``) and runs ``dmel_forward_prepared``. ``plan()`` sizes the per-batch buffers (device offsets,
frame offsets, output, workspace) once, so repeated calls allocate nothing new.
``forward_host()`` is the end-to-end call: host waveforms in, frame vectors (and codes) back in
host memory, through ``dmel_forward_host`` (the library overlaps the copies with the kernels).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import dmel


@dataclass
class Plan:
    sample_offsets_host: np.ndarray
    frame_offsets_host: np.ndarray
    sample_offsets: torch.Tensor   # device int64 [n_clips + 1]
    frame_offsets: torch.Tensor    # device int64 [n_clips + 1]
    n_samples: int
    n_frames: int
    out: torch.Tensor              # device [n_frames, D]
    codes: torch.Tensor            # device uint8 [n_frames, 80]
    workspace: torch.Tensor | None
    host_workspace: torch.Tensor | None  # device scratch of forward_host (its staging buffers)
    chunk_frames: int

    @property
    def n_clips(self) -> int:
        return self.sample_offsets_host.shape[0] - 1


class FrontEnd:
    def __init__(self, table: torch.Tensor, rms_weight: torch.Tensor | None = None, eps: float = 1e-6,
                 out_dtype: torch.dtype = torch.bfloat16, prepare: bool = False):
        assert table.is_cuda and table.dim() == 2 and table.shape[0] == dmel.TABLE_ROWS
        self.table = table.contiguous()
        self.rms_weight = None if rms_weight is None else rms_weight.to(table.dtype).contiguous()
        self.eps = float(eps)
        self.out_dtype = out_dtype
        self.dim = int(table.shape[1])
        self.prepared = None  # the table's Gram matrix, when prepared and used by this configuration
        n = dmel.dmel_table_prepare_size(self.dim, dmel._dtype_code(self.table)) if prepare else 0
        if n and self.rms_weight is not None:
            self.prepared = torch.empty(n, dtype=torch.uint8, device=self.table.device)
            dmel.dmel_table_prepare(self.table, self.prepared)

    def plan(self, sample_offsets_host, chunk_frames: int = 0, host_path: bool = False) -> Plan:
        """Buffers for batches with these clip boundaries; with host_path, also the staging
        workspace of forward_host (chunks of chunk_frames frames, 0: the library's default)."""
        so = np.ascontiguousarray(np.asarray(sample_offsets_host, np.int64))
        fo = dmel.dmel_frame_offsets(so)
        dev = self.table.device
        F = int(fo[-1])
        tcode = dmel._dtype_code(self.table)
        ws_bytes = dmel.dmel_workspace_size(F, self.dim, tcode, self.rms_weight is not None, True)
        hws = None
        if host_path:
            n = dmel.dmel_forward_host_workspace_size(so, self.dim, tcode, dmel._dtype_code(
                torch.empty(0, dtype=self.out_dtype)), self.rms_weight is not None, chunk_frames)
            hws = torch.empty(max(1, n), dtype=torch.uint8, device=dev)
        return Plan(
            sample_offsets_host=so,
            frame_offsets_host=fo,
            sample_offsets=torch.from_numpy(so).to(dev),
            frame_offsets=torch.from_numpy(fo).to(dev),
            n_samples=int(so[-1]),
            n_frames=F,
            out=torch.empty((F, self.dim), dtype=self.out_dtype, device=dev),
            codes=torch.empty((F, dmel.N_MEL), dtype=torch.uint8, device=dev),
            workspace=torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None,
            host_workspace=hws,
            chunk_frames=int(chunk_frames),
        )

    def forward(self, wav: torch.Tensor, plan: Plan, tails=None, tails_out=None, stream=None) -> torch.Tensor:
        """Frame vectors of device waveforms `wav` (fp32 [n_samples]) into plan.out; codes into
        plan.codes."""
        dmel.dmel_forward_prepared(wav, plan.sample_offsets, plan.frame_offsets, plan.n_frames, self.table, plan.out,
                                   self.prepared, rms_weight=self.rms_weight, eps=self.eps, tails=tails,
                                   tails_out=tails_out, codes_out=plan.codes, workspace=plan.workspace, stream=stream)
        return plan.out

    def forward_host(self, wav_host: torch.Tensor, plan: Plan, out_host: torch.Tensor, codes_host=None, stream=None):
        """End to end from host memory: fp32 waveforms (page-locked for overlap) in, frame vectors
        into out_host [n_frames, D] (and codes into codes_host [n_frames, 80] when given), both
        host tensors. Asynchronous: the results are there once the stream reaches this call."""
        assert plan.host_workspace is not None, "plan(..., host_path=True) sizes the staging workspace"
        dmel.dmel_forward_host(wav_host, plan.sample_offsets_host, self.table, out_host, rms_weight=self.rms_weight,
                               eps=self.eps, codes_host=codes_host, chunk_frames=plan.chunk_frames,
                               workspace=plan.host_workspace, stream=stream)
        return out_host
