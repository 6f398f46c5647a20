"""Convenience layer over the C ABI for callers that hold torch tensors.

``FrontEnd`` keeps the embedding table and RMSNorm weight on the device and runs
``dmel_forward`` on batches of clips. ``plan()`` sizes the per-batch buffers (device offsets,
frame offsets, output, workspace) once, so repeated calls allocate nothing new.
``forward_host()`` is the end-to-end call: pinned host waveforms in, codes back on the host,
frame vectors left on the device for the model that consumes them.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import dmel


@dataclass
class ChunkPlan:
    """A run of whole clips [clip0, clip1) of a batch, with offsets rebased to the run."""
    clip0: int
    clip1: int
    sample0: int
    sample1: int
    frame0: int
    frame1: int
    sample_offsets: torch.Tensor  # device int64, rebased to 0
    frame_offsets: torch.Tensor   # device int64, rebased to 0


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
    wav: torch.Tensor              # device fp32 [n_samples] (input staging for forward_host)
    chunks: list                   # ChunkPlan runs used by forward_host to overlap copies and compute

    @property
    def n_clips(self) -> int:
        return self.sample_offsets_host.shape[0] - 1


class FrontEnd:
    def __init__(self, table: torch.Tensor, rms_weight: torch.Tensor | None = None, eps: float = 1e-6,
                 out_dtype: torch.dtype = torch.bfloat16):
        assert table.is_cuda and table.dim() == 2 and table.shape[0] == dmel.TABLE_ROWS
        self.table = table.contiguous()
        self.rms_weight = None if rms_weight is None else rms_weight.to(table.dtype).contiguous()
        self.eps = float(eps)
        self.out_dtype = out_dtype
        self.dim = int(table.shape[1])

    def plan(self, sample_offsets_host, chunks: int = 4) -> Plan:
        """Buffers for batches with these clip boundaries; `chunks` runs of whole clips (balanced
        by frames) for the pipelined host path."""
        so = np.ascontiguousarray(np.asarray(sample_offsets_host, np.int64))
        fo = dmel.dmel_frame_offsets(so)
        dev = self.table.device
        F = int(fo[-1])
        n_clips = so.shape[0] - 1
        ws_bytes = dmel.dmel_workspace_size(F, self.dim, dmel._dtype_code(self.table), self.rms_weight is not None,
                                            True)
        runs = []
        k = max(1, min(int(chunks), n_clips))
        bounds = [0]
        for i in range(1, k):
            c = int(np.searchsorted(fo, F * i // k, side="left"))
            bounds.append(min(max(c, bounds[-1]), n_clips))
        bounds.append(n_clips)
        for c0, c1 in zip(bounds[:-1], bounds[1:]):
            if c1 <= c0:
                continue
            runs.append(ChunkPlan(c0, c1, int(so[c0]), int(so[c1]), int(fo[c0]), int(fo[c1]),
                                  torch.from_numpy(so[c0:c1 + 1] - so[c0]).to(dev),
                                  torch.from_numpy(fo[c0:c1 + 1] - fo[c0]).to(dev)))
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
            wav=torch.empty(int(so[-1]), dtype=torch.float32, device=dev),
            chunks=runs,
        )

    def forward(self, wav: torch.Tensor, plan: Plan, tails=None, tails_out=None, stream=None) -> torch.Tensor:
        """Frame vectors of device waveforms `wav` (fp32 [n_samples]) into plan.out; codes into
        plan.codes."""
        dmel.dmel_forward(wav, plan.sample_offsets, plan.frame_offsets, plan.n_frames, self.table, plan.out,
                          rms_weight=self.rms_weight, eps=self.eps, tails=tails, tails_out=tails_out,
                          codes_out=plan.codes, workspace=plan.workspace, stream=stream)
        return plan.out

    def forward_host(self, wav_host: torch.Tensor, plan: Plan, codes_host: torch.Tensor, copy_stream=None):
        """End to end from host memory: copies the pinned fp32 waveforms to the device, runs the
        front end, copies the codes (uint8 [n_frames, 80], pinned) back; the frame vectors stay
        in plan.out. The batch goes in plan.chunks runs of whole clips: the host-to-device copy
        of run i + 1 (on `copy_stream`) overlaps the kernels of run i (on the current stream).
        Asynchronous; the caller synchronises the current stream."""
        compute = torch.cuda.current_stream()
        copy = copy_stream if copy_stream is not None else self._copy_stream()
        copy.wait_stream(compute)  # the buffers are free once earlier work on them is done
        ready = []
        for r in plan.chunks:
            with torch.cuda.stream(copy):
                plan.wav[r.sample0:r.sample1].copy_(wav_host[r.sample0:r.sample1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy)
            ready.append(ev)
        for r, ev in zip(plan.chunks, ready):
            compute.wait_event(ev)
            if r.frame1 > r.frame0:
                dmel.dmel_forward(plan.wav[r.sample0:r.sample1], r.sample_offsets, r.frame_offsets,
                                  r.frame1 - r.frame0, self.table, plan.out[r.frame0:r.frame1],
                                  rms_weight=self.rms_weight, eps=self.eps, codes_out=plan.codes[r.frame0:r.frame1],
                                  workspace=plan.workspace, stream=compute)
                codes_host[r.frame0:r.frame1].copy_(plan.codes[r.frame0:r.frame1], non_blocking=True)
        return plan.out

    def _copy_stream(self):
        if getattr(self, "_copy", None) is None or self._copy.device != self.table.device:
            self._copy = torch.cuda.Stream(device=self.table.device)
        return self._copy
