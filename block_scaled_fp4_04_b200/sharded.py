"""The path split over ranks (one process per GPU, torch.distributed for the plumbing).

Two ways of splitting it, neither of which moves activations or weights:

- Weights split along N (tensor parallel): each rank holds N / world rows of B and
  computes its own columns of D with the plain ``gemm``; the activations are replicated.
  There is nothing to exchange.
- Activations split by rows: NVFP4's global scale depends on the amax of the whole
  tensor ("MXFP4 / NVFP4 video transcript", NVFP4 passage), so the ranks exchange one
  float -- an all-reduce (MAX) of their local amax -- and every rank then quantizes its
  rows with the whole tensor's g.  The codes and scales are bit-identical to quantizing
  the unsplit tensor.  MXFP4 has no global scale and needs no exchange.

Every step on the data runs in libfp4's kernels (fp4_amax, fp4_global_scale,
fp4_quantize); this module only passes pointers and issues the one collective.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import (BF16, F32, NVFP4, Quantized, Workspace, fp4_amax, fp4_global_scale, fp4_quantize_workspace_size,
               quantize)


def reduce_amax_(amax: torch.Tensor, group=None) -> torch.Tensor:
    """The maximum over all ranks of ``amax`` (one float per rank), in place.  A no-op
    outside an initialized process group."""
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


def quantize_rows(x_local: torch.Tensor, group=None, workspace: Optional[Workspace] = None,
                  stream=None) -> Quantized:
    """NVFP4 (16-blocks) quantization of this rank's rows of a tensor split by rows over
    the ranks of ``group``.  Returns this rank's codes and scales and the whole tensor's
    global scale (identical on every rank)."""
    x_local = x_local.contiguous()
    dev = x_local.device
    ws = (workspace or Workspace(dev)).get(fp4_quantize_workspace_size())
    amax = torch.empty(1, dtype=torch.float32, device=dev)
    dt = BF16 if x_local.dtype == torch.bfloat16 else F32
    fp4_amax(x_local, x_local.numel(), dt, amax, ws, ws.numel(), stream)
    reduce_amax_(amax, group)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    fp4_global_scale(amax, g, stream)
    return quantize(x_local, NVFP4, 16, global_in=g, workspace=workspace, stream=stream)
