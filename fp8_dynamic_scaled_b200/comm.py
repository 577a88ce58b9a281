"""FP8 communication between data-parallel shards, over torch.distributed.

Two exchanges that the FP8 path has when a tensor is split across ranks:

* per-tensor current scaling of a sharded tensor needs one global a_max, so that
  every shard uses the one scale of the whole tensor ([FFS] "FP8 formats, scaling
  and LLM inference", section "Current Scaling": in distributed runs the ranks
  synchronise the amax; section "Scale 怎样把 Tensor 塞进 E4M3" lists distributed
  amax reduction among the recipe's parts).  That is a 4-byte MAX all-reduce placed
  between the two halves of the scaling, ``fp8_amax`` and ``fp8_quantize_with_amax``;
* an FP8 payload collective: quantise, send codes plus scales instead of bf16, and
  hand the receiver a scale-aware operand ([FFS] section "FP8 通信也独立于计算":
  amax/scale -> cast/pack -> communication -> scale-aware consumer, about half the
  bytes of a bf16 payload plus the scales).  ``all_gather_fp8`` gathers the shards'
  codes and scales into exactly the operand layout ``fp8_scaled_gemm`` consumes.

The collectives themselves are torch.distributed calls (NCCL on GPUs); every
arithmetic step runs in libfp8's kernels through the binding.  The kernel calls
are grouped in ``DeviceOps`` so that the orchestration can be exercised with other
implementations of the same three operations.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable

import torch
import torch.distributed as dist

# fp8_scaling_t values (include/fp8.h) used here
FP8_SCALE_TENSOR, FP8_SCALE_ROW = 0, 1


@dataclass
class DeviceOps:
    """The device operations the collectives use.  ``amax(x)`` returns a 1-element
    fp32 tensor; ``quantize_with_amax(x, fmt, amax)`` and ``quantize(x, fmt, mode)``
    return (codes uint8 [rows, cols], scale tensor in the fp8_quantize layout)."""
    amax: Callable
    quantize_with_amax: Callable
    quantize: Callable


def libfp8_ops() -> DeviceOps:
    """The default: libfp8's kernels on the tensors' CUDA device."""
    from . import binding as b

    def amax(x):
        out = torch.empty(1, dtype=torch.float32, device=x.device)
        b.fp8_amax(x, out, workspace=b.workspace_for(0, x.shape[0], 0, x.shape[1], b.FP8_SCALE_TENSOR,
                                                     device=x.device))
        return out

    def quantize_with_amax(x, fmt, a):
        q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
        s = torch.empty(1, dtype=torch.float32, device=x.device)
        b.fp8_quantize_with_amax(x, fmt, a, q, s)
        return q, s

    def quantize(x, fmt, mode):
        q, s, _ = b.empty_quant_outputs(x.shape[0], x.shape[1], mode, device=x.device)
        b.fp8_quantize(x, fmt, mode, q, s, workspace=b.workspace_for(0, x.shape[0], 0, x.shape[1], mode,
                                                                      device=x.device))
        return q, s

    return DeviceOps(amax, quantize_with_amax, quantize)


def global_amax(x: torch.Tensor, group=None, ops: DeviceOps | None = None) -> torch.Tensor:
    """a_max of the whole tensor whose row shard ``x`` this rank holds: the local
    maximum, then a MAX all-reduce (the maximum is exact and order-free, so every
    rank ends with the same bits)."""
    ops = ops or libfp8_ops()
    a = ops.amax(x)
    if dist.is_initialized():
        dist.all_reduce(a, op=dist.ReduceOp.MAX, group=group)
    return a


def quantize_tensor_sharded(x: torch.Tensor, fmt: int, group=None, ops: DeviceOps | None = None):
    """Per-tensor current scaling of a row-sharded tensor: every rank casts its shard
    with the scale of the whole tensor.  Returns (codes of the shard, scale)."""
    ops = ops or libfp8_ops()
    return ops.quantize_with_amax(x, fmt, global_amax(x, group, ops))


def _all_gather_rows(t: torch.Tensor, group=None) -> torch.Tensor:
    """Concatenate every rank's equally shaped tensor along dim 0 (rank order)."""
    world = dist.get_world_size(group)
    if world == 1:
        return t
    if dist.get_backend(group) == "nccl":
        out = torch.empty((world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
        return out
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.cat(parts, dim=0)


def all_gather_fp8(x: torch.Tensor, fmt: int, mode: int, group=None, ops: DeviceOps | None = None):
    """Gather the row shards of a bf16 tensor as FP8: each rank quantises its shard and
    the codes (1 byte per element) and scales travel instead of bf16 (2 bytes).

    mode FP8_SCALE_ROW (per token): each shard is quantised on its own (no amax
    exchange); the gathered per-row scales line up with the gathered rows.
    mode FP8_SCALE_TENSOR: one global a_max first (``quantize_tensor_sharded``), so the
    single scale is the same on every rank and is returned as is.
    Returns (codes [world * rows, cols], scale) in the fp8_quantize layout of the
    gathered tensor, ready for fp8_scaled_gemm.  Shards must have equal shapes."""
    ops = ops or libfp8_ops()
    if mode == FP8_SCALE_TENSOR:
        q, s = quantize_tensor_sharded(x, fmt, group, ops)
        return _all_gather_rows(q, group), s
    if mode == FP8_SCALE_ROW:
        q, s = ops.quantize(x, fmt, mode)
        return _all_gather_rows(q, group), _all_gather_rows(s, group)
    raise ValueError("all_gather_fp8 supports per-tensor and per-row scaling")


def payload_bytes(rows: int, cols: int, mode: int) -> dict:
    """Bytes one rank contributes to the gather: FP8 codes plus scales, against bf16."""
    scale = 4 * rows if mode == FP8_SCALE_ROW else 0
    return {"fp8": rows * cols + scale, "bf16": 2 * rows * cols}
