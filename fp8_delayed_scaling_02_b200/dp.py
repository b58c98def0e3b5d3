"""Data-parallel delayed scaling: one FP8 scale for a tensor sharded over ranks.

When the activations (or gradients) of a linear are split across
data-parallel ranks, each rank sees only its shard, yet the per-tensor
delayed-scaling recipe folds the amax of the whole tensor into the history
ring.  Folding only the local amax would let the ranks' scales drift apart.

The cast itself needs only the scale published by the previous step, so the
quantize splits around one 4-byte collective:

1. ``ops.quantize_local``: every rank casts its shard with ``ring.scale``
   (the same codes ``ops.quantize`` writes), publishes ``ring.scale_inv``
   and this shard's amax over the raw values;
2. ``all_reduce_amax``: the ranks MAX-reduce that float (torch.distributed:
   NCCL over NVLink / NVSwitch on GPUs, gloo on CPUs);
3. ``ops.ring_fold``: every rank folds the global amax into its own copy of
   the ring, so rings that start equal stay equal.

The FP8-output GEMM splits the same way (``mm_fp8_out_dp``): each rank's
``ops.mm_ex`` writes its output rows' codes with the output ring's scale and
that shard's max |y|, the ranks MAX-reduce it, and every rank folds it.

Weights are replicated across data-parallel ranks and keep the single-rank
``ops.quantize``.
"""

import torch.distributed as dist

from . import ops


def all_reduce_amax(amax, group=None):
    """MAX-reduce the one-element float32 ``amax`` tensor in place over ``group``.

    A no-op when torch.distributed is not initialised or the group has one
    rank.  amax values are non-negative, so the float maximum is exact and
    independent of the reduction order.
    """
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


def quantize_dp(x, fmt, layout, ring, group=None, amax=None, out=None, out_t=None):
    """Cast this rank's shard ``x`` and fold the amax of the whole sharded tensor.

    Returns (out, out_t) like ``ops.quantize``.  Every rank of ``group`` must
    call it for the same tensor in the same order (it runs one collective).
    Kernels and the collective run on the current CUDA stream.
    """
    out, out_t, amax = ops.quantize_local(x, fmt, layout, ring, amax=amax, out=out, out_t=out_t)
    all_reduce_amax(amax, group)
    ops.ring_fold(ring, fmt, amax)
    return out, out_t


def mm_fp8_out_dp(a, b, sinv_a, sinv_b, out_fmt, ring, group=None, amax=None, **mm_kwargs):
    """FP8-output GEMM of this rank's rows ``a`` with the output's ring folded
    from the amax of the whole sharded output.

    ``mm_kwargs`` are ``ops.mm_ex``'s other keyword arguments (bias,
    bias_scale, bias_fmt, fmt_a, fmt_b, out, layouts, workspace).  Returns the
    codes.  Every rank of ``group`` must call it for the same output in the
    same order (it runs one collective).
    """
    import torch

    if amax is None:
        amax = torch.empty(1, dtype=torch.float32, device=a.device)
    out = ops.mm_ex(a, b, sinv_a, sinv_b, out_fmt=out_fmt, out_ring=ring, out_amax=amax, **mm_kwargs)
    all_reduce_amax(amax, group)
    ops.ring_fold(ring, out_fmt, amax)
    return out
