"""Data-parallel delayed scaling: one amax all-reduce per training step.

With ``fp8_set_ring_fold_mode(1)`` the linear entry points leave each ring's measured amax in
the ring's amax slot instead of folding it.  At the end of a step every rank calls
:func:`fold_rings_data_parallel` with its rings in the same order: the library gathers the
slots into one contiguous fp32 buffer, the ranks reduce it with MAX (``torch.distributed``:
NCCL between GPUs), and the library folds every ring with the reduced values.  All ranks then
hold identical history rings and publish identical steps, as if the whole global batch had been
quantized on one GPU.  This is plumbing around two library kernels and one collective; the
arithmetic (the gather and the fold) runs in the library.
"""

from __future__ import annotations

from . import _capi

__all__ = ["fold_rings_data_parallel"]


def fold_rings_data_parallel(rings, amax_buf, group=None, lib=_capi, stream=None):
    """Reduce the step's amax of every ring over the ranks of ``group`` and fold the rings.

    ``rings``: the same list of rings (``Ring`` or ``fp8_ring_t``, with the ``hist_idx`` the
    step's quantize used) on every rank.  ``amax_buf``: a float32 tensor of ``len(rings)``
    elements on the rings' device.  ``lib`` supplies ``fp8_scale_ring_collect_amax`` and
    ``fp8_scale_ring_fold`` (the library binding by default).
    """
    import torch.distributed as dist

    if len(rings) == 0:
        return
    if amax_buf.numel() < len(rings):
        raise ValueError("amax_buf holds fewer values than there are rings")
    buf = amax_buf[: len(rings)]
    lib.fp8_scale_ring_collect_amax(rings, buf, stream)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(buf, op=dist.ReduceOp.MAX, group=group)
    lib.fp8_scale_ring_fold(rings, buf, stream)
