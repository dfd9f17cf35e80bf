"""Row-sharded tensors across ranks (one process per GPU, torch.distributed).

Blocks never straddle rows, so a tensor split by rows quantizes, dequantizes and reduces its
errors shard by shard with no exchange, except for two per-tensor quantities:

* the global FP16 scale g: it depends on the absmax of the whole tensor.  g = RU_fp16(A / (6 Smax))
  is non-decreasing in A, so the g of the whole tensor is the largest shard g; positive binary16
  bit patterns order like their values, so one MAX all-reduce of the bit patterns gives it;
* the error record: sums and counts add over shards (one SUM all-reduce of 3 doubles and 5
  integers; the sums then depend on the rank order of the reduction only through the additions).

Each rank runs the library's kernels on its own shard; only these two small collectives cross
ranks (NCCL over NVLink on GPUs, gloo on the CPU in the tests).
"""
import torch
import torch.distributed as dist

from . import api

_FIELDS = api.STATS_FIELDS  # sse_elem, sse_max, sse_zero, numel, n_blocks, n_zero_blocks, ...


def combine_g_bits(local_bits, group=None, device=None):
    """The g of the whole tensor from each rank's shard g (binary16 bit pattern, int)."""
    t = torch.tensor([int(local_bits) & 0xFFFF], dtype=torch.int64, device=device)
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return int(t.item())


def combine_stats(local, group=None, device=None):
    """The error record of the whole tensor from each rank's shard record (a dict as returned by
    ErrorStats.to_dict()); means are recomputed from the combined sums."""
    sums = torch.tensor([local[k] for k in _FIELDS[:3]], dtype=torch.float64, device=device)
    cnts = torch.tensor([int(local[k]) for k in _FIELDS[3:]], dtype=torch.int64, device=device)
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(sums, op=dist.ReduceOp.SUM, group=group)
        dist.all_reduce(cnts, op=dist.ReduceOp.SUM, group=group)
    out = dict(zip(_FIELDS[:3], (float(v) for v in sums.tolist())))
    out.update(zip(_FIELDS[3:], (int(v) for v in cnts.tolist())))
    return api.record_dict(api.record_bytes(out))


def record_from_bytes(raw):
    """An error record (64 bytes, mx_error_stats_t) as a dict (with the means)."""
    return api.record_dict(raw)


def global_scale_sharded(x_local, fmt="e4m3", group=None):
    """g (binary16 bits) of a row-sharded tensor: this rank's shard through the library's kernel,
    then the MAX over ranks."""
    local = int(api.global_scale(x_local, fmt).item()) & 0xFFFF
    return combine_g_bits(local, group=group, device=x_local.device)


def quantize_with_stats_sharded(x_local, block=32, fmt="e4m3", g=None, group=None):
    """Fused quantize + pack + error reduction of this rank's shard; returns (packed, scales,
    the error record of the whole tensor)."""
    packed, scales, st = api.quantize_with_stats(x_local, block, fmt, g)
    return packed, scales, combine_stats(st.to_dict(), group=group, device=x_local.device)
