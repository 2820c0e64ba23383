"""The layer under tensor parallelism: shard selection per rank, and the
channel-sharded output sconv with its reduce-scatter / all-gather.

vLLM Recipes "thinkingmachines/Inkling", Overview, "Short convolution": the
sconv is sharded across the channel dimension with a reduce-scatter /
all-gather so that neither its cache nor its compute is replicated across
tensor-parallel ranks; Performance: sconv-aware TP sharding, each rank storing
only its channel shard of the sconv cache.

* Keys, values and the attention itself shard by kv head: rank r of N takes kv
  heads [r*Hkv/N, (r+1)*Hkv/N), the query heads that read them, their bias
  rows, and the channels of those kv heads in the sconv taps, states and the
  paged cache.  The sconv is depthwise, so a rank's key/value sconv needs
  nothing from other ranks, and every library call on a shard equals that
  shard's slice of the call on the whole layer (`kv_head_shard`).
* The output sconv acts on the sum of the ranks' partial outputs (those of a
  row-parallel projection).  `sconv_out_reduce_scatter` computes it without
  replicating it: a reduce-scatter over channels gives rank r the summed
  input of its channel shard, the library's sconv kernel convolves that shard
  (continuing from the rank's state shard), and an all-gather returns the
  full output to every rank.  The collectives go through torch.distributed
  (NCCL between GPUs, plain copies, no multicast).  When the ranks' buffers
  are mapped into each other's address space, `sconv_out_sharded` in the
  binding does all three steps in one kernel over peer memory instead.

Only marshalling and collectives live here; every arithmetic step of the path
runs in libinkling's kernels (``local_sconv`` may be replaced only to test the
collective logic on hosts without a GPU).
"""
from __future__ import annotations

import torch

from . import binding


def kv_head_shard(Hq: int, Hkv: int, world: int, rank: int):
    """(query heads, kv heads, kv channels) of rank ``rank`` of ``world`` as
    slices; kv heads must divide evenly over the ranks."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    if Hkv % world or Hq % Hkv:
        raise ValueError("kv heads must divide over the ranks and query heads over kv heads")
    hk, hq = Hkv // world, Hq // world
    return (slice(rank * hq, (rank + 1) * hq), slice(rank * hk, (rank + 1) * hk),
            slice(rank * hk * binding.HEAD_DIM, (rank + 1) * hk * binding.HEAD_DIM))


def channel_shard(C: int, world: int, rank: int) -> slice:
    """Channels [rank*C/world, (rank+1)*C/world) of the output sconv."""
    if C % (8 * world):
        raise ValueError("channels must be a multiple of 8 * world")
    cs = C // world
    return slice(rank * cs, (rank + 1) * cs)


def sconv_out_reduce_scatter(x_partial: torch.Tensor, w: torch.Tensor, state_shard,
                             group=None, local_sconv=None) -> torch.Tensor:
    """Output sconv of the sum over ranks of ``x_partial`` [B, T, C] (this
    rank's partial sum), sharded over channels.

    ``w`` [C, 4] holds the taps of all channels; ``state_shard``
    [B, 3, C/world] (or None for zero history) is this rank's shard of the
    sconv state, updated in place.  Returns the full output [B, T, C] on
    every rank.  The reduce-scatter sums in fp32 (in the collective's own
    order) and the sum is rounded once to bf16, as in the one-kernel form over
    peer memory (which sums in rank order)."""
    import torch.distributed as dist
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    B, T, C = x_partial.shape
    sl = channel_shard(C, world, rank)
    cs = sl.stop - sl.start
    # channel shards as the leading dimension: [world, B*T, cs]
    parts = x_partial.reshape(B * T, world, cs).transpose(0, 1).to(torch.float32).contiguous()
    mine = torch.empty((B * T, cs), dtype=torch.float32, device=x_partial.device)
    if world > 1:
        dist.reduce_scatter_tensor(mine, parts.reshape(world * B * T, cs), group=group)
    else:
        mine.copy_(parts[0])
    xs = mine.to(torch.bfloat16).reshape(B, T, cs)
    w_shard = w[sl].contiguous()
    if local_sconv is None:
        ys = binding.sconv_out(xs, w_shard, state_shard)
    else:
        ys = local_sconv(xs, w_shard, state_shard)
    gathered = torch.empty((world * B * T, cs), dtype=torch.bfloat16, device=x_partial.device)
    if world > 1:
        dist.all_gather_into_tensor(gathered, ys.reshape(B * T, cs).contiguous(), group=group)
    else:
        gathered.copy_(ys.reshape(B * T, cs))
    return gathered.reshape(world, B * T, cs).transpose(0, 1).reshape(B, T, C)
