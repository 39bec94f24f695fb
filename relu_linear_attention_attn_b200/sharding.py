"""Host-side sharding of the linear-attention op over ranks (one process per GPU).

Two ways to split the op, both from the structure of Eq. (1) ("Sana: Efficient
High-Resolution Image Synthesis with Linear Diffusion Transformers", section 2.1):

* batch sharding - every (b, h) is independent, so ranks take disjoint batch
  items and never talk to each other (weak scaling, no data-path collective);
* sequence sharding - the state S = sum_n phi(K_n)^T [V_n | 1] is a plain sum over
  tokens, so ranks form the state of their token range, sum the states with one
  all-reduce of B*H*D*(D+1) fp32, and apply it to their own queries.

The collectives go through torch.distributed (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations


def even_split(n: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous, balanced [start, start + count) of n items for `rank` of `world`."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError("bad split arguments")
    start = n * rank // world
    return start, n * (rank + 1) // world - start


def batch_shard(B: int, rank: int, world: int) -> tuple[int, int]:
    """The batch items a rank owns under batch sharding."""
    return even_split(B, rank, world)


def token_shard(N: int, rank: int, world: int) -> tuple[int, int]:
    """The tokens a rank owns under sequence sharding."""
    return even_split(N, rank, world)


def allreduce_state(kv, group=None):
    """Sum the ranks' partial states in place (one all-reduce of the fp32 state)."""
    import torch.distributed as dist
    dist.all_reduce(kv, op=dist.ReduceOp.SUM, group=group)
    return kv


def max_over_ranks(x: float, device=None, group=None) -> float:
    """The largest of the ranks' values (e.g. elapsed device time)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def sequence_parallel_forward(q, k, v, gq, gk, H: int, eps: float, group=None, stream=None):
    """Eq. (1) over a sequence split across ranks.  q, k, v hold this rank's token
    range (B, N_r, C) on its GPU; returns this rank's output rows.  The state of
    the whole sequence is the all-reduced sum of the ranks' states."""
    import relu_linear_attention_attn_b200 as sla
    kv = sla.kv_state(k, v, gk, H, eps, stream=stream)
    allreduce_state(kv, group=group)
    return sla.apply(q, gq, kv, H, eps, stream=stream)
