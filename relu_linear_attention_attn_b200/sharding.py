"""Host-side sharding of the linear-attention op over ranks (one process per GPU).

Two ways to split the op, both from the structure of Eq. (1) ("Sana: Efficient
High-Resolution Image Synthesis with Linear Diffusion Transformers", section 2.1):

* batch sharding - every (b, h) is independent, so ranks take disjoint batch
  items and never talk to each other (weak scaling, no data-path collective);
* sequence sharding - the state S = sum_n phi(K_n)^T [V_n | 1] is a plain sum over
  tokens, so ranks form the state of their token range, sum the states with one
  all-reduce of B*H*D*(D+1) fp32, and apply it to their own queries.

The Mix-FFN tail of the block shards its latent grid by rows with one halo-row
exchange between neighbouring ranks (below).

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
    """Sum the ranks' partial states in place (one all-reduce of the fp32 state).
    A single process (no process group, or a group of one) holds the whole state
    already and returns it unchanged."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return kv
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


def _on_stream(stream):
    """Make `stream` the current stream for the block (no-op for None), so the
    library's launches, torch's own work and the collectives, which order
    themselves after the current stream, all run in one order."""
    import contextlib

    import torch
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def sequence_parallel_forward(q, k, v, gq, gk, H: int, eps: float, group=None, stream=None):
    """Eq. (1) over a sequence split across ranks.  q, k, v hold this rank's token
    range (B, N_r, C) on its GPU; returns this rank's output rows.  The state of
    the whole sequence is the all-reduced sum of the ranks' states.  Everything
    runs on `stream` (default: the current stream), the all-reduce included."""
    import relu_linear_attention_attn_b200 as sla
    with _on_stream(stream):
        kv = sla.kv_state(k, v, gk, H, eps)
        allreduce_state(kv, group=group)
        return sla.apply(q, gq, kv, H, eps)


# ----------------------------------------------------------------------------- Mix-FFN
# The Mix-FFN ("Sana ...", section 2.2: 1x1 expand, 3x3 depthwise convolution with
# zero padding, GLU, 1x1 project) is token-local except for the convolution, which
# reads one grid row above and below.  Sharding the latent grid by rows therefore
# needs one real exchange step: each rank sends the first and last rows of its
# expanded activations U to its neighbours and receives theirs (the grid's outer
# edges get zero rows, which is the convolution's padding).  A rank keeps U with
# one spare row above and below its own rows, so no full-size copy is made.

def row_shard(Hs: int, rank: int, world: int) -> tuple[int, int]:
    """The grid rows [start, start + count) a rank owns under row sharding; every
    rank needs at least one row."""
    if Hs < world:
        raise ValueError("row sharding needs at least one grid row per rank")
    return even_split(Hs, rank, world)


def exchange_halo_rows(first, last, rank: int, world: int, group=None):
    """Swap boundary rows with the neighbouring ranks (point-to-point, all posted
    at once so no ordering can deadlock).  first / last: this rank's first and last
    grid rows (contiguous, same shape).  Returns (top, bottom): rank - 1's last row
    and rank + 1's first row, zeros at the grid's edges."""
    import torch
    top, bottom = torch.zeros_like(first), torch.zeros_like(last)
    if world == 1:
        return top, bottom
    import torch.distributed as dist
    ops = []
    if rank > 0:
        ops.append(dist.P2POp(dist.isend, first, rank - 1, group))
        ops.append(dist.P2POp(dist.irecv, top, rank - 1, group))
    if rank < world - 1:
        ops.append(dist.P2POp(dist.isend, last, rank + 1, group))
        ops.append(dist.P2POp(dist.irecv, bottom, rank + 1, group))
    for req in dist.batch_isend_irecv(ops):
        req.wait()
    return top, bottom


def mixffn_shard_expand(x_r, W1, b1, Ws: int, stream=None):
    """U of this rank's rows with a spare row above and below: (B, rows + 2, Ws, 2F)
    bf16, the spare rows zero.  x_r: (B, rows * Ws, C)."""
    import torch

    import relu_linear_attention_attn_b200 as sla
    B, Nr, C = x_r.shape
    rows = Nr // Ws
    if rows * Ws != Nr:
        raise ValueError("x_r must hold whole grid rows")
    F2 = W1.shape[1]
    with _on_stream(stream):
        U = torch.zeros(B, rows + 2, Ws, F2, dtype=x_r.dtype, device=x_r.device)
        for b in range(B):
            sla.gemm_bias(x_r[b], W1, b1, out=U[b, 1:rows + 1].view(rows * Ws, F2))
    return U


def mixffn_shard_finish(U, top, bottom, wdw, bdw, W2, b2, Ws: int, gate: str = "sigmoid",
                        stream=None):
    """Halo rows into U, then the convolution + GLU over the extended rows and the
    project of this rank's own rows: returns (B, rows * Ws, C)."""
    import torch

    import relu_linear_attention_attn_b200 as sla
    B, rows2, _, F2 = U.shape
    rows, F, C = rows2 - 2, F2 // 2, W2.shape[1]
    with _on_stream(stream):
        U[:, 0].copy_(top)
        U[:, rows + 1].copy_(bottom)
        Hg = sla.mixffn_dwconv_glu(U.view(B, rows2 * Ws, F2), wdw, bdw, rows2, Ws,
                                   gate).view(B, rows2, Ws, F)
        y = torch.empty(B, rows * Ws, C, dtype=U.dtype, device=U.device)
        for b in range(B):
            sla.gemm_bias(Hg[b, 1:rows + 1].reshape(rows * Ws, F), W2, b2, out=y[b])
    return y


def sequence_parallel_mixffn(x_r, W1, b1, wdw, bdw, W2, b2, Ws: int, rank: int, world: int,
                             gate: str = "sigmoid", group=None, stream=None):
    """The Mix-FFN of a latent grid split by rows across ranks: x_r holds this rank's
    rows (B, rows * Ws, C) on its GPU; returns this rank's output rows."""
    U = mixffn_shard_expand(x_r, W1, b1, Ws, stream=stream)
    rows = U.shape[1] - 2
    with _on_stream(stream):
        top, bottom = exchange_halo_rows(U[:, 1].contiguous(), U[:, rows].contiguous(), rank,
                                         world, group=group)
    return mixffn_shard_finish(U, top, bottom, wdw, bdw, W2, b2, Ws, gate, stream=stream)
