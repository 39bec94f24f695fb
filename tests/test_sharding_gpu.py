"""The product's sequence-sharded forward (sharding.sequence_parallel_forward) on
the GPU: each rank forms the state of its token range with sana_linattn_kv_state,
the ranks sum the states with one all-reduce, and each applies the sum to its own
queries with sana_linattn_apply (Eq. (1) of "Sana: Efficient High-Resolution Image
Synthesis with Linear Diffusion Transformers", section 2.1: the state is a plain
sum over tokens).

One GPU is available, so the two-rank case runs two processes on the same device
with a gloo process group (the all-reduce is staged through host memory); no
kernel of one rank waits on the other's."""
import os
import socket

import numpy as np
import pytest
import torch

from oracle import oracle as O
from parity import assert_close, to_dev
from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def test_single_rank_on_a_side_stream_equals_forward(cuda_lib):
    """World of one, launched on a non-current stream: the state, the (skipped)
    all-reduce and the apply stay ordered on that stream, and the result is the
    one-call forward bit for bit (same plan, partials summed in the same order)."""
    from relu_linear_attention_attn_b200 import sharding
    w = WORKLOADS["2048px-b8-lognormal"].scaled(B=2, N=3001, seed=71)
    x = make_inputs(w)
    d = to_dev(x)
    ref = cuda_lib.forward(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H, w.eps)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    out = sharding.sequence_parallel_forward(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H,
                                             w.eps, stream=side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert_close(out, O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps), "bf16")


SEQ_CASE = dict(B=2, N=2999, seed=72)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, outdir):
    import datetime
    import sys
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import relu_linear_attention_attn_b200 as sla
    from relu_linear_attention_attn_b200 import sharding
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        sla.load()
        torch.cuda.set_device(0)
        w = WORKLOADS["4096px-b2-overflow"].scaled(**SEQ_CASE)
        x = make_inputs(w)
        n0, cnt = sharding.token_shard(w.N, rank, world)
        sl = slice(n0, n0 + cnt)
        part = {n: x[n][:, sl].contiguous().cuda() for n in ("q", "k", "v")}
        gq = None if x["gq"] is None else x["gq"].cuda()
        gk = None if x["gk"] is None else x["gk"].cuda()
        out = sharding.sequence_parallel_forward(part["q"], part["k"], part["v"], gq, gk, w.H,
                                                 w.eps)
        torch.cuda.synchronize()
        np.save(os.path.join(outdir, f"out{rank}.npy"), out.float().cpu().numpy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_on_one_gpu_match_the_oracle(cuda_lib, tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = np.concatenate([np.load(os.path.join(tmp_path, f"out{r}.npy")) for r in range(world)],
                         axis=1)
    w = WORKLOADS["4096px-b2-overflow"].scaled(**SEQ_CASE)
    x = make_inputs(w)
    ref = O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps)
    assert got.shape == ref.shape
    assert_close(got, ref, "bf16", "sequence-sharded forward, 2 ranks")
