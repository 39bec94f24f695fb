"""Multi-rank host logic on CPU: world size 2, gloo backend.

Sequence sharding: each rank forms the state of its token range (with the fp64
oracle standing in for the GPU), the states are summed with one all-reduce, and
each rank applies the summed state to its own queries; the result must equal the
single-process forward.  Batch sharding: the ranks' batch ranges tile the batch.
The max-over-ranks timing reduction is checked too."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import sys
        root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
        sys.path.insert(0, root)
        from oracle import oracle as O
        from relu_linear_attention_attn_b200 import sharding
        from relu_linear_attention_attn_b200.synthetic import CONFIGS, make_inputs

        w = CONFIGS[2].scaled(B=2, N=301, C=128, H=4, seed=91)      # ragged split
        x = make_inputs(w)
        n0, cnt = sharding.token_shard(w.N, rank, world)
        sl = slice(n0, n0 + cnt)
        S = torch.from_numpy(O.kv_state(x["k"][:, sl], x["v"][:, sl], x["gk"], w.H, w.eps))
        sharding.allreduce_state(S)
        out = O.apply(x["q"][:, sl], x["gq"], S.numpy(), w.H, w.eps)
        b0, bc = sharding.batch_shard(5, rank, world)
        t = sharding.max_over_ranks(1.5 + rank)
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), S=S.numpy(), out=out, n0=n0, cnt=cnt,
                 b0=b0, bc=bc, t=t)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    outdir = str(tmp_path_factory.mktemp("gloo"))
    mp.start_processes(_worker, args=(WORLD, _free_port(), outdir), nprocs=WORLD, join=True,
                       start_method="spawn")
    return [dict(np.load(os.path.join(outdir, f"rank{r}.npz"))) for r in range(WORLD)]


def test_sequence_sharded_state_and_output_match_single_process(results):
    from oracle import oracle as O
    from relu_linear_attention_attn_b200.synthetic import CONFIGS, make_inputs
    w = CONFIGS[2].scaled(B=2, N=301, C=128, H=4, seed=91)
    x = make_inputs(w)
    S_full = O.kv_state(x["k"], x["v"], x["gk"], w.H, w.eps)
    ref = O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps)
    for r in results:
        np.testing.assert_allclose(r["S"], S_full, rtol=1e-12, atol=1e-12)
        n0, cnt = int(r["n0"]), int(r["cnt"])
        np.testing.assert_allclose(r["out"], ref[:, n0:n0 + cnt], rtol=1e-11, atol=1e-13)
    assert sum(int(r["cnt"]) for r in results) == w.N


def test_batch_shards_tile_the_batch(results):
    covered = []
    for r in results:
        covered += list(range(int(r["b0"]), int(r["b0"]) + int(r["bc"])))
    assert covered == list(range(5))


def test_max_over_ranks(results):
    assert all(float(r["t"]) == 1.5 + (WORLD - 1) for r in results)


def test_even_split_edges():
    from relu_linear_attention_attn_b200.sharding import even_split
    assert [even_split(3, r, 4) for r in range(4)] == [(0, 0), (0, 1), (1, 1), (2, 1)]
    assert [even_split(10, r, 3) for r in range(3)] == [(0, 3), (3, 3), (6, 4)]
    with pytest.raises(ValueError):
        even_split(3, 4, 4)
