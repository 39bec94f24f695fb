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
        from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs

        w = WORKLOADS["2048px-b8-lognormal"].scaled(B=2, N=301, C=128, H=4, seed=91)      # ragged split
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
    from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs
    w = WORKLOADS["2048px-b8-lognormal"].scaled(B=2, N=301, C=128, H=4, seed=91)
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


# ----------------------------------------------------------------------------- Mix-FFN rows
MIX_WORLD = 3          # a middle rank exchanges with both neighbours


def _mix_case():
    from relu_linear_attention_attn_b200.synthetic import MIXFFN_WORKLOADS
    return MIXFFN_WORKLOADS["mixffn-tiny"].scaled(B=2, Hs=8, Ws=5, C=16, F=8, gate="silu", seed=92)


def _mix_worker(rank, world, port, outdir):
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
        from relu_linear_attention_attn_b200.synthetic import make_mixffn_inputs

        w = _mix_case()
        x = make_mixffn_inputs(w)
        f = lambda t: None if t is None else t.double().numpy()
        y0, cnt = sharding.row_shard(w.Hs, rank, world)
        x_r = f(x["x"])[:, y0 * w.Ws:(y0 + cnt) * w.Ws]
        # the expand of this rank's rows, with the fp64 oracle standing in for the GPU
        U = torch.from_numpy(O.linear(x_r, f(x["W1"]), f(x["b1"]))).reshape(w.B, cnt, w.Ws,
                                                                         2 * w.F)
        top, bottom = sharding.exchange_halo_rows(U[:, 0].contiguous(), U[:, -1].contiguous(),
                                                  rank, world)
        U_ext = torch.cat([top[:, None], U, bottom[:, None]], dim=1).numpy()
        Hg = O.dwconv_glu(U_ext.reshape(w.B, (cnt + 2) * w.Ws, 2 * w.F), f(x["wdw"]), f(x["bdw"]),
                          cnt + 2, w.Ws, w.gate).reshape(w.B, cnt + 2, w.Ws, w.F)[:, 1:cnt + 1]
        y = O.linear(Hg.reshape(w.B, cnt * w.Ws, w.F), f(x["W2"]), f(x["b2"]))
        np.savez(os.path.join(outdir, f"mix{rank}.npz"), y=y, y0=y0, cnt=cnt,
                 top=top.numpy(), bottom=bottom.numpy())
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def mix_results(tmp_path_factory):
    outdir = str(tmp_path_factory.mktemp("gloo_mix"))
    mp.start_processes(_mix_worker, args=(MIX_WORLD, _free_port(), outdir), nprocs=MIX_WORLD,
                       join=True, start_method="spawn")
    return [dict(np.load(os.path.join(outdir, f"mix{r}.npz"))) for r in range(MIX_WORLD)]


def test_row_sharded_mixffn_matches_single_process(mix_results):
    from oracle import oracle as O
    from relu_linear_attention_attn_b200.synthetic import make_mixffn_inputs
    w = _mix_case()
    x = make_mixffn_inputs(w)
    f = lambda t: None if t is None else t.double().numpy()
    ref = O.mixffn_forward(f(x["x"]), f(x["W1"]), f(x["b1"]), f(x["wdw"]), f(x["bdw"]), f(x["W2"]),
                           f(x["b2"]), w.Hs, w.Ws, w.gate)
    got = np.concatenate([r["y"] for r in mix_results], axis=1)
    assert [int(r["cnt"]) for r in mix_results] == [2, 3, 3]
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_halo_rows_are_the_neighbours_rows_and_zero_at_the_edges(mix_results):
    from oracle import oracle as O
    from relu_linear_attention_attn_b200.synthetic import make_mixffn_inputs
    w = _mix_case()
    x = make_mixffn_inputs(w)
    U = O.linear(x["x"].double().numpy(), x["W1"].double().numpy(),
                 x["b1"].double().numpy()).reshape(w.B, w.Hs, w.Ws, 2 * w.F)
    for r in mix_results:
        y0, cnt = int(r["y0"]), int(r["cnt"])
        exp_top = U[:, y0 - 1] if y0 > 0 else np.zeros_like(U[:, 0])
        exp_bot = U[:, y0 + cnt] if y0 + cnt < w.Hs else np.zeros_like(U[:, 0])
        np.testing.assert_array_equal(r["top"], exp_top)
        np.testing.assert_array_equal(r["bottom"], exp_bot)


def test_row_shard_needs_a_row_per_rank():
    from relu_linear_attention_attn_b200.sharding import row_shard
    assert [row_shard(8, r, 3) for r in range(3)] == [(0, 2), (2, 3), (5, 3)]
    with pytest.raises(ValueError):
        row_shard(2, 0, 3)
