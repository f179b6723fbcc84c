"""The column-parallel (output-channel) split on CPU ranks (gloo, world
size 2): each rank keeps its slice of the packed weights and computes its
columns of Y from the full X; the gathered Y equals the one-rank Y bit for
bit.  The local layer is the oracle here (test code); on GPUs it is
tq_w4a4_lr_layer and the gather runs over NCCL."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

SHAPE = dict(M=16, K=1024, N=512, r=32, had_block=128)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_local_layer(X, L1t, Wq_loc, s_w_loc, L2t_loc, b):
    """The oracle's layer on this rank's channels (test stand-in for the
    GPU layer): codes of the full X, integer sums with the local weight
    codes, the low-rank branch with the local rows of L2^T."""
    import oracle
    a = oracle.quantize_act(X, b)
    acc = oracle.int_gemm(a["qx"], oracle.unpack_int4(Wq_loc.numpy()))
    _, lr = oracle.lowrank(X, L1t, L2t_loc)
    return torch.from_numpy(oracle.epilogue(a["s_x"], s_w_loc.numpy().astype(np.float64), acc, lr))


def _packed_layer():
    import oracle
    import synth
    sh = synth.CONFIGS["decode"].with_(**SHAPE)
    L = synth.make_layer(sh, seed=5)
    w = oracle.pack_weight(L["Rt"], sh.had_block)
    Wq = torch.from_numpy(w["Wq"])
    s_w = torch.from_numpy(w["s_w"])
    return L, Wq, s_w


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from rank_int4_gemm_b200 import column_parallel as cp
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L, Wq, s_w = _packed_layer()
        Wq_l, s_w_l, L2t_l = cp.shard_layer(Wq, s_w, L["L2t"], rank, world)
        assert Wq_l.shape[0] == SHAPE["N"] // world
        Y = cp.column_parallel_layer(L["X"], L["L1t"], Wq_l, s_w_l, L2t_l, SHAPE["had_block"],
                                     world, local_layer=_oracle_local_layer)
        q.put((rank, Y.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_gather_the_one_rank_output_exactly():
    import oracle
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    L, Wq, s_w = _packed_layer()
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], SHAPE["had_block"])
    for r in range(world):
        assert res[r].shape == (SHAPE["M"], SHAPE["N"])
        assert np.array_equal(res[r], o["Y64"]), r   # every rank has the whole Y, exactly


def test_channel_ranges_partition_the_channels():
    from rank_int4_gemm_b200 import column_parallel as cp
    for N, world in ((4096, 8), (14336, 4), (512, 2), (64, 1)):
        got = [cp.channel_range(N, r, world) for r in range(world)]
        assert got[0][0] == 0 and got[-1][1] == N
        assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
        assert all((n1 - n0) % 8 == 0 for n0, n1 in got)
    with pytest.raises(ValueError):
        cp.channel_range(4096, 0, 3)          # 4096 / 3 is not a whole number of 8-channel groups
    with pytest.raises(ValueError):
        cp.channel_range(512, 2, 2)           # no such rank


def test_single_rank_gather_is_identity():
    from rank_int4_gemm_b200 import column_parallel as cp
    y = torch.arange(12.0).reshape(3, 4)
    assert cp.gather_columns(y, 1) is y
