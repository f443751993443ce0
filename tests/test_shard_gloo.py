"""World-size-2 data parallelism on CPU (gloo): shards by whole sequences, each
rank computes its shard's gradients (oracle on CPU), the parameter gradients
are all-reduced, and everything matches the single-process full batch."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from hstu_jagged_pointwise_b200 import shard, workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _global_batch():
    return W.make_causal([5, 30, 9, 17, 1, 26, 12], H=2, d=4, dtype=torch.float32, seed=41, alpha=30.0,
                         random_affine=True, with_grad=True)


def _sub(w, seqs):
    off, rows = shard.shard_rows(w.offsets, seqs)
    lens = np.diff(off)
    s = W.make_causal(lens, H=w.H, d=w.d, dtype=w.dtype, seed=0, alpha=w.alpha,
                      ts_list=[w.ts[w.offsets[b]:w.offsets[b + 1]] for b in seqs], with_grad=True)
    rt = torch.as_tensor(rows)
    for n in ("q", "k", "v", "u", "grad"):
        setattr(s, n, getattr(w, n)[rt])
    s.rab_pos, s.rab_time, s.gamma, s.beta = w.rab_pos, w.rab_time, w.gamma, w.beta
    return s, rows


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _global_batch()
        parts = shard.partition_sequences(w.lengths, world)
        mine = shard.rank_sequences(w.lengths, world, rank)       # what bench.py's ranks take
        assert mine == parts[rank]
        s, rows = _sub(w, mine)
        g = oracle.layer_bwd(s)
        grads = {"d_rab_pos": torch.tensor(g["d_rab_pos"]), "d_rab_time": torch.tensor(g["d_rab_time"]),
                 "d_gamma": torch.tensor(g["dgamma"]), "d_beta": torch.tensor(g["dbeta"])}
        shard.allreduce_param_grads(grads)
        q.put((rank, parts, rows, {k: v.numpy() for k, v in grads.items()}, g["dq"], g["dk"], g["dv"], g["du"]))
    finally:
        dist.destroy_process_group()


def test_partition_covers_and_balances():
    L = np.array([4096, 3000, 10, 2000, 2000, 500, 64, 64, 7])
    parts = shard.partition_sequences(L, 3)
    flat = sorted(b for p in parts for b in p)
    assert flat == list(range(len(L)))
    cost = [sum(int(L[b]) ** 2 for b in p) for p in parts]
    assert max(cost) - min(cost) <= int(L.max()) ** 2
    assert shard.partition_sequences([], 2) == [[], []]


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_match_single_process(world):
    import oracle
    w = _global_batch()
    ref = oracle.layer_bwd(w)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    covered = []
    for rank, parts, rows, grads, dq, dk, dv, du in res:
        covered += list(rows)
        for k, rk in (("d_rab_pos", "d_rab_pos"), ("d_rab_time", "d_rab_time"), ("d_gamma", "dgamma"),
                      ("d_beta", "dbeta")):
            np.testing.assert_allclose(grads[k], ref[rk], rtol=1e-12, atol=1e-14)
        for got, name in ((dq, "dq"), (dk, "dk"), (dv, "dv"), (du, "du")):
            np.testing.assert_allclose(got, ref[name][rows], rtol=1e-12, atol=1e-14)
    assert sorted(covered) == list(range(w.T))


def _balanced_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _global_batch()
        start, tokens, weights = oracle.pack_balanced(w.offsets, world)
        seqs = shard.bin_sequences(start, rank)
        s, rows = _sub(w, seqs)
        g = oracle.layer_bwd(s)
        n = max(len(seqs), 1)
        # this rank's per-sample mean of the parameter gradients, re-weighted by its share of samples
        grads = {"d_rab_pos": torch.tensor(g["d_rab_pos"]) / n, "d_rab_time": torch.tensor(g["d_rab_time"]) / n,
                 "d_gamma": torch.tensor(g["dgamma"]) / n, "d_beta": torch.tensor(g["dbeta"]) / n}
        shard.allreduce_param_grads(grads, weight=float(weights[rank]))
        q.put((rank, seqs, int(tokens[rank]), {k: v.numpy() for k, v in grads.items()}))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_token_balanced_bins_give_the_batch_mean_gradient(world):
    """MTGR's dynamic batches: each rank takes one token-balanced bin (different sample
    counts), and the weighted all-reduce of per-rank mean gradients is the batch mean."""
    import oracle
    w = _global_batch()
    ref = oracle.layer_bwd(w)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_balanced_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    seqs = sorted(b for _, sq, _, _ in res for b in sq)
    assert seqs == list(range(w.B))
    assert len({len(sq) for _, sq, _, _ in res}) > 1             # the bins hold different sample counts
    for _, _, tok, grads in res:
        assert abs(tok - w.T / world) <= w.lengths.max()
        for k, rk in (("d_rab_pos", "d_rab_pos"), ("d_rab_time", "d_rab_time"), ("d_gamma", "dgamma"),
                      ("d_beta", "dbeta")):
            np.testing.assert_allclose(grads[k], ref[rk] / w.B, rtol=1e-12, atol=1e-14)
