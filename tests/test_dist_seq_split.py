"""Host logic of the sequence split on CPU (gloo, world size 2 and 3): each
rank runs `seq_split_fwd` on its own segment with CPU stand-ins for the three
library calls (built on the fp64 oracle), the (M, N) exchange goes through
the process group, and every rank's outputs and final state must equal one
oracle pass over the whole sequence.  A rank that raises, and a segment
handed to the wrong rank, are caught."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """Stand-ins for gdr_seg_fwd / gdr_seg_combine / gdr_seg_fixup (fp64)."""

    @staticmethod
    def seg_fwd(q, k, v, la, be):
        import oracle
        n = lambda t: t.double().numpy()
        B, T, H, dk = q.shape
        o0, N = oracle.gdr_fwd(n(q), n(k), n(v), n(la), n(be), None)
        eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
        qt, M = oracle.gdr_fwd(n(q), n(k), np.zeros((B, T, H, dk)), n(la), n(be), eye)
        return tuple(torch.from_numpy(x) for x in (o0, qt, N, M))

    @staticmethod
    def seg_combine(M_all, N_all, r, S0):
        S = torch.zeros_like(N_all[0]) if S0 is None else S0.double().clone()
        S_in = S.clone() if r == 0 else None
        for j in range(M_all.shape[0]):
            S = torch.einsum("bhij,bhjk->bhik", S, M_all[j]) + N_all[j]
            if j + 1 == r:
                S_in = S.clone()
        return S_in, S

    @staticmethod
    def seg_fixup(qt, S_in, o):
        o += torch.einsum("bhij,bthj->bthi", S_in, qt)
        return o


def _inputs(T, seed):
    sys.path.insert(0, ROOT)
    import synth
    return synth.gdr_inputs(2, T, 2, 8, 6, "f32", seed=seed, s0_std=0.3)


def _bounds(T, world):
    cuts = [0] + [T * (i + 1) // world + (i % 2) * 5 for i in range(world - 1)] + [T]
    return cuts


def _worker(rank, world, port, T, seed, out, swap):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from gated_delta_rule_91_b200.seq_split import seq_split_fwd
    x = _inputs(T, seed)
    cuts = _bounds(T, world)
    seg = rank if not swap else (world - 1 - rank)  # swap: a segment on the wrong rank
    a, b = cuts[seg], cuts[seg + 1]
    sl = {n: x[n][:, a:b].double() for n in ("q", "k", "v", "log_alpha", "beta")}
    o, S_T = seq_split_fwd(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["beta"], x["S0"].double(),
                           ops=OracleOps)
    out[rank] = (seg, o.numpy(), S_T.numpy())
    dist.destroy_process_group()


def _run(world, T, seed, swap=False):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, T, seed, out, swap), nprocs=world, join=True)
        return dict(out)


def _reference(T, seed):
    import oracle
    x = _inputs(T, seed)
    n = lambda t: t.double().numpy()
    return oracle.gdr_fwd(n(x["q"]), n(x["k"]), n(x["v"]), n(x["log_alpha"]), n(x["beta"]), n(x["S0"]))


@pytest.mark.parametrize("world,T", [(2, 150), (3, 97)])
def test_split_sequence_equals_one_pass(world, T):
    res = _run(world, T, seed=world)
    o_ref, S_ref = _reference(T, world)
    cuts = _bounds(T, world)
    for rank, (seg, o, S_T) in res.items():
        np.testing.assert_allclose(o, o_ref[:, cuts[seg]:cuts[seg + 1]], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(S_T, S_ref, rtol=1e-10, atol=1e-12)


def test_segment_on_the_wrong_rank_is_detected():
    # ranks must hold consecutive segments in rank order; swapped segments
    # give a different (wrong) composition, which the comparison catches
    world, T = 2, 150
    res = _run(world, T, seed=7, swap=True)
    o_ref, _ = _reference(T, 7)
    cuts = _bounds(T, world)
    seg, o, _ = res[0]
    assert not np.allclose(o, o_ref[:, cuts[seg]:cuts[seg + 1]], rtol=1e-6, atol=1e-8)


def _failing_worker(rank, world, port):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=20))
    from gated_delta_rule_91_b200.seq_split import seq_split_fwd

    class Broken(OracleOps):
        @staticmethod
        def seg_fwd(*a):
            raise RuntimeError("segment forward failed")

    x = _inputs(40, 1)
    sl = {n: x[n][:, rank * 20:(rank + 1) * 20].double() for n in ("q", "k", "v", "log_alpha", "beta")}
    ops = Broken if rank == 1 else OracleOps
    try:
        seq_split_fwd(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["beta"], None, ops=ops)
    finally:
        dist.destroy_process_group()


def test_a_failing_rank_fails_the_job():
    port = _free_port()
    with pytest.raises(Exception):
        mp.spawn(_failing_worker, args=(2, port), nprocs=2, join=True)
