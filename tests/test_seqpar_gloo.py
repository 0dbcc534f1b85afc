"""The sequence split across ranks (selective_state_space_20_b200.seqpar) on
CPU with the gloo backend: each rank holds a shard of the timesteps; the
per-shard steps are replaced by fp64 stand-ins built on the oracle, so what
runs here is the exchange itself -- the all-gather of the shard summaries in
rank order and the fold of the shards before each rank.  Concatenated, the
ranks' outputs must equal the oracle's scan of the whole sequence, and the
last rank's state its final state (world sizes 2 and 3, with and without an
initial state)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(seed, batch=2, dim=5, L=96, N=4):
    rng = np.random.default_rng(seed)
    f = lambda x: torch.tensor(np.asarray(x, dtype=np.float32))  # noqa: E731
    return dict(u=f(rng.normal(size=(batch, dim, L))), delta=f(0.5 * rng.normal(size=(batch, dim, L))),
                A=f(-rng.uniform(0.2, 3.0, size=(dim, N))), B=f(rng.normal(size=(batch, N, L))),
                C=f(rng.normal(size=(batch, N, L))), D=f(rng.uniform(0.5, 1.5, size=dim)),
                z=f(rng.normal(size=(batch, dim, L))), delta_bias=f(rng.uniform(-3.0, -1.0, size=dim)))


def _cpu_ops():
    """fp64 stand-ins for the three per-shard steps (the oracle and numpy)."""
    import oracle

    def summary(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True):
        _, last = oracle.scan(u, delta, A, B, C, D=D, z=z, delta_bias=delta_bias, delta_softplus=delta_softplus)
        x = delta.double().numpy() + (0.0 if delta_bias is None else delta_bias.double().numpy()[None, :, None])
        dl = np.logaddexp(0.0, x) if delta_softplus else x
        return torch.tensor(dl.sum(axis=-1)), torch.tensor(last)

    def initial(A, all_sums, all_h, rank, h0=None):
        if rank == 0:
            return h0
        h = np.zeros(all_h.shape[1:]) if h0 is None else h0.double().numpy()
        a = A.double().numpy()[None, :, :]
        for k in range(rank):
            h = np.exp(a * all_sums[k].numpy()[:, :, None]) * h + all_h[k].numpy()
        return torch.tensor(h)

    def outputs(u, delta, A, B, C, h_in, D=None, z=None, delta_bias=None, delta_softplus=True, out=None):
        o, s = oracle.scan(u, delta, A, B, C, D=D, z=z, delta_bias=delta_bias, delta_softplus=delta_softplus,
                           h0=h_in)
        return torch.tensor(o), torch.tensor(s)

    return {"summary": summary, "initial": initial, "outputs": outputs}


def _worker(rank, world, port, seed, with_h0, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist
    from selective_state_space_20_b200 import seqpar
    dist.init_process_group("gloo", rank=rank, world_size=world)
    p = _problem(seed)
    L = p["u"].shape[-1]
    bounds = np.linspace(0, L, world + 1).astype(int)  # uneven shards are fine
    lo, hi = int(bounds[rank]), int(bounds[rank + 1])
    shard = {k: (v[..., lo:hi].contiguous() if k in ("u", "delta", "z", "B", "C") else v) for k, v in p.items()}
    h0 = torch.tensor(np.random.default_rng(seed + 1).normal(size=(2, 5, 4))) if with_h0 else None
    out, last = seqpar.scan_sequence_parallel(**shard, h0=h0, _ops=_cpu_ops())
    dist.destroy_process_group()
    q.put((rank, out.numpy(), last.numpy()))


@pytest.mark.parametrize("world,with_h0", [(2, False), (3, True)])
def test_sequence_split_matches_one_scan(world, with_h0):
    import oracle
    seed, port = 11 + world, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, seed, with_h0, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = dict((r, (o, s)) for r, o, s in (q.get(timeout=180) for _ in range(world)))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    p = _problem(seed)
    h0 = np.random.default_rng(seed + 1).normal(size=(2, 5, 4)) if with_h0 else None
    ro, rs = oracle.scan(**p, h0=h0)
    got = np.concatenate([res[r][0] for r in range(world)], axis=-1)
    assert got.shape == ro.shape
    assert np.max(np.abs(got - ro)) <= 1e-10 * max(1.0, np.max(np.abs(ro)))
    assert np.max(np.abs(res[world - 1][1] - rs)) <= 1e-10 * max(1.0, np.max(np.abs(rs)))


def _bench_worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    from selective_state_space_20_b200 import inputs
    w, r, _ = bench.dist_setup()
    wl = inputs.custom(1, 6, 64, 4, "fp32", seed=5, name="tiny split")
    ms, elems = bench.seqpar_run(wl, w, r, steps=2, warmup=1, device=torch.device("cpu"), ops=_cpu_ops())
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((r, ms, elems))


def test_bench_sequence_split_mode_two_ranks():
    """bench.py --seqpar's timing loop on two gloo ranks with the CPU
    stand-ins: every rank reports the same (maximum) time per step and the
    elements of the whole sequence."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_bench_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = {r: (ms, el) for r, ms, el in (q.get(timeout=10) for _ in range(world))}
    assert res[0] == res[1] and res[0][0] > 0 and res[0][1] == 1 * 6 * 64
