"""Multi-rank path on CPU (gloo, world size 2): canvases sharded across ranks
with global canvas offsets give the same trajectories as one process, and the
timing reduction takes the maximum over ranks."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shard(B, world, rank):
    base, extra = divmod(B, world)
    return rank * base + min(rank, extra), base + (1 if rank < extra else 0)


def _trajectory(offset, count, B, L, V, steps, seed):
    """Oracle trajectory of canvases offset .. offset+count-1 (global indices)."""
    import oracle as O
    import synth
    w = synth.WORKLOADS["tiny"].replace(B=B, L=L, V=V, num_steps=steps, seed=seed)
    cfg = O.Config(B=count, L=L, V=V, group_size=64, canvas_offset=offset, **w.sampler_config())
    st = O.State(cfg).init()
    for s in range(steps):
        lg = synth.generate_host(w, s, b0=offset, nb=count)
        for i in range(count):
            O.step_canvas(st, i, lg[i], s)
    return st


def _worker(rank, world, port, B, L, V, steps, seed, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        off, cnt = _shard(B, world, rank)
        st = _trajectory(off, cnt, B, L, V, steps, seed)
        # gather variable-size shards through fixed-size padded buffers
        pad = (B + world - 1) // world
        cv = torch.full((pad, L), -1, dtype=torch.int32)
        cm = torch.zeros((pad, L), dtype=torch.uint8)
        sp = torch.zeros((pad,), dtype=torch.uint8)
        cv[:cnt] = torch.from_numpy(st.canvas)
        cm[:cnt] = torch.from_numpy(st.committed)
        sp[:cnt] = torch.from_numpy(st.stop)
        outs = [[torch.empty_like(t) for _ in range(world)] for t in (cv, cm, sp)]
        for o, t in zip(outs, (cv, cm, sp)):
            dist.all_gather(o, t)
        # max-over-ranks timing reduction as bench.py does it
        t = torch.tensor([10.0 + rank], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            res = []
            for r in range(world):
                o, c = _shard(B, world, r)
                res.append((outs[0][r][:c].numpy(), outs[1][r][:c].numpy(), outs[2][r][:c].numpy()))
            q.put((res, float(t.item())))
    finally:
        dist.destroy_process_group()


def test_sharded_oracle_trajectories_match_single_process():
    B, L, V, steps, seed, world = 5, 16, 700, 10, 3, 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, B, L, V, steps, seed, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res, tmax = q.get(timeout=300)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert tmax == 10.0 + world - 1
    full = _trajectory(0, B, B, L, V, steps, seed)
    cv = np.concatenate([r[0] for r in res])
    cm = np.concatenate([r[1] for r in res])
    sp = np.concatenate([r[2] for r in res])
    assert np.array_equal(cv, full.canvas)
    assert np.array_equal(cm, full.committed)
    assert np.array_equal(sp, full.stop)


# ----------------------------------------------------------------------------- vocabulary slices

def _slice_worker(rank, world, port, L, V, bounds, seed, q):
    """Rank r owns vocabulary slice r: its per-position slice records, all-gathered
    in rank (= slice) order, combine to the full-vocabulary results on every rank."""
    import oracle as O
    import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.WORKLOADS["tiny"].replace(B=1, L=L, V=V, seed=seed)
        cfg = O.Config(B=1, L=L, V=V, group_size=64, **w.sampler_config())
        lg = synth.generate_host(w, 3, b0=0, nb=1)[0]  # the full row set; each rank reads its slice
        lo, hi = bounds[rank], bounds[rank + 1]
        inv_T = 1.0 / O.temperature(cfg, 3)
        rec = torch.zeros((L, 6), dtype=torch.float64)
        for l in range(L):
            sl = O.slice_record(cfg, np.ascontiguousarray(lg[l, lo:hi]), lo, inv_T, 0, l, 3)
            rec[l] = torch.tensor([sl.S, sl.W, sl.zmax, sl.gscore, sl.amax, sl.sample],
                                  dtype=torch.float64)
        allr = [torch.empty_like(rec) for _ in range(world)]
        dist.all_gather(allr, rec)
        out = []
        for l in range(L):
            slices = []
            for r in range(world):
                v = allr[r][l].tolist()
                slices.append(O.Slice(S=v[0], W=v[1], zmax=v[2], gscore=v[3], amax=int(v[4]),
                                      sample=int(v[5])))
            out.append(O.combine_slices(slices, inv_T))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_vocabulary_sharded_records_combine_to_the_full_row():
    import oracle as O
    import synth
    L, V, seed, world = 8, 640, 5, 2
    bounds = [0, 256, 640]
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_slice_worker, args=(r, world, port, L, V, bounds, seed, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1]  # every rank combines to the same results
    w = synth.WORKLOADS["tiny"].replace(B=1, L=L, V=V, seed=seed)
    cfg = O.Config(B=1, L=L, V=V, group_size=64, **w.sampler_config())
    lg = synth.generate_host(w, 3, b0=0, nb=1)[0]
    inv_T = 1.0 / O.temperature(cfg, 3)
    for l in range(L):
        H, pm, am, x = res[0][l]
        H0, pm0, am0, _ = O.row_stats(lg[l], inv_T)
        x0, margin, _ = O.sample(cfg, lg[l], inv_T, 0, l, 3)
        assert am == am0 and abs(H - H0) < 1e-12 and abs(pm - pm0) < 1e-12
        if margin > 1e-9:
            assert x == x0
