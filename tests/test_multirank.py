"""World-size-2 gloo check (CPU) of the benchmark's multi-rank timing rule:
every rank's device time is gathered, the slowest rank's time divides all
ranks' work (weak scaling, no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ms = [100.0, 125.0][rank]          # rank 1 is the slow one
    all_ms = bench.gather_floats(ms, world)
    value, ms_per_step = bench.aggregate(all_ms, [3.5e12 * 10] * world, 10)
    q.put((rank, all_ms, value, ms_per_step))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, all_ms, value, ms_per_step in res:
        assert all_ms == [100.0, 125.0]
        assert ms_per_step == 12.5
        assert value == pytest.approx(2 * 3.5e13 / 0.125)


def _ulysses_worker(rank, world, port, q):
    """gloo ranks on CPU: the Ulysses exchanges around a CPU attention (the
    oracle's, injected; the library's own kernels need the GPU) and the sharded
    gate decision, against the unsharded results."""
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from oracle import attention as A
    from oracle import gate as G
    from diffusion_transformer_denoising_dit_b200 import synth, ulysses
    try:
        import dataclasses
        w = dataclasses.replace(synth.WORKLOADS["tiny"], H=4)     # 4 heads, 288 tokens, d = 64
        qf, kf, vf = synth.qkv(w)                                   # the whole sequence (same on every rank)
        pos = synth.positions(w.T, w.G)
        n = w.N // world
        sl = slice(rank * n, (rank + 1) * n)
        qs, ks, vs = (t[:, :, sl].contiguous().float() for t in (qf, kf, vf))
        # round trip and layout
        heads = ulysses.seq_to_head(qs)
        hp = w.H // world
        ok_layout = torch.equal(heads, qf[:, rank * hp:(rank + 1) * hp].float())
        ok_round = torch.equal(ulysses.head_to_seq(heads), qs)
        # attention: the oracle on head shards, exchanged back
        def attend(q, k, v, cos, sin):
            return torch.from_numpy(A.attention(q, k, v, pos=pos.numpy(), axes=w.axes, theta=w.theta))
        o = ulysses.attention(qs.double(), ks.double(), vs.double(), attend=attend)
        full = A.attention(qf, kf, vf, pos=pos.numpy(), axes=w.axes, theta=w.theta)
        err = float(np.abs(o.numpy() - full[:, :, sl]).max())
        # the overlapped form, head chunk by head chunk: the same result bit for bit
        for chunks in [c for c in (1, 2, 4) if (w.H // world) % c == 0]:
            oo = ulysses.attention_overlapped(qs.double(), ks.double(), vs.double(), attend=attend, chunks=chunks)
            err = max(err, float((oo - o).abs().max()) * 1e12)
        # sharded gate: shard totals, all-reduce, one decision everywhere
        cur, prev = synth.gate_pair(288, 128, 0.1)
        m = 288 // world
        rows = slice(rank * m, (rank + 1) * m)

        def sums(a, b):
            a64, b64 = a.double(), b.double()
            return torch.tensor([float((a64 - b64).abs().sum()), float(b64.abs().sum())], dtype=torch.float64)

        def finalize(t, thr):
            rel = float(t[0] / t[1])
            return rel, rel < thr

        rel, skip = ulysses.gate(cur[rows], prev[rows], 0.12, sums=sums, finalize=finalize)
        ref_rel = G.relative_l1(cur, prev)
        q.put((rank, ok_layout, ok_round, err, rel, skip, ref_rel))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_exchange_and_sharded_gate(world):
    """2 and 4 gloo ranks (4 heads: 2 or 1 per rank; 288 tokens: 144 or 72 per rank)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ulysses_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=200) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [r[0] for r in res] == list(range(world))
    for rank, ok_layout, ok_round, err, rel, skip, ref_rel in res:
        assert ok_layout and ok_round
        assert err < 1e-12
        assert abs(rel - ref_rel) < 1e-12 * max(1.0, ref_rel)
        assert skip == (ref_rel < 0.12)
    assert len({r[4] for r in res}) == 1  # every rank holds the same rel
