"""The N > 1 path of bench.py (independent weak-scaled replicas, job time = max over
ranks) on CPU with the gloo backend, world size 2."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 20.0][rank]
        m = bench.reduce_max(local_ms, torch.device("cpu"))
        v = bench.job_throughput(world, 10, m)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_two_rank_job_time_is_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in got:
        assert m == 20.0                          # the slowest rank sets the job time
        assert abs(v - 2 * 10 / 0.020) < 1e-9      # both replicas' steps over that time


def test_single_process_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5
    assert bench.job_throughput(1, 20, 10.0) == 2000.0


def test_reference_arm_non_zero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0 and p.stdout.strip() == ""


# ----------------------------------------------------------------------------
# sequence-sharded decode: the host side (shard ranges, shard lengths, the gather
# in rank order) with the float64 oracle as each rank's decode, world size 2 and 3
# ----------------------------------------------------------------------------
def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import numpy as np
    from long_context_decoding_eta_b200 import synth
    from long_context_decoding_eta_b200.sharded import gather_parts, shard_lengths, shard_range
    from oracle import eta_oracle as O
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.TINY.with_(B=2, ctx=1024, seed=95)
        g = synth.generate(w, "cpu", lengths=torch.tensor([1000, 333], dtype=torch.int32))
        K, V, qq = (g[k].double().numpy() for k in ("K", "V", "q"))
        scale = O.default_scale(w.d)
        tau = O.predict_tau(qq, g["W"].double().numpy(), np.full(w.Hq, 0.3))
        t0, t1 = shard_range(w.ctx, w.blk, world, rank)
        Ls = shard_lengths(g["lengths"], t0, t1).numpy().astype(np.int64)
        meta = O.cache_meta(K[:, :, t0:t1], Ls, w.blk)
        sc = O.screen(qq, tau, meta, scale)
        o, lse = O.decode(qq, tau, K[:, :, t0:t1], V[:, :, t0:t1], Ls, sc["union_idx"], w.blk,
                          scale, 0.05)
        o_parts, lse_parts = gather_parts(torch.from_numpy(o), torch.from_numpy(lse))
        om, lm = O.lse_merge(o_parts.numpy(), lse_parts.numpy())
        L = g["lengths"].numpy().astype(np.int64)
        mf = O.cache_meta(K, L, w.blk)
        sf = O.screen(qq, tau, mf, scale)
        o_ref, lse_ref = O.decode(qq, tau, K, V, L, sf["union_idx"], w.blk, scale, 0.05)
        q.put((rank, (t0, t1), float(np.abs(om - o_ref).max()), float(np.abs(lm - lse_ref).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_sharded_decode_host_path(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    ranges = [r[1] for r in got]
    assert ranges[0][0] == 0 and ranges[-1][1] == 1024            # the shards tile the cache
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    for rank, rng, eo, el in got:
        assert eo < 1e-10 and el < 1e-10, (rank, eo, el)


def test_shard_range_and_lengths():
    sys.path.insert(0, ROOT)
    from long_context_decoding_eta_b200.sharded import shard_lengths, shard_range
    for T_max, blk, world in ((4096, 64, 3), (1024, 128, 8), (640, 64, 4)):
        rs = [shard_range(T_max, blk, world, r) for r in range(world)]
        assert rs[0][0] == 0 and rs[-1][1] == T_max
        assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
        assert all(t0 % blk == 0 and t1 % blk == 0 for t0, t1 in rs)
        lens = torch.tensor([0, 1, T_max - 1, T_max, blk * 3 + 5], dtype=torch.int32)
        tot = sum(shard_lengths(lens, t0, t1).to(torch.int64) for t0, t1 in rs)
        assert torch.equal(tot, lens.to(torch.int64))
    with pytest.raises(ValueError):
        shard_range(100, 64, 2, 0)


def test_clock_sampler_without_nvidia_smi_reports_unavailable(tmp_path, monkeypatch):
    """On a host without nvidia-smi the sampler records nothing and says so."""
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setattr(bench, "CLOCK_LOG_DIR", str(tmp_path))
    monkeypatch.setenv("PATH", str(tmp_path))          # no nvidia-smi on this PATH
    with bench.Clocks(0) as clk:
        pass
    assert clk.summary()["reasons"] == ["unavailable"]


def test_operating_point_overrides():
    """--density / --density-kind / --tau-mode change only what they name, and the
    default run keeps the workload as defined."""
    import types
    sys.path.insert(0, ROOT)
    import bench
    base = bench.workload_by_name("long")
    none = types.SimpleNamespace(density=0.0, density_kind="", tau_mode="")
    assert bench.with_overrides(base, none) is base
    pt = types.SimpleNamespace(density=0.38, density_kind="head", tau_mode="")
    w = bench.with_overrides(base, pt)
    assert (w.density, w.density_kind, w.tau_mode) == (0.38, "head", base.tau_mode)
    assert (w.B, w.ctx, w.blk, w.seed) == (base.B, base.ctx, base.blk, base.seed)
    assert w.name != base.name
