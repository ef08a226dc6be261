"""Multi-rank host logic on CPU ranks (gloo), no GPU.

  * bench.py's replica timing: the barrier and the max over ranks that
    every rank takes part in;
  * bench.py --impl reference under torchrun with two ranks: rank 0 alone
    runs the oracle and prints one JSON line, the other rank exits 0;
  * the sequence split (linear_attention_simple_b200.seqpar) over 2, 3 and 4
    ranks, with an oracle-backed set of per-segment calls standing in for
    libgla's kernels, against the oracle run on the unsplit sequence.  This
    checks the exchange, the rank order and the direction of each fold; the
    kernels themselves are checked on the GPU (tests/test_gpu_seqpar.py).
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from linear_attention_simple_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _entry(rank, world, port, fn, args):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        fn(rank, world, *args)
    finally:
        dist.destroy_process_group()


def _spawn(fn, world, *args):
    mp.spawn(_entry, args=(world, _free_port(), fn, args), nprocs=world, join=True)


# ------------------------------------------------------------ bench replicas

def _bench_helpers(rank, world):
    import bench
    bench.barrier(world)
    # every rank sees the slowest rank's time
    assert bench.max_over_ranks(0.25 * (rank + 1), world, device="cpu") == 0.25 * world
    assert bench.max_over_ranks(-1.0 * rank, world, device="cpu") == 0.0
    bench.barrier(world)


@pytest.mark.parametrize("world", [2, 3])
def test_bench_barrier_and_max_over_ranks(world):
    _spawn(_bench_helpers, world)


def test_bench_reference_arm_two_ranks():
    env = dict(os.environ, GLA_ORACLE_UNITS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


# ------------------------------------------------------ sequence split

class OracleOps:
    """The per-segment calls of seqpar, on the host in fp64 (test only)."""

    @staticmethod
    def segment_state_fwd(k, v, a):
        from oracle import recurrent
        kk, vv, aa = k.numpy(), v.numpy(), a.numpy()
        _, s = recurrent.fwd(np.zeros_like(kk), kk, vv, aa)
        return torch.from_numpy(s), torch.from_numpy(aa.sum(axis=1))

    @staticmethod
    def segment_state_bwd(q, dO, a, scale):
        from oracle import recurrent
        qq, gg = q.numpy(), dO.numpy()
        ds = recurrent.bwd(qq, np.zeros_like(qq), np.zeros_like(gg), a.numpy(), gg, scale=scale)[4]
        return torch.from_numpy(ds)

    @staticmethod
    def state_fold(s, g, reverse, s_in):
        x = torch.zeros(s.shape[1:], dtype=s.dtype) if s_in is None else s_in.clone()
        order = range(s.shape[0] - 1, -1, -1) if reverse else range(s.shape[0])
        for j in order:
            x = torch.exp(g[j])[..., None, None] * x + s[j]
        return x

    @staticmethod
    def chunk_fwd(q, k, v, a, s0, scale):
        from oracle import recurrent
        o, _ = recurrent.fwd(q.numpy(), k.numpy(), v.numpy(), a.numpy(),
                             None if s0 is None else s0.numpy(), scale=scale)
        return torch.from_numpy(o)

    @staticmethod
    def chunk_bwd(q, k, v, a, dO, s0, ds_final, scale):
        from oracle import recurrent
        g = recurrent.bwd(q.numpy(), k.numpy(), v.numpy(), a.numpy(), dO.numpy(),
                          None if s0 is None else s0.numpy(),
                          None if ds_final is None else ds_final.numpy(), scale=scale)
        return tuple(torch.from_numpy(x) for x in g[:4])


def _seq_inputs(lengths):
    B, H, dk, dv = 2, 3, 5, 4
    d = inputs.chunk_inputs(B, sum(lengths), H, dk, dv, dtype=torch.float64, seed=77, s0_std=0.3,
                            with_dO=True)
    d["a"] = d["a"].double()
    d["dsT"] = inputs.randn((B, H, dk, dv), 78, std=0.3, dtype=torch.float64)
    return d


def _seqpar_rank(rank, world, lengths):
    from linear_attention_simple_b200 import seqpar
    from oracle import recurrent
    d = _seq_inputs(lengths)
    lo = sum(lengths[:rank])
    hi = lo + lengths[rank]
    mine = {n: d[n][:, lo:hi].contiguous() for n in ("q", "k", "v", "a", "dO")}
    o, s_final = seqpar.chunk_fwd_seqpar(mine["q"], mine["k"], mine["v"], mine["a"], s0=d["s0"],
                                         ops=OracleOps)
    full = [d[n].numpy() for n in ("q", "k", "v", "a", "dO")]
    ro, rs = recurrent.fwd(*full[:4], d["s0"].numpy())
    np.testing.assert_allclose(o.numpy(), ro[:, lo:hi], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(s_final.numpy(), rs, rtol=1e-9, atol=1e-11)

    grads = seqpar.chunk_bwd_seqpar(mine["q"], mine["k"], mine["v"], mine["a"], mine["dO"], s0=d["s0"],
                                    ds_final=d["dsT"], ops=OracleOps)
    ref = recurrent.bwd(*full, d["s0"].numpy(), d["dsT"].numpy())
    for g, r in zip(grads[:4], ref[:4]):
        np.testing.assert_allclose(g.numpy(), r[:, lo:hi], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(grads[4].numpy(), ref[4], rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("lengths", [[9, 14], [5, 0, 9], [1, 7, 3], [3, 0, 5, 2]])
def test_seqpar_split_over_gloo_ranks_matches_unsplit(lengths):
    _spawn(_seqpar_rank, len(lengths), lengths)
