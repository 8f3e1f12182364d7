"""World-size-2 gloo test of the weak-scaling host logic that bench.py runs
(long_context_rope_b200.dist_util.Dist, with gloo instead of NCCL): the
process group comes up from the torchrun environment variables, each rank
draws its own sequence (different seeds), the barrier passes, times are
reduced with a max over ranks, and the whole-job rate counts every rank's
tokens."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    from long_context_rope_b200 import dist_util, synth
    d = dist_util.Dist("gloo", timeout_s=60)
    try:
        seed = d.seed(0)
        w = synth.WORKLOADS["tiny_f32"]
        x = synth.draw(w, seed=seed)
        first = float(x["k_raw"][0, 0, 0, 0])
        d.barrier()
        t = d.max(1.0 + rank)
        rate = dist_util.whole_job_rate(w.seq_len, t, d.world)
        q.put((d.rank, seed, first, t, rate))
    finally:
        d.close()


def test_weak_scaling_host_logic_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, f0, t0, rate0), (r1, s1, f1, t1, rate1) = res
    assert (r0, r1) == (0, 1)
    assert s0 != s1 and f0 != f1          # independent sequences
    assert t0 == t1 == 2.0                # max over ranks
    assert rate0 == rate1 == 2 * 1024 / 2.0


def test_single_process_is_identity(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    from long_context_rope_b200 import dist_util
    d = dist_util.Dist("gloo")
    assert (d.world, d.rank, d.active) == (1, 0, False)
    assert d.max(3.5) == 3.5
    d.barrier()
    d.close()
