"""The multi-GPU form of the benchmark is N independent replicas (the layer
has no exchange step): every rank times its own copy of the path, the ranks
meet at barriers around the timed region, and rank 0 reports the slowest
rank's time. This checks that host logic with world_size 2 on CPU (gloo),
including a rank that is slower than the other and a rank that fails."""
import multiprocessing as mp
import os
import socket


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, q, fail_rank):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    try:
        w, r, local = bench.dist_env()
        assert (w, r, local) == (world, rank, rank)
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=5))
        bench.barrier(world)
        if rank == fail_rank:
            raise RuntimeError("planted failure on the host")
        got = bench.max_over_ranks(values[rank], world, torch.device("cpu"))
        bench.barrier(world)
        q.put((rank, "ok", got))
    except Exception as e:  # reported to the parent, never a hang
        q.put((rank, "error", repr(e)))
    finally:
        if dist.is_initialized():
            try:
                dist.destroy_process_group()
            except Exception:
                pass


def _run(values, fail_rank=-1, timeout=60):
    world = len(values)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, values, q, fail_rank)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        rank, kind, val = q.get(timeout=timeout)
        out[rank] = (kind, val)
    for p in procs:
        p.join(timeout=timeout)
        if p.is_alive():
            p.kill()
    return out


def test_max_over_ranks_takes_the_slowest_replica():
    out = _run([0.25, 0.31])
    assert out[0] == ("ok", 0.31) and out[1] == ("ok", 0.31)


def test_a_failing_rank_ends_the_other_with_an_error_not_a_hang():
    out = _run([0.25, 0.31], fail_rank=1)
    assert out[1][0] == "error" and "planted failure" in out[1][1]
    assert out[0][0] == "error"     # its collective timed out or saw the peer leave


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(1.5, 1, None) == 1.5
    bench.barrier(1)
