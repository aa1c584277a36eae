"""Multi-rank host logic with world_size 2 on the gloo backend (CPU)."""
import io
import os
import socket
from contextlib import redirect_stdout

import torch.multiprocessing as mp

from fp8_quantized_adam_b200 import ranks, workloads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, mode):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    try:
        ranks.init("gloo", timeout_s=20)
        if mode == "max":
            m = ranks.max_over_ranks(1.5 + rank)
            ranks.barrier()
            q.put((rank, m, ranks.shard_seed(3, rank)))
            ranks.finish()
        elif mode == "peer_exits":
            if rank == 1:
                return  # leaves between steps, before the collective
            try:
                ranks.max_over_ranks(1.0)
                q.put((rank, "no error"))
            except Exception as e:  # the surviving rank learns of it
                q.put((rank, "error:" + type(e).__name__))
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, "exception:%r" % e))


def _spawn(mode, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, mode)) for r in range(world)]
    for p in procs:
        p.start()
    out = []
    for _ in range(world if mode == "max" else 1):
        out.append(q.get(timeout=120))
    for p in procs:
        p.join(timeout=120)
    return out


def test_max_over_ranks_and_shard_seeds_world2():
    res = sorted(_spawn("max"))
    assert [r[1] for r in res] == [2.5, 2.5]  # every rank sees the max
    assert res[0][2] != res[1][2] and res[0][2] == 3  # distinct shards, rank 0 = the workload's seed


def test_rank_that_leaves_is_detected_by_its_peer():
    (rank, status), = _spawn("peer_exits")
    assert rank == 0 and status.startswith("error:")


def test_partition_covers_every_tensor_once_and_balances():
    specs = workloads.layout("llama2_7b")
    numels = [s.numel for s in specs]
    for world in (1, 2, 4, 8):
        parts = ranks.partition_by_numel(numels, world)
        flat = sorted(i for p in parts for i in p)
        assert flat == list(range(len(specs)))
        loads = [sum(numels[i] for i in p) for p in parts]
        assert max(loads) - min(loads) <= max(numels)


def test_reference_arm_prints_only_on_rank0(monkeypatch):
    import bench

    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.reference_arm(type("A", (), {"workload": "llama2_7b", "steps": 1, "warmup": 0, "gpus": 2})())
    assert buf.getvalue() == ""
