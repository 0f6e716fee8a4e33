"""Host logic of the multi-rank bench on CPU: two gloo ranks, as `torchrun --nproc-per-node 2` would
start them. The path shards by (batch, KV head) with no exchange, so the only collectives are the
barrier around the timed region and the max over ranks of the measured times."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    try:
        w, r, local = bench.dist_setup()
        assert (w, r, local) == (world, rank, rank)
        assert torch.distributed.get_backend() == "gloo"
        bench.barrier(w)
        # each rank reports its own time; every rank must get the slowest one
        got = bench.reduce_max(1.5 + 2.0 * rank, w, "cpu")
        # the reference arm runs on rank 0 only; the others return without work
        class A:
            workload, steps, warmup = "tiny_f32", 1, 3
        ref = bench.run_reference(A, w, r) if r != 0 else "skipped"
        bench.barrier(w)
        q.put((rank, got, ref))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_barrier_and_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    out = sorted(q.get(timeout=5) for _ in range(world))
    assert [o[1] for o in out] == [3.5, 3.5]          # max over ranks, on every rank
    assert out[1][2] is None                           # rank 1 does no reference work


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        assert k not in os.environ or os.environ[k] in ("0", "1")
    assert bench.reduce_max(2.5, 1, "cpu") == 2.5
    bench.barrier(1)


def test_traffic_entry_goes_stale_with_the_source(tmp_path, monkeypatch):
    """A stored ncu figure is reported only for the kernel sources it was captured from."""
    sys.path.insert(0, ROOT)
    import json
    import bench
    f = tmp_path / "traffic.json"
    good = bench.source_hash("corrected_attention_kernel")
    f.write_text(json.dumps({"corrected_attention_kernel": {
        "w_ok": {"dram_bytes_per_launch": 123, "source_sha256": good, "command": "c"},
        "w_old": {"dram_bytes_per_launch": 456, "source_sha256": "0" * 64, "command": "c"}}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.ncu_traffic("corrected_attention_kernel", "w_ok") == 123
    assert bench.ncu_traffic("corrected_attention_kernel", "w_old") is None
    assert bench.ncu_traffic("corrected_attention_kernel", "missing") is None
    assert bench.ncu_traffic("quantize_append_kernel", "w_ok") is None
