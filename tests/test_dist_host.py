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


def _shard_rank_main(rank: int, world: int, port: int, q):
    """One rank of a problem split by (batch, KV head): the rank's pairs through the oracle."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import math
    import oracle
    from quantized_kv_cache_19_b200 import shard
    from quantized_kv_cache_19_b200.workloads import WORKLOADS, make_inputs
    torch.distributed.init_process_group("gloo")
    try:
        w = _shard_workload(WORKLOADS)
        x = {k: v.float().numpy() for k, v in make_inputs(w, device="cpu").items()}
        start, stop = shard.pair_ranges(w.B * w.Hkv, world)[rank]
        part = shard.shard_inputs(x, w.B, w.Hq, w.Hkv, start, stop)
        O = L = None
        if stop > start:
            cache = oracle.build_cache(part["K_src"], part["V_src"], w.bits, w.group, w.meta)
            O, L = oracle.corrected_attention(part["Q"], cache, part["K_cur"], part["V_cur"], correct=1,
                                              causal=w.causal, scale=1.0 / math.sqrt(w.d))
        got = [None] * world
        torch.distributed.all_gather_object(got, (start, stop, O, L))
        if rank == 0:
            q.put(got)
    finally:
        torch.distributed.destroy_process_group()


def _shard_workload(WORKLOADS):
    # GQA (two query heads per KV head), three batches of three KV heads: nine pairs over the ranks
    return WORKLOADS["prefill_gqa"].with_(B=3, Hq=6, Hkv=3, d=64, group=32, Lq=5, Lcur=7, Lc=40, seed=77)


@pytest.mark.parametrize("n_pairs,world", [(9, 2), (32, 8), (3, 4), (0, 2), (1, 1), (130, 7)])
def test_pair_ranges_cover_every_pair_once(n_pairs, world):
    sys.path.insert(0, ROOT)
    from quantized_kv_cache_19_b200 import shard
    ranges = shard.pair_ranges(n_pairs, world)
    assert len(ranges) == world
    seen = [i for a, b in ranges for i in range(a, b)]
    assert seen == list(range(n_pairs))
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1


def test_stitch_rejects_gaps_and_overlaps():
    sys.path.insert(0, ROOT)
    import numpy as np
    from quantized_kv_cache_19_b200 import shard
    a = np.zeros((2, 1, 3))
    with pytest.raises(ValueError):
        shard.stitch([(0, 2, a), (3, 5, a)], B=1, Hq=5, Hkv=5, concat=np.concatenate)
    with pytest.raises(ValueError):
        shard.stitch([(0, 2, a), (1, 3, a)], B=1, Hq=3, Hkv=3, concat=np.concatenate)
    with pytest.raises(ValueError):
        shard.stitch([(0, 2, a)], B=1, Hq=3, Hkv=3, concat=np.concatenate)


def test_two_gloo_ranks_split_one_problem_by_kv_head():
    """Two ranks each take a contiguous half of the (batch, KV head) pairs of one problem, with no
    exchange during the computation; the outputs put back in order equal the single-process
    oracle's on the whole problem."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_shard_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    parts = q.get(timeout=180)          # read before joining: a child exits once its data is taken
    for p in procs:
        p.join(timeout=60)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    sys.path.insert(0, ROOT)
    import math
    import numpy as np
    import oracle
    from quantized_kv_cache_19_b200 import shard
    from quantized_kv_cache_19_b200.workloads import WORKLOADS, make_inputs
    w = _shard_workload(WORKLOADS)
    assert [(a, b) for a, b, _, _ in parts] == [(0, 4), (4, 9)]
    O = shard.stitch([(a, b, o) for a, b, o, _ in parts], w.B, w.Hq, w.Hkv, np.concatenate)
    L = shard.stitch([(a, b, l) for a, b, _, l in parts], w.B, w.Hq, w.Hkv, np.concatenate)
    x = {k: v.float().numpy() for k, v in make_inputs(w, device="cpu").items()}
    cache = oracle.build_cache(x["K_src"], x["V_src"], w.bits, w.group, w.meta)
    O_ref, L_ref = oracle.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1,
                                              causal=w.causal, scale=1.0 / math.sqrt(w.d))
    assert O.shape == O_ref.shape and L.shape == L_ref.shape
    np.testing.assert_allclose(O, O_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(L, L_ref, rtol=1e-12, atol=1e-12)
