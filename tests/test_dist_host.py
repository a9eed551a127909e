"""Host-side multi-rank logic of the benchmark on CPU with gloo, world size 2: the
per-step time is the maximum over ranks, and the reference arm runs on rank 0 only.
Ranks are spawned processes (no GPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    got = bench.max_over_ranks(10.0 + 5.0 * rank)
    w, r, l = bench.dist_setup()

    class A:
        gpus, steps, warmup = world, 1, 0

    # the reference arm returns immediately without work on ranks other than 0
    ref_rc = bench.run_reference(A, None) if rank != 0 else 0
    out.put((rank, got, (w, r, l), ref_rc))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_rank_roles_with_gloo():
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
    assert [r[1] for r in res] == [15.0, 15.0]
    assert [r[2] for r in res] == [(2, 0, 0), (2, 1, 1)]
    assert res[1][3] == 0


def test_single_process_max_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5


def test_attention_traffic_record_follows_the_kernel_source(tmp_path):
    """The roofline's DRAM traffic comes from the committed ncu record only while the
    attention kernel's source is the one it was captured from; any edit voids it."""
    import hashlib
    import json
    import bench
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = os.path.join(root, "free_sparse_attention_b200", "csrc", "attention_tc.cu")
    with open(os.path.join(root, "profiles", "attn_tc_hunyuan720p.json")) as f:
        rec = json.load(f)
    # per launch = captured bytes scaled from the captured heads to the 24-head layer
    assert rec["dram_bytes_per_launch"] == rec["dram_bytes_captured"] * 24 / rec["captured_heads"]
    with open(src, "rb") as f:
        body = f.read()
    got = bench.traffic_from_profile(src)
    if hashlib.sha256(body).hexdigest() == rec["kernel_sha256"]:
        assert got == rec["dram_bytes_per_launch"]
    else:
        assert got is None
    changed = tmp_path / "attention_tc.cu"
    changed.write_bytes(body + b"\n")
    assert bench.traffic_from_profile(str(changed)) is None
