"""The multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2, 127.0.0.1).

The layer shards by image: each rank owns B distinct images of the seeded stream and the ranks
exchange nothing on the data path.  What the ranks do share is host plumbing: the max over ranks
of the timed region, the whole-job throughput, and the reference arm that only rank 0 runs.
"""
import contextlib
import io
import json
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    from pooled_selective_scan_b200 import inputs, workload
    from pooled_selective_scan_b200.configs import by_name

    res = {}
    # max over ranks of a per-rank time
    res["max"] = bench.reduce_max(1.25 + rank)
    # image shards: disjoint, covering the global batch, built from the global ids
    cfg = by_name("fastvim_t_224_tiny")
    mine = workload.shard_images(cfg, rank, WORLD)
    got = [None] * WORLD
    dist.all_gather_object(got, list(mine))
    res["shards"] = got
    t = workload.layer_tensors(cfg, "cpu", first_image=mine.start)
    shp = inputs.token_shape(cfg)
    res["x_matches_global_ids"] = all(
        np.array_equal(t["x"][i].numpy(), inputs.image_x(cfg.seed, mine.start + i, shp)) for i in range(cfg.B))
    res["z_matches_global_ids"] = all(
        np.array_equal(t["z"][i].numpy(), inputs.image_z(cfg.seed, mine.start + i, shp)) for i in range(cfg.B))
    # the reference arm: rank 0 alone runs the oracle and prints one line; the others exit 0
    a = bench.parse(["--impl", "reference", "--gpus", str(WORLD), "--steps", "1", "--warmup", "3",
                     "--config", "fastvim_t_224_tiny"])
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.run_reference(a, cfg, cfg.pool_axes[0])
    res["ref_rc"] = rc
    res["ref_out"] = buf.getvalue()
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    out = tmp_path_factory.mktemp("ranks")
    mp.start_processes(rank_main, args=(free_port(), str(out)), nprocs=WORLD, join=True, start_method="spawn")
    return [json.load(open(out / f"rank{r}.json")) for r in range(WORLD)]


def test_max_over_ranks(results):
    assert [r["max"] for r in results] == [2.25, 2.25]


def test_image_shards_are_disjoint_and_cover_the_global_batch(results):
    B = 2  # batch of the tiny 224 px workload
    for r in results:
        assert r["shards"] == [[0, 1], [2, 3]]
        assert sorted(sum(r["shards"], [])) == list(range(WORLD * B))
        assert r["x_matches_global_ids"] and r["z_matches_global_ids"]


def test_reference_arm_runs_on_rank_zero_only(results):
    assert all(r["ref_rc"] == 0 for r in results)
    assert results[1]["ref_out"] == ""
    lines = [ln for ln in results[0]["ref_out"].splitlines() if ln.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["n_gpus"] == WORLD and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle"
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0


def test_whole_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.weak_scaling_value(1000, 4, 0.5) == 8000.0
    assert bench.weak_scaling_value(1000, 1, 0.5) == 2000.0
