"""Host-side logic of bench.py without a GPU: the max-over-ranks timing on a
world-size-2 gloo process group, and the reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.max_over_ranks(1.5 + rank)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_max_over_ranks_single_process():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "3", "--ref-seconds", "2",
                        "--workload", "attn_B1_H16_L1024_d64"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TOPS" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["higher_is_better"] is True
    # a non-zero rank of a reference run exits quietly
    env = dict(os.environ, RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_variant_argument_checks():
    for extra in (["--method", "index", "--scale-block", "128"], ["--method", "decode", "--lsum", "codes"],
                  ["--q-path", "fused", "--scale-block", "64"], ["--scale-block", "64", "--lsum", "codes"],
                  ["--method", "index", "--p-levels", "255"], ["--scale-block", "64", "--p-levels", "255"],
                  ["--p-levels", "128"], ["--warmup", "2"]):
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *extra], capture_output=True,
                           text=True, timeout=120, cwd=ROOT)
        assert r.returncode != 0, extra


def test_kernel_hashes_per_method():
    sys.path.insert(0, ROOT)
    import bench
    hashes = {m: bench.kernel_sources_sha(m) for m in ("online", "index", "decode")}
    assert len(set(hashes.values())) == 3
    assert all(len(h) == 16 and int(h, 16) >= 0 for h in hashes.values())


def test_cpu_baseline_variants_run_the_oracle():
    sys.path.insert(0, ROOT)
    import bench
    from int8_quantized_attention_token_b200.workloads import by_name
    w = by_name("attn_B1_H1_L128_d64")
    for kw, word in (({}, "online"), ({"method": "index"}, "IndexSoftmax"), ({"blk": 64}, "block"),
                     ({"lcodes": True}, "online"), ({"p_levels": 255, "lcodes": True}, "online")):
        r = bench.cpu_baseline(w, budget_s=0.2, **kw)
        assert r["kind"] == "oracle" and r["value"] > 0 and word in r["sample"]
