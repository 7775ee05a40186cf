"""Host-side logic of bench.py, on CPU: byte models, the max-over-ranks
reduction across two gloo ranks, and the oracle (reference) arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_scan_bytes_130m():
    # 25.17M channel-tokens x (3 x 2 B in + 4 B out) + B/C + states + params
    n = bench.scan_bytes(8, 1536, 16, 2048, 2, 4)
    assert n == 8 * 1536 * 2048 * 10 + 8 * 2048 * 32 * 2 + 8 * 1536 * 16 * 4 + 1536 * 16 * 4 + 2 * 1536 * 4
    assert abs(n / 1e6 - 253.6) < 0.1


def test_decode_bytes():
    n = bench.decode_bytes(256, 5120, 16, 2, 4)
    assert abs(n / 1e6 - 181.3) < 0.1


def test_bwd_bytes_130m():
    # per channel-token: u, delta, z (bf16) + dout (fp32) read, du, ddelta, dz (fp32) written
    n = bench.bwd_bytes(8, 1536, 16, 2048, 2, 4)
    ct = 8 * 1536 * 2048
    assert n == (ct * (3 * 2 + 4 + 12) + 8 * 2048 * 32 * (2 + 4) + 8 * 1536 * 32 * 16 * 4
                 + 8 * 1536 * 16 * 4 + 2 * (1536 * 16 * 4 + 2 * 1536 * 4))
    assert abs(n / 1e6 - 583.0) < 0.1


def test_ssd_models():
    # x bf16 in, y fp32 out per (token, head, p); dt per (token, head); B, C per (token, group)
    n = bench.ssd_bytes(4, 2048, 80, 64, 128, 1, 2, 4)
    assert n == 4 * 2048 * 80 * (64 * 6 + 2) + 4 * 2048 * 2 * 128 * 2 + 3 * 80 * 4 + 4 * 80 * 64 * 128 * 4
    # per (b, h, 32-token chunk): C S (Q N P) + C B^T (Q Q N) + G' X (Q Q P) + B'^T X (N Q P), x2
    f = bench.ssd_flops(4, 2048, 80, 64, 128)
    per = 2 * (32 * 128 * 64 + 32 * 32 * 128 + 32 * 32 * 64 + 128 * 32 * 64)
    assert f == 4 * 80 * 64 * per


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    bench.init_dist(world, "gloo")
    v = bench.max_over_ranks(float(10 * (rank + 1)), world)
    bench.barrier(world)
    out[rank] = v
    torch.distributed.destroy_process_group()


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == 20.0 and out[1] == 20.0


def test_reference_arm_line():
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env,
                       timeout=120, cwd=ROOT)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_warmup_floor():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "1"])


def test_traffic_records_are_keyed_on_existing_kernel_sources():
    # every DRAM-traffic record names a kernel whose source list exists, so a
    # change to one kernel invalidates only that kernel's record
    import json
    for k, paths in bench.KERNEL_SOURCES.items():
        for p in paths + bench._SHARED_SOURCES:
            assert os.path.exists(os.path.join(bench.ROOT, p)), p
        assert len(bench.csrc_digest(k)) == 16
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        recs = json.load(f)
    assert set(recs) <= set(bench.KERNEL_SOURCES)
    for rec in recs.values():
        assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
