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
    # per (b, h, 128-token chunk): C S (Q N P) + C B^T (Q Q N) + G' X (Q Q P) + B'^T X (N Q P), x2
    f = bench.ssd_flops(4, 2048, 80, 64, 128)
    per = 2 * (128 * 128 * 64 + 128 * 128 * 128 + 128 * 128 * 64 + 128 * 128 * 64)
    assert f == 4 * 80 * 16 * per


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


# ------------------------------------------------- (b, d) shard plan ----

def test_shard_ranges_cover_every_channel_once():
    from selective_state_space_40_b200 import shard
    for batch, dim, world in [(8, 1536, 2), (4, 5120, 8), (1, 2048, 8), (3, 100, 2), (1, 8, 4), (2, 40, 3)]:
        seen = {}
        for r in range(world):
            b0, b1, d0, d1 = shard.shard_range(batch, dim, world, r)
            assert d0 % 8 == 0 or d0 == d1
            for b in range(b0, b1):
                for d in range(d0, d1):
                    assert (b, d) not in seen
                    seen[(b, d)] = r
        assert len(seen) == batch * dim


def _shard_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import oracle
    from selective_state_space_40_b200 import binding as mb
    from selective_state_space_40_b200 import shard
    from selective_state_space_40_b200 import synthetic as syn

    bench.init_dist(world, "gloo")
    try:
        res = {}
        for batch, dim in ((4, 48), (3, 40)):  # batch rows split; channel blocks split
            w = syn.scaled(syn.M130, batch=batch, dim=dim, seqlen=96, in_dtype=torch.float32, seed=batch + dim)
            inp = syn.scan_inputs(w)
            inp["A"] = syn.a_matrix_varied(dim, 16, 5)
            full = dict(inp, y=torch.zeros(batch, dim, 96), initial_state=0.2 * torch.ones(batch, dim, 16),
                        last_state=torch.zeros(batch, dim, 16))
            v = shard.shard_views(full, batch, dim, world, rank)
            b0, b1, d0, d1 = shard.shard_range(batch, dim, world, rank)
            # the rank's C-ABI arguments: the full tensors' strides, offset pointers
            dims = mb.scan_dims_for(v["u"], v["delta"], v["B"], v["C"], v["z"], v["y"])
            assert (dims.batch, dims.dim) == (b1 - b0, d1 - d0)
            assert (dims.u_sb, dims.u_sd, dims.B_sb, dims.B_sn) == (full["u"].stride(0), full["u"].stride(1),
                                                                     full["B"].stride(0), full["B"].stride(1))
            assert v["u"].data_ptr() == full["u"].data_ptr() + (b0 * full["u"].stride(0) + d0 * full["u"].stride(1)) * 4
            assert v["A"].data_ptr() == full["A"].data_ptr() + d0 * 16 * 4
            # the rank's share through the oracle, gathered and reassembled
            f = lambda t: t.to(torch.float64).numpy()  # noqa: E731
            y, last = oracle.scan(f(v["u"]), f(v["delta"]), f(v["A"]), f(v["B"]), f(v["C"]), f(v["D"]), f(v["z"]),
                                  f(v["delta_bias"]), True, h0=f(v["initial_state"]))
            parts = [None] * world
            dist.all_gather_object(parts, (b0, b1, d0, d1, y, last))
            if rank == 0:
                yfull, lfull = oracle.scan(f(inp["u"]), f(inp["delta"]), f(inp["A"]), f(inp["B"]), f(inp["C"]),
                                           f(inp["D"]), f(inp["z"]), f(inp["delta_bias"]), True,
                                           h0=f(full["initial_state"]))
                ys = yfull * float("nan")
                ls = lfull * float("nan")
                for pb0, pb1, pd0, pd1, py, pl in parts:
                    ys[pb0:pb1, pd0:pd1] = py
                    ls[pb0:pb1, pd0:pd1] = pl
                res[(batch, dim)] = bool((ys == yfull).all() and (ls == lfull).all())
        if rank == 0:
            out.put(res)
    finally:
        dist.destroy_process_group()


def test_shard_plan_reassembles_over_two_gloo_ranks():
    """Two gloo ranks each take their (b, d) shard of the scan's arguments
    (views with the full strides and offset pointers, A/D/bias sliced by
    channel), run it, and the gathered pieces equal the unsharded call bit for
    bit (the oracle stands in for the kernels on the CPU)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == {(4, 48): True, (3, 40): True}


def test_ssd_bound_names_the_slower_roofline():
    # the 2.7B-class SSD layer: 257 MB and 53.7 GFLOP; at 6650 GB/s and 1590 TFLOP/s the bytes take longer
    assert bench.ssd_bound(257164224, 53687091200, 6650.0, 1590.0).startswith("hbm")
    assert bench.ssd_bound(1, 10 ** 15, 6650.0, 1590.0).startswith("tensor")
