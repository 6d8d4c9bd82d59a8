"""Host-side logic of bench.py, on the CPU: the FLOP/byte bookkeeping, the
oracle sample plan, the traffic lookup, and the multi-rank path (weak
scaling: each rank its own batch; the only collectives are the barrier and the
max-over-ranks timing reduction), run as two gloo ranks."""

import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def test_workload_bookkeeping():
    w = synth.workload(4)
    assert (w.B, w.H, w.N, w.d, w.causal) == (2, 32, 8192, 128, True)
    assert w.flops == 4 * 2 * 32 * 8192 ** 2 * 128 / 2
    assert w.algorithmic_bytes == 4 * 2 * 32 * 8192 * 128 * 2 + 2 * 32 * 8192 * 4
    w1 = synth.workload(1)
    assert w1.flops == 4 * 256 * 256 * 64 and not w1.causal
    assert abs(synth.workload(5).scale - 1 / 128 ** 0.5) < 1e-15


def test_sample_plan_counts_allowed_keys():
    w = synth.workload(4)
    idx, flops = bench.sample_plan(w, 3)
    assert idx == [8189, 8190, 8191]
    assert flops == 4.0 * (8190 + 8191 + 8192) * 128
    w2 = synth.workload(2)
    idx, flops = bench.sample_plan(w2, 10)
    assert flops == 4.0 * 10 * 512 * 64


def test_inputs_are_seeded_and_rank_distinct():
    a = synth.draw_qkv(1, 2, 16, 64, seed=bench.rank_seed(1224, 0))
    b = synth.draw_qkv(1, 2, 16, 64, seed=bench.rank_seed(1224, 0))
    c = synth.draw_qkv(1, 2, 16, 64, seed=bench.rank_seed(1224, 1))
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert not torch.equal(a[0], c[0])
    assert a[0].dtype == torch.bfloat16 and a[0].is_contiguous()


def test_traffic_is_null_unless_kernel_matches(tmp_path, monkeypatch):
    f = tmp_path / "t.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.load_traffic("long_context_causal") is None
    f.write_text(json.dumps({"kernel_source_sha256": "0" * 64, "workload": "long_context_causal",
                             "bytes_per_launch": 123}))
    assert bench.load_traffic("long_context_causal") is None
    f.write_text(json.dumps({"kernel_source_sha256": bench.kernel_source_sha(),
                             "workload": "long_context_causal", "bytes_per_launch": 123}))
    assert bench.load_traffic("long_context_causal") == 123
    assert bench.load_traffic("other") is None
    # several entries, one per (workload, kernel source)
    f.write_text(json.dumps({"entries": [
        {"kernel_source": "exact_attention_122_b200/csrc/fa_fwd_sm100.cu",
         "kernel_source_sha256": bench.kernel_source_sha(), "workload": "a", "bytes_per_launch": 1},
        {"kernel_source": "exact_attention_122_b200/csrc/fa_bwd_sm100.cu",
         "kernel_source_sha256": bench.kernel_source_sha(bench.BWD_KERNEL_SOURCE),
         "workload": "a_bwd", "bytes_per_launch": 2},
        {"kernel_source": "exact_attention_122_b200/csrc/fa_bwd_sm100.cu",
         "kernel_source_sha256": "0" * 64, "workload": "b_bwd", "bytes_per_launch": 3}]}))
    assert bench.load_traffic("a") == 1
    assert bench.load_traffic("a_bwd", bench.BWD_KERNEL_SOURCE) == 2
    assert bench.load_traffic("a_bwd") is None                     # wrong source for that entry
    assert bench.load_traffic("b_bwd", bench.BWD_KERNEL_SOURCE) is None   # stale sha


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = bench.dist_env()
        per_rank_ms = [3.5, 7.25][rank]
        m = bench.max_over_ranks(per_rank_ms)
        seed = bench.rank_seed(1224, r)
        dist.barrier()
        out.put((rank, w, r, lr, m, seed))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_gloo():
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
    assert [r[1] for r in res] == [2, 2]
    assert [r[2] for r in res] == [0, 1]
    assert all(r[4] == 7.25 for r in res)          # max over ranks, seen by every rank
    assert res[0][5] != res[1][5]                   # independent batches per rank


def test_single_process_max_is_identity():
    assert bench.max_over_ranks(4.0) == 4.0


def test_cli_rejects_short_warmup():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_l2_rotation_plan():
    """Steps that move less than twice the 126 MB L2 cycle through copies of
    their buffers: enough that twice the L2 streams between two uses of one
    copy, at most one copy per launch; big steps use one set of buffers."""
    L2 = 126 * 1000 * 1000
    assert bench.rotation_copies(synth.workload(4).algorithmic_bytes, 300) == 1
    assert bench.rotation_copies(synth.workload(5).algorithmic_bytes, 10) == 1
    for idx in (1, 2, 3):
        b = synth.workload(idx).algorithmic_bytes
        c = bench.rotation_copies(b, 100000)
        assert c >= 2 and (c - 1) * b >= 2 * L2 and (c - 2) * b < 2 * L2
        assert bench.rotation_copies(b, 4) == 4       # capped by the launch count
    assert bench.rotation_copies(2 * L2, 5) == 1
    assert bench.rotation_copies(2 * L2 - 1, 5) == 3
    assert "no flush" in bench.l2_note(600_000_000, 1)
    assert "flushed" in bench.l2_note(25_000_000, 11)
    with pytest.raises(SystemExit):
        bench.require_beyond_l2(30_000_000, 20, "--fp8")
    bench.require_beyond_l2(600_000_000, 20, "--fp8")
    assert bench.fwd_kernel_name(128) == "fa_fwd_kernel<128,4>"
    assert bench.fwd_kernel_name(64) == "fa_fwd_kernel<64,8>"


def test_auto_schedule_resolution():
    """"auto" picks the dynamic schedule from 4 to 12 units of 256 rows per SM."""
    from exact_attention_122_b200 import resolve_schedule

    assert resolve_schedule("auto", 2, 32, 8192, 148) == "static"      # 2048 units >= 12 x 148
    assert resolve_schedule("auto", 1, 32, 8192, 148) == "dynamic"     # 1024
    assert resolve_schedule("auto", 1, 32, 4096, 148) == "static"      # 512 < 592
    assert resolve_schedule("auto", 8, 12, 1024, 148) == "static"      # 384
    assert resolve_schedule("auto", 1, 37, 4096, 148) == "dynamic"     # 592 = 4 x 148
    assert resolve_schedule("auto", 1, 37, 4095, 148) == "dynamic"     # ceil(4095/256) = 16
    assert resolve_schedule("auto", 1, 37, 3840, 148) == "static"      # 555
    assert resolve_schedule("auto", 1, 16, 32768, 148) == "static"     # 2048
    assert resolve_schedule("auto", 1, 111, 4096, 148) == "static"     # 1776 = 12 x 148
    assert resolve_schedule("auto", 1, 111, 4095, 148) == "static"     # ceil(4095/256) = 16
    assert resolve_schedule("auto", 1, 110, 4096, 148) == "dynamic"    # 1760 < 1776
    for s in ("static", "dynamic"):
        assert resolve_schedule(s, 1, 1, 1, 148) == s
    with pytest.raises(ValueError):
        resolve_schedule("fast", 1, 1, 1, 148)
    assert bench.bench_schedule("auto", synth.workload(4)) == "static"
    assert bench.bench_schedule("auto", synth.workload(5)) == "static"
    assert bench.bench_schedule("auto", synth.workload(2)) == "static"
