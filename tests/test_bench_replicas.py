"""Host logic of the multi-GPU bench on CPU: every rank runs an independent replica, the job's
time is the max over ranks (gloo here, NCCL on GPUs) and the throughput counts all ranks'
units.  No data-path collective exists to test: the path does not exchange data."""
import os

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    d = bench.init_dist(world, "gloo")
    assert bench.dist_env() == (rank, rank, world)
    local_seconds = 1.0 + rank                     # rank 1 is the slow one
    m = bench.reduce_max(local_seconds, d, torch.device("cpu"))
    out[rank] = (m, bench.aggregate(10.0, world, m))
    d.barrier()
    d.destroy_process_group()


def test_two_rank_max_and_aggregate():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, 29517, out), nprocs=world, join=True)
    assert out[0] == out[1] == (2.0, 10.0)        # 2 ranks x 10 units / 2.0 s


def test_single_rank_is_identity():
    assert bench.reduce_max(3.5, None, torch.device("cpu")) == 3.5
    assert bench.aggregate(7.0, 1, 2.0) == 3.5


def test_arg_defaults_fit_the_contract():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.steps >= 1 and a.impl == "ours"


def test_op_summary_excludes_the_side_stream_op():
    # event times (ms over K=10 steps) shaped like the QKV step: the side-stream op's time is the
    # largest but it overlaps the others, so it has no share and is not the dominant op
    per_op = {"w": 1.6, "a": 0.4, "gemm": 1.0, "kv": 0.2, "deq": 1.4}
    work = {"w": ("hbm", 1e8), "a": ("hbm", 5e7), "gemm": ("tensor", 2.65e11), "kv": ("hbm", 7e7),
            "deq": ("hbm", 8.8e8)}
    k, dom = bench.summarize_ops(per_op, 10, work, {"w"}, 6500.0, 5500.0)
    assert dom == "deq"
    assert k["w"]["share"] is None and "side" in k["w"]["stream"]
    assert abs(sum(v["share"] for v in k.values() if v["share"] is not None) - 1.0) < 1e-3
    assert k["deq"]["share"] == round(1.4 / 3.0, 4)
    # 8.8e8 B in 0.14 ms = 6285.7 GB/s; 2.65e11 FLOP in 0.1 ms = 2650 TFLOP/s
    assert k["deq"]["us_per_launch"] == 140.0 and abs(k["deq"]["achieved"] - 6285.7) < 0.1
    assert k["gemm"]["unit"] == "TFLOP/s" and abs(k["gemm"]["frac"] - 2650 / 5500) < 1e-4


def test_profiled_traffic_is_used_only_for_matching_sources(tmp_path, monkeypatch):
    # the roofline's `traffic` comes from a committed ncu summary only while the kernel sources
    # it names hash to the digest recorded with the capture
    csrc = tmp_path / "bit_kv_cache_24_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("kernel v1")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.kernel_source_digest(["k.cu"])
    (tmp_path / "profiles" / "k_case.md").write_text(
        f"# k\n\n- kernel_source_digest: `{digest}`\n- dram_bytes_per_launch: `123456`\n")
    assert bench.profiled_traffic("k_case", digest) == 123456.0
    (csrc / "k.cu").write_text("kernel v2")            # the kernel changed after the capture
    assert bench.profiled_traffic("k_case", bench.kernel_source_digest(["k.cu"])) is None
    assert bench.profiled_traffic("missing_case", digest) is None


def test_attention_slots_option():
    assert bench.parse_args([]).attn_slots == bench.SLOTS
    assert bench.parse_args(["--op", "attention", "--attn-slots", "1"]).attn_slots == 1
