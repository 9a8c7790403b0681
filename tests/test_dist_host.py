"""The multi-process path of bench.py on CPU: two ranks over gloo, launched as
the driver launches N replicas (RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* in
the environment). The layer does not shard, so N GPUs run N independent
replicas and the only collectives are the start/end barrier and the max of the
ranks' device times; these tests check that plumbing and the whole-job
throughput it feeds, without a GPU."""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    w, r, local = bench.dist_env()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=datetime.timedelta(seconds=30))
    try:
        bench.barrier(w)
        ms = bench.max_over_ranks(times[r], w)
        val = bench.job_tokens_per_s(32, w, 100, ms)
        bench.barrier(w)
        q.put((r, w, local, ms, val))
    finally:
        dist.destroy_process_group()


def _run(world, times):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        out = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    return out


def test_two_gloo_ranks_take_the_slowest_time():
    out = _run(2, [10.0, 12.5])
    assert [(r, w, local) for r, w, local, _, _ in out] == [(0, 2, 0), (1, 2, 1)]
    assert all(ms == 12.5 for _, _, _, ms, _ in out)
    # whole-job throughput: both replicas' tokens over the slowest rank's time
    assert all(val == pytest.approx(32 * 2 * 100 / 0.0125) for *_, val in out)


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.job_tokens_per_s(32, 1, 10, 2.0) == pytest.approx(32 * 10 / 0.002)
    bench.barrier(1)  # no process group: nothing to wait for


def test_algorithmic_bytes_and_flops_of_the_decode_step():
    """The roofline denominators bench.py reports, recomputed by hand for the
    decode layer with 5 active experts holding 8, 8, 8, 4, 4 of the 32 x 8 slots
    (bf16: 2 bytes per element, no scales)."""
    sys.path.insert(0, ROOT)
    import torch

    import bench
    from routed_shared_experts_b200 import configs
    cfg = configs.DECODE_BF16
    counts = torch.zeros(cfg.E, dtype=torch.int64)
    counts[:5] = torch.tensor([8, 8, 8, 4, 4])
    ab = bench.algorithmic_bytes(cfg, counts)
    H, I, Is, T, E = cfg.H, cfg.I, cfg.Is, cfg.T, cfg.E
    rows = 32
    w13, w2 = 2 * I * H * 2, H * I * 2
    assert ab["active_experts"] == 5
    assert ab["stage1"] == 5 * w13 + T * H * 2 + rows * I * 2
    assert ab["stage2"] == 5 * w2 + rows * I * 2 + 2 * T * H * 2 + rows * 4
    shared = 3 * H * Is * 2
    assert ab["layer"] == 5 * (w13 + w2) + shared + T * H * 2 + T * H * 2 + T * E * 4 + H * 2
    assert ab["flops"] == 6 * rows * H * I + 6 * T * H * Is


def test_mx_and_fp8_bytes_count_their_scales():
    sys.path.insert(0, ROOT)
    from routed_shared_experts_b200 import synth
    n = 4096 * 1024
    assert synth.matrix_bytes("bf16", n) == 2 * n
    assert synth.matrix_bytes("fp8", n) == n + 4
    assert synth.matrix_bytes("mxfp8", n) == n + n // 32
    assert synth.matrix_bytes("mxfp4", n) == n // 2 + n // 32
    assert synth.activation_bytes("fp8", 10, 4096) == 10 * 4096 + 40
    assert synth.activation_bytes("mxfp4", 10, 4096) == 10 * 4096 + 10 * 128


def test_weight_copies_put_every_step_over_three_l2s():
    """Steps that read less than 3x the 126 MB L2 cycle through enough weight
    copies that every step's weights come from HBM; larger steps use one."""
    sys.path.insert(0, ROOT)
    import bench
    for step in (1.8e6, 138e6, 230e6, 0.81e9, 11.6e9):
        n = bench.weight_copies(step)
        assert n * step >= 3 * bench.L2_BYTES
        assert n == 1 or (n - 1) * step < 3 * bench.L2_BYTES
        assert "come from HBM" in bench.l2_note(step, n)
    assert bench.weight_copies(0.81e9) == 1 and bench.weight_copies(1.8e6) == 210


def test_traffic_records_follow_the_kernel_code_not_its_comments():
    sys.path.insert(0, ROOT)
    import bench
    src = "// a comment\nint f(int x) { /* inline\n block */ return x + 1; }  // trailing\n\n"
    assert bench._code_only(src) == "int f(int x) {  return x + 1; }"
    edited = src.replace("a comment", "another comment").replace("trailing", "tail")
    assert bench._code_only(edited) == bench._code_only(src)
    assert bench._code_only(src.replace("x + 1", "x + 2")) != bench._code_only(src)
    # every recorded figure is keyed to a hash of that form, and looked up by it
    import json
    rows = json.load(open(os.path.join(os.path.dirname(bench.__file__), "profiles", "traffic.json")))
    assert rows and all(len(r["src_sha"]) == 16 and r["dram_bytes_per_launch"] > 0 for r in rows)
