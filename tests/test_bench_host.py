"""Host-side logic of bench.py for N > 1 ranks, run as two gloo ranks on CPU.

The block shards by tokens with no exchange step, so N GPUs run N independent
replicas; what ranks share is the bookkeeping: every rank agrees on the step
count (maximum over ranks), the timed duration is the slowest rank's, and the
reported value is the tokens all ranks processed over that duration.
"""
import importlib.util
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist          # noqa: E402
import torch.multiprocessing as mp        # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        b = _bench()
        K = int(b.max_over_ranks(100 + 7 * rank, dist, world, "cpu", torch.int64))
        ms = float(b.max_over_ranks(10.0 + rank * 2.5, dist, world, "cpu", torch.float64))
        value = b.job_rate(8 * K, world, ms / 1e3)
        q.put((rank, K, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_steps_and_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, K, ms, value in got:
        assert K == 107                  # the larger step count
        assert ms == pytest.approx(12.5)  # the slowest rank
        assert value == pytest.approx(8 * 107 * world / 12.5e-3)


def test_single_rank_is_a_no_op():
    b = _bench()
    assert b.max_over_ranks(3.5, None, 1, "cpu", torch.float64) == 3.5
    assert b.job_rate(1000, 1, 0.5) == 2000


def test_reference_arm_runs_on_rank_zero_only(capsys, monkeypatch):
    b = _bench()
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    args = b.parse()
    assert b.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_code_hash_ignores_comments_but_not_code():
    b = _bench()
    src = "int f(int a) {\n    return a + 1;   // one more\n}\n/* block\n comment */\n"
    assert b.code_hash(src) == b.code_hash("int f(int a) { return a + 1; }")
    assert b.code_hash(src) == b.code_hash(src.replace("one more", "the next integer"))
    assert b.code_hash(src) != b.code_hash(src.replace("a + 1", "a + 2"))


def test_work_model_counts_each_tensor_once():
    """Algorithmic bytes / FLOPs of the decode workload, written out by hand:
    the up kernel streams each active expert's gate_up once (2I x H bf16)
    plus x and h; the step adds the down weights, the router, h twice, the
    fp32 accumulator three times and y."""
    b = _bench()
    from sigmoid_top_routing_b200 import inputs as G
    wl = G.WORKLOADS["lfm2_decode_t8"]
    inp = G.make_inputs(wl, with_experts=False)
    counts = [0] * wl.E
    for e in (0, 3, 5):
        counts[e] = 2
    m = b.work_model(inp, counts)
    T, H, E, k, I = wl.T, wl.H, wl.E, wl.k, wl.I
    P = T * k
    assert m["active_experts"] == 3
    assert m["w1_bytes_per_expert"] == 2 * I * H * 2
    assert m["up_bytes"] == 3 * 2 * I * H * 2 + T * H * 2 + P * I * 2
    assert m["up_flops"] == 2.0 * P * 2 * I * H
    assert m["flops"] == 2.0 * P * (2 * I * H + H * I)
    assert m["step_bytes"] == (3 * (2 * I * H + H * I) * 2 + T * H * 2 + E * H * 4 + 2 * P * I * 2
                               + 3 * T * H * 4 + T * H * 2)


def _all_active(wl):
    return [1] * wl.E


@pytest.mark.parametrize("name,bound", [
    ("lfm2_decode_t8", "hbm"), ("lfm2_prefill_t4096", "tensor"), ("nemotron_relu2_t2048", "hbm"),
    ("affine4_t1", "hbm"), ("affine4_t8", "hbm"), ("affine4_t64", "hbm"), ("affine4_t512", "hbm"),
    ("affine4_t8192", "tensor")])
def test_roofline_bound_of_every_configuration(name, bound):
    """The up kernel's bound follows from its FLOPs per algorithmic byte
    against the ridge of the measured peaks (sustained GEMM / HBM copy)."""
    b = _bench()
    from sigmoid_top_routing_b200 import inputs as G
    wl = G.WORKLOADS[name]
    m = b.work_model(G.make_inputs(wl, with_experts=False), _all_active(wl))
    pk = {"hbm_gbs": 6548.8, "bf16_tflops": 1628.7, "bf16_tflops_sustained": 1380.3}
    assert b.ridge_flop_per_byte(pk) == pytest.approx(1380.3e3 / 6548.8)
    r = b.roofline_of(m, 100.0, pk, "measured", None)
    assert r["bound"] == bound
    if bound == "hbm":
        assert r["achieved"] == pytest.approx(m["up_bytes"] / 100e-6 / 1e9)
        assert r["peak"] == 6548.8 and r["nominal_peak"] == 7700.0
    else:
        assert r["achieved"] == pytest.approx(m["up_flops"] / 100e-6 / 1e12)
        assert r["peak"] == 1380.3 and r["nominal_peak"] == 2250.0
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])


def test_graph_block_fits_any_step_count():
    b = _bench()
    assert b.block_steps(20, 2) == 20
    assert b.block_steps(100, 2) == 32
    assert b.block_steps(7, 2) == 6
    assert b.block_steps(1, 2) == 2          # K < n_sets: only single-step graphs replay
    assert b.block_steps(40, 3) == 30
    # the event pairs the last replays of K steps leave behind
    assert b.replayed_events(20, 20, 20, 2) == [("block", range(20))]
    assert b.replayed_events(1, 2, 2, 2) == [("single", range(1))]
    assert b.replayed_events(45, 32, 32, 2) == [("block", range(32)), ("single", range(2))]


def test_side_workloads_selection():
    b = _bench()
    assert b.side_workloads("none", "lfm2_prefill_t4096") == []
    allw = b.side_workloads("all", "lfm2_prefill_t4096")
    assert "lfm2_decode_t8" in allw and "affine4_t8192" in allw and "lfm2_prefill_t4096" not in allw
    assert b.side_workloads("affine4_t1,lfm2_prefill_t4096", "lfm2_prefill_t4096") == ["affine4_t1"]


def test_reference_arm_config_matches_ours(capsys, monkeypatch):
    """Both arms describe the workload with the same config dict."""
    import json
    b = _bench()
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1",
                                      "--warmup", "0"])
    args = b.parse()
    assert b.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    from sigmoid_top_routing_b200 import inputs as G
    assert line["config"] == b.config_of(G.WORKLOADS["tiny"], b.parse(["--workload", "tiny"]))
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
