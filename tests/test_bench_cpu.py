"""bench.py host logic on CPU: multi-rank timing reduction over 2 gloo ranks, the
algorithmic byte / work counts, and the CPU-baseline leg."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, local = bench.dist_env()
    dist = bench.init_dist(w, "gloo", timeout_s=30)
    bench.barrier(dist)
    # rank 1 is the slow rank; the job time is the slowest rank's
    mx = bench.max_over_ranks(dist, 1.5 + r)
    total = bench.sum_over_ranks(dist, 1000 * (r + 1))
    bench.barrier(dist)
    dist.destroy_process_group()
    out.put((r, w, local, mx, total))


def test_two_gloo_ranks_reduce_time_and_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [x[0] for x in res] == [0, 1]
    for r, w, local, mx, total in res:
        assert w == 2 and local == r
        assert mx == 2.5            # max over ranks
        assert total == 3000.0      # work of all ranks


def test_single_rank_reductions_are_identity():
    assert bench.max_over_ranks(None, 3.25) == 3.25
    assert bench.sum_over_ranks(None, 7.0) == 7.0


def test_scan_counts_mamba130m():
    c = bench.scan_counts(8, 1536, 2048, 16, 2, 2)
    assert c["tokch"] == 8 * 2048 * 1536
    assert c["exps"] == 8 * 2048 * 1536 * 16
    # x, delta, z in and y out (2 B each) + B, C + A, D, bias + final state
    expect = 8 * 1536 * 2048 * 8 + 2 * 8 * 2048 * 16 * 2 + 1536 * 16 * 4 + 2 * 1536 * 4 + 8 * 1536 * 16 * 4
    assert c["bytes"] == expect
    assert abs(c["bytes"] / 1e6 - 203.2) < 0.1


def test_step_counts_decode():
    c = bench.step_counts(256, 5120, 16, 2, 2)
    assert c["tokch"] == 256 * 5120
    assert abs(c["bytes"] / 1e6 - 178.6) < 0.5


def test_oracle_rate_is_bounded_and_reports_cores():
    r = bench.oracle_rate("tiny", threads=2, budget_s=0.2)
    assert r["kind"] == "oracle" and r["cores"] == 2 and r["value"] > 0
    assert r["seconds"] < 5.0


def test_reference_arm_prints_one_line(capsys):
    rc = bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1"])
    assert rc == 0
    import json
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 2 and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["unit"] == bench.UNIT and d["higher_is_better"] is True


@pytest.mark.parametrize("world", [1])
def test_dist_env_defaults(world, monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 1, 0)


def test_conv_counts_mamba130m():
    c = bench.conv_counts(8, 1536, 2048, 4, 2, 2)
    assert c["tokch"] == 8 * 1536 * 2048
    # x in, u out (2 B each) + taps and bias + the final window (3 fp32 per row)
    assert c["bytes"] == 8 * 1536 * 2048 * 4 + 1536 * 5 * 4 + 8 * 1536 * 3 * 4
    assert abs(c["bytes"] / 1e6 - 100.8) < 0.1


def test_conv_step_counts():
    c = bench.conv_step_counts(256, 5120, 4, 2, 2)
    assert c["tokch"] == 256 * 5120
    assert c["bytes"] == 256 * 5120 * (24 + 4) + 5120 * 20


def test_workload_kinds():
    assert [bench.workload_kind(n) for n in ("mamba130m", "decode", "conv130m", "conv2p8b", "convstep")] \
        == ["scan", "decode", "conv", "conv", "convstep"]


@pytest.mark.parametrize("name", ["conv130m", "convstep"])
def test_conv_oracle_rate_single_core(name):
    r = bench.oracle_rate(name, threads=4, budget_s=0.2)
    assert r["kind"] == "oracle" and r["cores"] == 1 and r["value"] > 0


def test_bwd_counts_mamba130m():
    c = bench.bwd_counts(8, 1536, 2048, 16, 2, 2)
    assert c["tokch"] == 8 * 2048 * 1536 and c["exps"] == 2 * 8 * 2048 * 1536 * 16
    # x, delta, z, dy in and dx, ddelta, dz out (2 B each) + B, C in and dB, dC out + params
    expect = 8 * 1536 * 2048 * 14 + 2 * 8 * 2048 * 16 * 4 + 2 * (1536 * 16 * 4 + 2 * 1536 * 4)
    assert c["bytes"] == expect
    assert bench.workload_kind("bwd130m") == "bwd"


def test_bwd_oracle_rate_single_core():
    r = bench.oracle_rate("bwd130m", threads=4, budget_s=0.2)
    assert r["kind"] == "oracle" and r["cores"] == 1 and r["value"] > 0


def test_multi_token_decode_counts():
    one = bench.step_counts(256, 5120, 16, 2, 2)
    four = bench.steps_counts(4, 256, 5120, 16, 2, 2)
    state = 2 * 256 * 5120 * 16 * 4
    params = 5120 * 16 * 4 + 5120 * 4
    assert four["tokch"] == 4 * one["tokch"]
    assert four["bytes"] == state + 4 * (one["bytes"] - state - params) + params
    r = bench.oracle_rate("decode4", threads=2, budget_s=0.1)
    assert r["value"] > 0 and r["cores"] == 1


def test_ssd_counts():
    c = bench.ssd_counts(8, 2048, 24, 64, 128, 2, 2)
    toks = 8 * 2048 * 24
    assert c["bytes"] == toks * (64 * 2 + 2 * 128 * 2 + 4 + 64 * 2)
    # 16 chunks of 128 tokens per (sequence, head): scores Q x Q x N, masked scores times x
    # Q x Q x P, and the two state products Q x N x P
    assert c["flops"] == 8 * 24 * 16 * 2 * (128 * 128 * 128 + 128 * 128 * 64 + 2 * 128 * 128 * 64)
    assert c["tokch"] == toks * 64
    r = bench.oracle_rate("ssd130m", threads=2, budget_s=0.1)
    assert r["value"] > 0


@pytest.mark.parametrize("name", ["mamba130m", "decode", "ssd130m", "bwd130m", "decode4", "conv130m",
                                  "convstep"])
def test_oracle_sample_and_call_for_every_workload_kind(name):
    kind, inp, units, what = bench._oracle_sample(name, 4096)
    assert kind == bench.workload_kind(name) or (kind == "scan" and name == "mamba130m")
    assert units > 0 and what
    bench._oracle_call(kind, inp, 2)


def test_grid_fill_workloads_and_segment_option():
    """The 2.8b shape at d_inner 4736 / 5920 (592 and 740 CTAs of 32 channels, an even 4 or
    5 per SM on 148 SMs) are scan workloads that differ from mamba2p8b in d_inner only,
    and --segments parses for the scan sweeps (0, the default, leaves the plan automatic)."""
    from selective_state_space_45_b200 import inputs
    base = inputs.CONFIGS["mamba2p8b"]
    for name, dim in (("mamba2p8b_d4736", 4736), ("mamba2p8b_d5920", 5920)):
        c = inputs.CONFIGS[name]
        assert bench.workload_kind(name) == "scan"
        assert c["dim"] == dim and 4 * (dim // 32) in (592, 740)
        assert {k: v for k, v in c.items() if k != "dim"} == {k: v for k, v in base.items() if k != "dim"}
        assert "d_inner %d" % dim in bench.describe_workload(name)
        assert bench.parse_args(["--workload", name]).workload == name
    assert bench.parse_args([]).segments == 0
    assert bench.parse_args(["--workload", "long1m", "--segments", "8"]).segments == 8
