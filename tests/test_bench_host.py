"""Host logic of bench.py: roofline bookkeeping and the multi-rank aggregation
(world size 2 over gloo on the CPU, one process per rank)."""

import os
import socket

import pytest

import bench
from workloads import MINUTE


def test_algorithmic_bytes_is_900_per_token_head():
    w = MINUTE
    base = bench.algorithmic_bytes(w, False, False) - w.B * w.n_frames * w.H * 4
    assert base == 900 * w.B * w.T * w.H
    st = w.B * w.H * w.d_k * w.d_v * 4
    assert bench.algorithmic_bytes(w, True, True) == bench.algorithmic_bytes(w, False, False) + 2 * st


def test_chunked_flops_constant():
    C, d = 64, 112
    assert bench.CHUNKED_FLOPS_PER_TOKEN_HEAD == 10 * C * d + 6 * d * d


def test_single_rank_aggregate():
    v, slowest = bench.aggregate_throughput(1000.0, 0.5, 1)
    assert v == 2000.0 and slowest == 0.5


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    bench.dist_init("gloo", world, timeout_s=60)
    bench.barrier(world)
    elapsed = 1.0 + rank          # rank 1 is the slowest
    value, slowest = bench.aggregate_throughput(100.0, elapsed, world)
    q.put((rank, value, slowest))
    dist.destroy_process_group()


def test_two_rank_gloo_aggregate_takes_slowest_rank():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, value, slowest in res:
        assert slowest == 2.0                 # max over ranks
        assert value == pytest.approx(100.0 * 2 / 2.0)


def test_reference_arm_other_ranks_do_no_work():
    args = bench.parse_args(["--impl", "reference"])
    assert bench.run_reference(args, MINUTE, rank=1, world=2) is None


def test_attention_flops_match_the_oracle_key_sets():
    """The bench's closed-form count of visible (query, key) pairs against the oracle's
    key sets, block by block, at the minute-scale shape and a ragged one."""
    from oracle import attention_reference as A
    from workloads import MINUTE
    for w in (MINUTE, MINUTE.with_(T=5000, H=3)):
        bl = 3 * w.frame_len
        pairs = sum((min(w.T, (b + 1) * bl) - b * bl) * len(A.block_keys(b, w.T, w.frame_len, 3, 2, 1))
                    for b in range(-(-w.T // bl)))
        assert bench.attention_flops(w) == 2 * (w.d_k + w.d_v) * pairs * w.B * w.H
    assert bench.attention_flops(MINUTE) == 8132067328000


def test_softmax_and_bidir_modes_parse():
    a = bench.parse_args(["--layer", "softmax", "--steps", "2"])
    assert a.layer == "softmax" and a.direction == "causal"
    a = bench.parse_args(["--direction", "bidir"])
    assert a.layer == "gdn" and a.direction == "bidir"


def test_fp8_algorithmic_bytes_are_564_per_token_head():
    """e4m3 q, k, v: one byte per element in, the bf16 output and the beta logit as before."""
    w = MINUTE
    gates = w.B * w.n_frames * w.H * 4
    assert bench.algorithmic_bytes(w, False, False, in_elem=1) - gates == 564 * w.B * w.T * w.H


@pytest.mark.parametrize("argv", [[], ["--inputs", "fp8"], ["--workload", "block"], ["--workload", "sessions"],
                                  ["--workload", "clip241"], ["--direction", "bidir"], ["--path", "ws"]])
def test_both_arms_report_the_same_config_keys(argv):
    """The reference arm and ours build `config` with the same function, so the keys match
    for every workload and mode (the driver compares them)."""
    a = bench.parse_args(argv)
    w = bench.workload_of(a)
    cfg = bench.run_config(a, w)
    for key in ("workload", "B", "H", "T", "d_k", "d_v", "frame_len", "chunk_len", "direction",
                "gate_placement", "api", "inputs"):
        assert key in cfg, key
    assert ("gdn_forward_fp8" in cfg["api"]) == ("--inputs" in argv)
    assert cfg["inputs"].startswith("q, k, v as e4m3") == ("--inputs" in argv)


def test_fp8_reference_arm_runs_on_the_widened_inputs():
    """The reference arm with --inputs fp8 times the oracle on the e4m3 inputs' values and
    prints the same config as our arm."""
    a = bench.parse_args(["--impl", "reference", "--inputs", "fp8", "--workload", "block",
                          "--steps", "1", "--warmup", "0", "--cpu-seconds", "0.2"])
    w = bench.workload_of(a)
    line = bench.run_reference(a, w, 0, 1)
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["config"] == bench.run_config(a, w)
