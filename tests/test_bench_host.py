"""Host logic of bench.py: FLOP accounting, replica aggregation and max-over-ranks timing, with
world-size-2 gloo process groups on the CPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from block_causal_streaming_b200.workloads import (TINY, WAN13B_5STEP, WAN14B, WP_RANK0,
                                                   small_case)


def _visible_pairs(wl):
    """Count (query, key) pairs allowed by the mask rule, by brute force over chunk indices."""
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    ids = np.concatenate([np.full(off[c + 1] - off[c], c) for c in range(wl.num_chunks)])
    q_ids = ids[off[nctx]:]
    return int((ids[None, :] <= q_ids[:, None]).sum())


@pytest.mark.parametrize("wl", [TINY,
                                small_case("acct", 3, 128, (50, 7), (33, 0, 90), 16, seed=1),
                                small_case("acct2", 2, 64, (), (300,), 64, seed=2)],
                         ids=lambda w: w.name)
def test_flop_accounting_counts_only_visible_pairs(wl):
    assert bench.attention_flops(wl) == 4 * wl.head_dim * wl.heads * _visible_pairs(wl)


def test_flop_accounting_of_benchmark_workloads():
    # 4*D*H*sum(len_c * end_c): 5 chunks of 4680 after 2 context chunks, H=12, D=128
    assert bench.attention_flops(WAN13B_5STEP) == 4 * 128 * 12 * sum(
        4680 * 4680 * (c + 1) for c in range(2, 7))


def test_row_flops_matches_total():
    wl = TINY
    assert bench.rows_flops(wl, range(wl.t_q), wl.heads) == bench.attention_flops(wl)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    bench.init_dist(world, "gloo")
    try:
        bench.barrier(world)
        t = bench.max_over_ranks(1.0 + rank, world)       # rank 1 is the slower one
        results[rank] = (t, bench.aggregate(10.0, world, t))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_replicas_take_the_slowest_rank_gloo():
    world = 2
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world,
                           start_method="spawn", join=True)
        got = dict(results)
    assert got[0] == got[1] == (2.0, 10.0)     # 2 ranks x 10 units / 2.0 s


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    class A:
        config, steps, warmup, cpu_seconds = 2, 1, 3, 1.0
    assert bench.reference_arm(A, world=2, rank=1) is None


def test_arguments_are_checked():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_workload_selection():
    assert bench.workload_of("wan13b_5step") is WAN13B_5STEP
    assert bench.workload_of("wan14b") is WAN14B
    assert bench.workload_of("wp_rank0") is WP_RANK0
    with pytest.raises(SystemExit):            # the 30-layer round is a parity case, not a bench line
        bench.main(["--workload", "wan13b_round30"])
    # one rank's call: one 4680-token chunk against 8 chunks of keys
    assert (WP_RANK0.t_q, WP_RANK0.t_kv, WP_RANK0.num_ctx_chunks) == (4680, 37440, 7)
    assert bench.attention_flops(WP_RANK0) == 4 * 128 * 12 * 4680 * 37440


def test_both_arms_print_the_same_config(monkeypatch):
    """The reference arm times the oracle on the workload the GPU arm runs, and says so with the
    same `config` object (the GPU arm calls workload_config with the same arguments)."""
    class A:
        workload, steps, warmup, cpu_seconds = "wan13b_5step", 1, 3, 0.05
    monkeypatch.setattr(bench, "oracle_sample",
                        lambda wl, inp, target_s, seed=0: (1.0, {"rows": 4, "heads": wl.heads,
                                                                 "seconds": 0.01, "flop": 1,
                                                                 "threads": 3}))
    line = bench.reference_arm(A, world=1, rank=0)
    assert line["cpu_baseline"]["cores"] == 3          # the threads the oracle ran with
    assert line["config"] == bench.workload_config(WAN13B_5STEP, 1, False)
    assert line["config"]["chunks"] == "2 ctx + 5 active x 4680"
    assert "633 MB" in line["config"]["l2"]
