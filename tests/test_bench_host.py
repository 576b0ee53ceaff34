"""The benchmark's host arithmetic on CPU: the algorithmic bytes behind every
GB/s figure, the committed DRAM-traffic table it reads, and its argument
checks.  The byte counts are written out from the definitions (dispatch reads
x once and writes K rows per token; combine gathers K rows and writes one;
4-byte ids, weights and destinations), not from the function under test."""
import pytest

import bench
from load_balancing_plan_b200 import inputs


def test_dispatch_and_combine_bytes_of_the_workloads():
    # mid: T = 8 * 4096 tokens, K = 8, rows of 7168 bf16
    T, K, row = 8 * 4096, 8, 7168 * 2
    ab = bench.alg_bytes(inputs.WORKLOADS["mid"].cfg())
    assert ab["dispatch"] == T * row + T * K * row + T * K * 4 + T * K * 4 == 4_229_955_584
    assert ab["combine"] == T * K * row + T * row + T * K * 4 + T * K * 4 == 4_229_955_584
    assert ab["plan"] == T * K * 4
    # training: four times the tokens
    ab = bench.alg_bytes(inputs.WORKLOADS["training"].cfg())
    assert ab["dispatch"] == ab["combine"] == 16_919_822_336


def test_weight_and_gradient_bytes():
    cfg = inputs.WORKLOADS["mid"].cfg()
    w_elems, g_elems = 2 * 7168 * 2048, 7168 * 2048
    ab = bench.alg_bytes(cfg, n_replicas=8, n_rx=3, w_elems=w_elems, g_elems=g_elems)
    # prefetch: each replicated expert read once (bf16), written to each slot
    assert ab["prefetch"] == 2 * w_elems * 3 + 2 * w_elems * 8
    # reduce_grad: home read + write per replicated expert, replica read + zero (fp32)
    assert ab["reduce_grad"] == 4 * g_elems * (2 * 3 + 2 * 8)


def test_backward_pair_bytes():
    cfg = inputs.WORKLOADS["training"].cfg()
    T, K, row = 16 * 8192, 8, 7168 * 2
    ab = bench.alg_bytes(cfg)
    # combine_backward: grad_out once, K expert rows read, K grad rows written,
    # weights and dest read and grad_w written (4 bytes each)
    assert ab["combine_backward"] == T * row + 2 * T * K * row + 12 * T * K
    # dispatch_backward: K grad rows read, grad_x written, dest read
    assert ab["dispatch_backward"] == T * K * row + T * row + 4 * T * K


def test_recorded_traffic_reads_the_committed_table():
    for kernel in ("dispatch", "combine"):
        for wl in ("training", "mid"):
            b, src = bench.recorded_traffic(kernel, wl)
            assert b is not None and b > 0 and "ncu" in src
            # DRAM traffic of a launch is within a few percent of its algorithmic bytes
            ab = bench.alg_bytes(inputs.WORKLOADS[wl].cfg())[kernel]
            assert 0.9 < b / ab < 1.05
    assert bench.recorded_traffic("dispatch", "no-such-workload") == (None, None)


def test_arguments():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])          # at least 3 warm-up steps
    with pytest.raises(SystemExit):
        bench.main(["--only", "no_such_kernel"])
