"""Host logic of the benchmark's step (no GPU): the step's calls group each
quantizer variant's tensors into one call, the launch count follows the
grouped launches, and the algorithmic bytes follow the formats' definitions
(2 bytes read + 0.5 written per bf16 element, one scale byte per block, one
macro byte per 128 elements; "Unveiling the Potential of Quantization with
MXFP4", Sec.2 and Sec.4)."""
import bench
import microscaling_block_quantization_b200 as mx


def test_step_calls_group_each_variant():
    plan = bench.step_plan(mx)
    calls = bench.step_calls(plan)
    q = [c for c in calls if c[3] == "q"]
    d = [c for c in calls if c[3] == "d"]
    assert [c[0] for c in q] == ["mxfp4_row", "nvfp4_row", "had32_mxfp4", "mbs_oas_mxfp4"]
    assert all(c[1] == ("A", "W") for c in q)
    assert [c[1] for c in d] == [("A",), ("W",)]
    # every launch of the plan is in exactly one call, with its configuration
    flat = sorted((n, t) for n, ts, _, _ in calls for t in ts)
    assert flat == sorted((n, t) for n, t, _, _ in plan)
    cfg = {(n, t): c for n, t, c, _ in plan}
    assert all(cfg[(n, t)] == c for n, ts, c, _ in calls for t in ts)


def test_launch_count_of_the_step():
    calls = bench.step_calls(bench.step_plan(mx))
    n = sum(bench.launches_per_call(c, k, len(ts)) for _, ts, c, k in calls)
    # 4 grouped quantizer launches, 1 grouped tensor-amax launch (NVFP4), 2 dequantizers
    assert n == 7
    assert bench.launches_per_call(mx.NVFP4, "q", 5) == 4      # two launches of up to 4 tensors, each with its amax
    assert bench.launches_per_call(mx.MXFP4, "q", 4) == 1
    assert bench.launches_per_call(mx.MXFP4, "d", 2) == 2


def test_algorithmic_bytes():
    rows, cols = 8192, 4096
    n = rows * cols
    assert bench.algo_bytes(mx.MXFP4, rows, cols, "q") == 2 * n + n // 2 + n // 32
    assert bench.algo_bytes(mx.NVFP4, rows, cols, "q") == 2 * n + n // 2 + n // 16
    mbs = mx.Config(macro_block=128, rule=mx.RULE_OAS, oas_tau=7.0)
    assert bench.algo_bytes(mbs, rows, cols, "q") == 2 * n + n // 2 + n // 32 + n // 128
    assert bench.algo_bytes(mx.Config(axis=mx.AXIS_2D), rows, cols, "q") == 2 * n + n // 2 + n // 1024
    assert bench.algo_bytes(mx.MXFP4, rows, cols, "d") == n // 2 + n // 32 + 2 * n
    assert bench.algo_bytes(mx.Config(elem=mx.E2M3), rows, cols, "q", in_bytes=4) == 4 * n + n + n // 32
