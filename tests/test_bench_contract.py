"""Host-side checks of bench.py's output contract (no GPU): defaults, the
shared config dict of both arms, and the Eq. 6 and top-k helpers it reports."""
import bench


def test_defaults_run_one_gpu_with_three_warmups():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.steps >= 1
    assert a.impl == "resa" and a.workload == "long256k"


def test_both_arms_share_one_config():
    wl = bench.WORKLOADS["long256k"]
    cfg = bench.bench_config("long256k", wl)
    assert set(cfg) == {"workload", "description", "step", "l2", "parallelism"}
    assert cfg == bench.bench_config("long256k", wl)
    assert "28 layers" in cfg["step"]


def test_topk_rule_reproduces_the_printed_counts():
    # 10 % of the complete blocks, at least 16, capped at M: 205 of 2048 and
    # 1638 of 16384 (the Qwen-32K and 256K workloads' top-k)
    assert bench.topk_rule(32768 + 1) == 205
    assert bench.topk_rule(262144 + 1) == 1638
    assert bench.topk_rule(2048 + 1) == 16
    assert bench.topk_rule(100) == 6       # M = 6 < 16: every complete block
    assert bench.topk_rule(262144 + 1, bs=64) == 410


def test_schedule_lengths_grow_one_token_a_step():
    s = bench.Schedule([1000, 2000], 32, 2)
    assert s.decode_L(0, 0) == [1001, 2001]
    assert s.rect_L(0) == [1032, 2032]          # the cycle's 32nd token
    assert s.decode_L(1, 0) == [1033, 2033]
