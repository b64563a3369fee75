"""The bench's step schedule, on the host: problems spread over lanes by
estimated cost, quantize calls longest sweep chain first, and the default
worker cap of the factorisation."""
import bench
from workloads import problems_for


def _stack(cid, layers):
    return [p for l in range(layers) for p in problems_for(cid, layer=l)]


def test_quantize_order_longest_chain_first():
    probs = _stack(3, 2)          # TinyLlama: 15872x2048 (16 blocks), 2048x5632 (44 blocks)
    order = bench.quantize_order(probs)
    blocks = [-(-probs[k].n // probs[k].block) for k in order]
    assert blocks == sorted(blocks, reverse=True)
    assert probs[order[0]].n == 5632 and probs[order[-1]].n == 2048
    assert sorted(order) == list(range(len(probs)))


def test_quantize_order_ties_by_rows():
    probs = _stack(1, 1)          # SmolLM: 4608x576 (5 blocks), 576x1536 (12 blocks)
    order = bench.quantize_order(probs)
    assert [probs[k].n for k in order] == [1536, 576]


def test_lane_plans_balance_and_cover():
    probs = _stack(2, 3)          # Qwen2.5-0.5B: 3 layers, two problems each
    plans = bench.lane_plans(probs, 4)
    assert len(plans) == 4
    assert sorted(k for p in plans for k in p) == list(range(len(probs)))
    loads = [sum(bench.est_cost(probs[k]) for k in p) for p in plans]
    # the greedy gives no lane more than the lightest lane plus the largest problem
    assert max(loads) <= min(loads) + max(bench.est_cost(p) for p in probs) + 1e-12
    # the most expensive problem starts first on some lane
    first = max(range(len(probs)), key=lambda k: bench.est_cost(probs[k]))
    assert any(p and p[0] == first for p in plans)


def test_lane_plans_fewer_problems_than_lanes():
    probs = _stack(1, 1)
    plans = bench.lane_plans(probs, 4)
    assert len(plans) == 2 and sorted(k for p in plans for k in p) == [0, 1]


def test_factor_workers_default():
    class Props:
        multi_processor_count = 148

    import torch
    orig = torch.cuda.get_device_properties
    torch.cuda.get_device_properties = lambda dev: Props()
    try:
        assert bench.factor_workers(-1, 44, None) == 88
        assert bench.factor_workers(-1, 2, None) == 0
        assert bench.factor_workers(100, 44, None) == 100
        assert bench.factor_workers(0, 44, None) == 0
    finally:
        torch.cuda.get_device_properties = orig
