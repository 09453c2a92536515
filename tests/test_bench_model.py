"""The benchmark's algorithmic byte / FLOP model against the step arithmetic
of the full shape (no GPU): FLOPs 2 T x active parameters + attention, bytes =
every weight once (all experts touched) + the KV read + activations."""
import importlib.util
import os

import pytest

from synth import FULL

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_step_flops_and_weight_bytes(bench):
    T, L = 256, 4096
    by, fl = bench.step_work(FULL, L, T, 128)
    # 2 T x 3.75B active parameters + 30 layers x 4 x 16 heads x 256 x 256 x 4352 keys
    assert fl == pytest.approx(2 * T * FULL.active_params_per_token() + 30 * 4 * 16 * T * (L + T) * 256)
    assert fl == pytest.approx(2.467e12, rel=1e-3)
    weights = FULL.total_params() * 2                      # 25.16B bf16 parameters
    kv = 30 * 2 * 8 * (L + T) * 256 * 2
    assert weights == pytest.approx(50.32e9, rel=1e-3)
    assert kv == pytest.approx(1.07e9, rel=1e-2)
    act = by - weights - kv
    assert 0 < act < 0.05 * by                             # activations: a few percent of the step


def test_fp8_experts_halve_the_expert_bytes(bench):
    bf = bench.expert_gate_up_bytes(FULL, 128, 256)
    f8 = bench.expert_gate_up_bytes(FULL.with_(expert_fp8=1), 128, 256)
    w_bf = 128 * 2 * FULL.ffn_expert * FULL.d_model * 2
    assert bf > w_bf and f8 < 0.52 * bf
    by, _ = bench.step_work(FULL, 4096, 256, 128)
    by8, _ = bench.step_work(FULL.with_(expert_fp8=1), 4096, 256, 128)
    experts = 30 * 128 * 3 * FULL.ffn_expert * FULL.d_model * 2
    assert by - by8 == pytest.approx(experts / 2)
