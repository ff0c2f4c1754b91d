"""SLO-aware stream-batch scheduler model: fit, deadline rule, online adaptation."""
import random

import pytest

from causal_dit_kv_b200.scheduler import AdaptiveBatcher, LatencyModel, choose_batch, fit_from_measurements, knee_batch


def test_fit_recovers_a_linear_model():
    true = LatencyModel(alpha=0.012, beta=0.0031)
    pts = [(t, b, s, true.latency(t, b, s)) for t in (1, 2, 4) for b in (1, 3, 8) for s in (1, 2)]
    m = fit_from_measurements(pts)
    assert m.alpha == pytest.approx(true.alpha, rel=1e-9)
    assert m.beta == pytest.approx(true.beta, rel=1e-9)


def test_fit_with_noise_and_degenerate_input():
    rng = random.Random(3)
    true = LatencyModel(alpha=0.02, beta=0.004)
    pts = [(2, b, 1, true.latency(2, b) * (1 + 0.01 * rng.uniform(-1, 1))) for b in range(1, 17)]
    m = fit_from_measurements(pts)
    assert abs(m.beta - true.beta) / true.beta < 0.05
    with pytest.raises(ValueError):
        LatencyModel.fit([(4, 0.1), (4, 0.2)])        # one batch size only


def test_deadline_rule_worked_cases():
    m = LatencyModel(alpha=0.01, beta=0.002)
    # deadline T / f = 4 / 30 s; 0.01 + 0.008 B <= 0.1333 -> B <= 15
    assert choose_batch(m, 4, 30.0, frames_available=1000) == 15
    # only 40 frames collected: B * 4 <= 40
    assert choose_batch(m, 4, 30.0, frames_available=40) == 10
    # two denoising steps double the effective batch: 0.01 + 0.016 B <= 0.1333 -> B <= 7
    assert choose_batch(m, 4, 30.0, frames_available=1000, steps=2) == 7
    # a deadline no batch meets
    assert choose_batch(LatencyModel(0.1, 0.01), 2, 30.0, 1000) is None


def test_chosen_batch_is_the_fastest_feasible_one():
    m = LatencyModel(alpha=0.015, beta=0.0025)
    t, fps = 2, 24.0
    b = choose_batch(m, t, fps, 10_000)
    assert m.latency(t, b) <= t / fps < m.latency(t, b + 1)
    rates = [m.frame_rate(t, k) for k in range(1, b + 1)]
    assert rates == sorted(rates)                         # throughput grows with B up to the choice


def test_knee_reaches_the_bandwidth_limit():
    m = LatencyModel(alpha=0.002, beta=0.001)          # rate 2B / (0.002 + 0.002 B): 875 at B = 7, 889 at B = 8
    b = knee_batch(m, 2, efficiency=0.88)
    assert b == 8
    limit = 1.0 / m.beta
    assert m.frame_rate(2, b) >= 0.88 * limit > m.frame_rate(2, b - 1)


def test_adaptive_batcher_converges_to_the_rule():
    true = LatencyModel(alpha=0.008, beta=0.0017)
    ab = AdaptiveBatcher(t=2, target_fps=20.0, steps=1, max_batch=64)
    b = ab.next_batch(frames_available=500)
    for _ in range(20):
        ab.observe(b, true.latency(2, b))
        b = ab.next_batch(frames_available=500)
    assert b == choose_batch(true, 2, 20.0, 500)
