"""SLO-aware stream-batch scheduler model (host side).

Source: qq8o.cn walkthrough of StreamDiffusionV2, "SLO-aware batching
scheduler" and "Multi-pipeline orchestration extension".  The pages model
one iteration's latency as memory-bound: L(T, B) = (A(T, B) + P_model) /
(eta * BW), with the activation traffic A growing linearly in B*T, so
L(T, B) = alpha + beta * B * T for a fixed model and GPU.  An iteration
processes B streams of T frames each; the achieved frame rate is
f = B * T / L(T, B), which grows with B until the roofline knee.  To keep up
with a live source at f_target frames per second per stream, an iteration
must finish before T new frames have arrived, L(T, B) <= T / f_target, and
B * T cannot exceed the frames already collected.  With n denoising steps
run as a batch multiplier (every micro-step emits a fully denoised chunk),
the latency becomes L(T, n * B).

Readings where the pages' formulas are blank: the linear form above is the
plainest one the text supports (it states A is O(BT) and names no other
term); the scheduler picks the largest B that meets the deadline, which is
where f = B T / L is highest under the constraint; the online adjustment
refits alpha, beta from observed latencies (least squares over a sliding
window) and re-plans.

Nothing here touches the GPU: measured (B*T, latency) pairs come from the
caller (bench.py can produce them from the library's own kernels).
"""
from __future__ import annotations

from collections import deque
from dataclasses import dataclass
from typing import Iterable, Optional, Sequence, Tuple


@dataclass
class LatencyModel:
    """L(T, B) = alpha + beta * B * T (seconds)."""

    alpha: float
    beta: float

    def latency(self, t: int, b: int, steps: int = 1) -> float:
        return self.alpha + self.beta * steps * b * t

    def frame_rate(self, t: int, b: int, steps: int = 1) -> float:
        """Frames per second of all streams together: B * T / L(T, n B)."""
        return b * t / self.latency(t, b, steps)

    @staticmethod
    def fit(samples: Iterable[Tuple[int, float]]) -> "LatencyModel":
        """Least-squares fit from (effective frames per iteration n*B*T, latency s)."""
        xs, ys = [], []
        for x, y in samples:
            xs.append(float(x))
            ys.append(float(y))
        if len(xs) < 2 or max(xs) == min(xs):
            raise ValueError("need latencies at two or more distinct batch sizes")
        n = len(xs)
        mx, my = sum(xs) / n, sum(ys) / n
        sxx = sum((x - mx) ** 2 for x in xs)
        sxy = sum((x - mx) * (y - my) for x, y in zip(xs, ys))
        beta = sxy / sxx
        alpha = my - beta * mx
        return LatencyModel(alpha=alpha, beta=beta)


def choose_batch(model: LatencyModel, t: int, target_fps: float, frames_available: int,
                 steps: int = 1, max_batch: int = 64) -> Optional[int]:
    """Largest B with L(T, n B) <= T / target_fps and B * T <= frames_available.

    Returns None when even B = 1 misses the deadline (the chunk length T or the
    step count must change instead)."""
    if t < 1 or target_fps <= 0 or steps < 1:
        raise ValueError("t, target_fps and steps must be positive")
    deadline = t / target_fps
    best = None
    for b in range(1, max_batch + 1):
        if b * t > frames_available:
            break
        if model.latency(t, b, steps) <= deadline:
            best = b
    return best


class AdaptiveBatcher:
    """Online version: observes each iteration's latency, refits the model over
    the last `window` observations and re-plans B for the next iteration."""

    def __init__(self, t: int, target_fps: float, steps: int = 1, max_batch: int = 64, window: int = 32,
                 initial: Optional[LatencyModel] = None, start_batch: int = 1):
        self.t, self.target_fps, self.steps, self.max_batch = t, target_fps, steps, max_batch
        self.obs: deque = deque(maxlen=window)
        self.model = initial
        self.batch = start_batch

    def observe(self, batch: int, latency_s: float) -> None:
        self.obs.append((self.steps * batch * self.t, latency_s))
        if len({x for x, _ in self.obs}) >= 2:
            self.model = LatencyModel.fit(self.obs)

    def next_batch(self, frames_available: int) -> int:
        """B for the next iteration.  Until two batch sizes have been seen it
        probes upwards by one stream per iteration."""
        if self.model is None or len({x for x, _ in self.obs}) < 2:
            self.batch = min(self.batch + 1, self.max_batch, max(1, frames_available // self.t))
            return self.batch
        b = choose_batch(self.model, self.t, self.target_fps, frames_available, self.steps, self.max_batch)
        self.batch = b if b is not None else 1
        return self.batch


def knee_batch(model: LatencyModel, t: int, steps: int = 1, efficiency: float = 0.9, max_batch: int = 64) -> int:
    """Smallest B whose frame rate reaches `efficiency` of the model's limit
    1 / (beta * n) (the bandwidth roofline of the linear model)."""
    limit = 1.0 / (model.beta * steps) if model.beta > 0 else float("inf")
    for b in range(1, max_batch + 1):
        if model.frame_rate(t, b, steps) >= efficiency * limit:
            return b
    return max_batch


def fit_from_measurements(points: Sequence[Tuple[int, int, int, float]]) -> LatencyModel:
    """points: (T, B, steps, latency_s) of measured iterations."""
    return LatencyModel.fit((s * b * t, lat) for t, b, s, lat in points)
