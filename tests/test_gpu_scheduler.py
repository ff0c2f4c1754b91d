"""The scheduler's latency model fitted to this GPU's own step times."""
import pytest

from causal_dit_kv_b200.scheduler import choose_batch, fit_from_measurements

pytestmark = pytest.mark.gpu

SHAPE = dict(layers=2, heads=4, head_dim=128, frame_h=16, frame_w=16, chunk_frames=1, sink_frames=1,
             window_frames=4, embed_dim=256, motion=(16, 16, 16))


def test_step_latency_fit_and_choice():
    from causal_dit_kv_b200.slo_profile import measure_step_latency
    pts = [(1, b, 1, measure_step_latency(SHAPE, b)) for b in (1, 4, 16)]
    assert all(lat > 0 for *_, lat in pts)
    model = fit_from_measurements(pts)
    assert model.beta > 0                                   # more streams cost more
    b = choose_batch(model, 1, target_fps=1.0 / (2 * pts[-1][3]), frames_available=64)
    assert b is not None and b >= 1
