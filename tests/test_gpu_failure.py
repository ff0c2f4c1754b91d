"""Failure detection on the GPU without faulting it (B200).

A device wait that nothing completes runs out after its bound, records the
failure in the cache's status word and returns; the host reads the word
(SDV2_E_DEVICE), the word is cleared, and the CUDA context stays usable for
the next calls, which still match the oracle.
"""
import pytest
import torch

from harness import ATTN_MAX_ABS, ATTN_MEAN_ABS, PairedStream, attn_errors, cache_bits_equal

pytestmark = pytest.mark.gpu

TINY = dict(batch=1, layers=1, heads=2, head_dim=64, frame_h=4, frame_w=4, chunk_frames=1, sink_frames=1,
            window_frames=2)


def test_bounded_wait_reports_and_context_survives():
    from causal_dit_kv_b200 import binding as B
    ps = PairedStream(seed=1201, **TINY)
    assert ps.gpu.check() == B.SDV2_OK
    B.sdv2_cache_selftest_wait(ps.gpu.handle, 200_000_000)      # 0.2 s bound, nothing arrives
    assert ps.gpu.check() == B.SDV2_E_DEVICE
    assert "status" in B.sdv2_last_error()
    assert ps.gpu.check() == B.SDV2_OK                            # cleared after being reported
    for step in range(3):                                         # the context still works
        ps.step_idx = step
        f0 = ps.advance()
        q, k, v = ps.inputs(0)
        ps.append(0, f0, k, v)
        out, want = ps.attention(0, f0, q)
        mx, mean = attn_errors(out, want)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS
        assert all(cache_bits_equal(ps, 0)[:2])
    torch.cuda.synchronize()
    assert ps.gpu.check() == B.SDV2_OK


def test_selftest_rejects_unbounded_limit():
    from causal_dit_kv_b200 import binding as B
    ps = PairedStream(seed=1202, **TINY)
    for bad in (0, 3_000_000_000):
        with pytest.raises(B.SDV2Error) as e:
            B.sdv2_cache_selftest_wait(ps.gpu.handle, bad)
        assert e.value.status == B.SDV2_E_ARG
