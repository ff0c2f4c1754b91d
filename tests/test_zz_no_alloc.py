"""Allocation-free motion entry point (B200).

sdv2_motion_noise_rate_noalloc serves callers that cannot call cudaMalloc
where they run the step (a host framework that owns all device memory, a
real-time loop that must not allocate): its per-call scratch sits in a fixed
device array the library holds.  These tests call it through the C ABI and
check it against sdv2_motion_noise_rate on two calls in a row (the second
call finds the shared array holding the first call's contents), and that it
refuses sizes beyond that array.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import synth
from harness import MOTION_REL

pytestmark = pytest.mark.gpu


def _handle(B, cfg):
    nbytes = B.sdv2_motion_bytes(cfg)
    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    return buf, B.sdv2_motion_create(cfg, buf, nbytes)


def test_noalloc_matches_regular_entry_point_on_two_calls():
    from causal_dit_kv_b200 import binding as B
    cfg = B.make_motion_config(2, 2, 16, 64, 64, window=4, sigma=2.0, lam=0.9)
    buf_a, ha = _handle(B, cfg)
    buf_b, hb = _handle(B, cfg)
    rate_a = torch.zeros(2, dtype=torch.float32, device="cuda")
    rate_b = torch.zeros(2, dtype=torch.float32, device="cuda")
    d_a = torch.zeros((2, 2), dtype=torch.float32, device="cuda")
    d_b = torch.zeros((2, 2), dtype=torch.float32, device="cuda")
    gen = synth.motion_latents(4001, 2, 2, 16, 64, 64, n_chunks=2)
    try:
        for call in range(2):
            x = next(gen).cuda()
            B.sdv2_motion_noise_rate(ha, x, rate_a, d_a)
            B.sdv2_motion_noise_rate_noalloc(hb, x, rate_b, d_b)
            torch.cuda.synchronize()
            ra, rb = rate_a.cpu().numpy().astype(np.float64), rate_b.cpu().numpy().astype(np.float64)
            assert np.all(np.abs(rb - ra) <= MOTION_REL * np.abs(ra)), (call, ra, rb)
            da, db = d_a.cpu().numpy().astype(np.float64), d_b.cpu().numpy().astype(np.float64)
            first = da < 0
            assert np.array_equal(first, db < 0)
            assert np.all(np.abs(db[~first] - da[~first]) <= MOTION_REL * np.abs(da[~first])), (call, da, db)
        assert B.sdv2_motion_check(hb) == 0
    finally:
        B.sdv2_motion_destroy(ha)
        B.sdv2_motion_destroy(hb)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from causal_dit_kv_b200 import binding as B
    # 8 streams x 64 frames x 32 blocks of 2048 elements = 16384 partial sums: the limit
    ok_cfg = B.make_motion_config(8, 64, 16, 64, 64)
    big_cfg = B.make_motion_config(9, 64, 16, 64, 64)
    for cfg, fits in ((ok_cfg, True), (big_cfg, False)):
        buf, h = _handle(B, cfg)
        x = torch.zeros((cfg.batch, cfg.chunk_frames, 16, 64, 64), dtype=torch.float32, device="cuda")
        rate = torch.zeros(cfg.batch, dtype=torch.float32, device="cuda")
        try:
            if fits:
                B.sdv2_motion_noise_rate_noalloc(h, x, rate)
                torch.cuda.synchronize()
            else:
                with pytest.raises(B.SDV2Error) as e:
                    B.sdv2_motion_noise_rate_noalloc(h, x, rate)
                assert e.value.status == B.SDV2_E_SHAPE
                assert "16384" in str(e.value)
        finally:
            B.sdv2_motion_destroy(h)
