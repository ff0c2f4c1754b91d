"""Pins for the oracle's bf16 rounding and ring/phase mapping (CPU only)."""
import collections
import os

import numpy as np
import pytest
import torch

from oracle import (bf16_decode, bf16_encode, bf16_round, rope_phase, slot_frames, slot_of_frame,
                    valid_slot_counts)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if line:
                yield line.split()


def test_bf16_hand_derived_cases():
    for hexval, bits in _rows("bf16_rne_cases.txt"):
        x = float.fromhex(hexval)
        got = int(bf16_encode(np.array([x]))[0])
        assert got == int(bits, 16), (hexval, hex(got), bits)


def test_bf16_matches_torch_on_fp32_values():
    # For inputs that are exact fp32 values, fp64->bf16 RNE equals torch's fp32->bf16 RNE.
    g = torch.Generator().manual_seed(5)
    x = torch.randn(200_000, generator=g) * torch.exp(torch.randn(200_000, generator=g) * 8)
    x = torch.cat([x, torch.tensor([0.0, -0.0, 1e-40, -1e-41, 3.0e38, -3.39e38])])
    want = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = bf16_encode(x.numpy().astype(np.float64))
    assert np.array_equal(got, want)


def test_bf16_decode_roundtrip_all_patterns():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        vals = bf16_decode(bits)
    finite = np.isfinite(vals)
    assert np.array_equal(bf16_encode(vals[finite]), bits[finite])
    # every finite bf16 value is a fixed point of the rounding
    assert np.array_equal(bf16_round(vals[finite]), vals[finite])


def _deque_sim(S, W, n_frames):
    """Literal simulation: sinks fixed, window a FIFO of at most W frames."""
    sinks, window = [], collections.deque()
    states = []
    for f in range(n_frames):
        if len(sinks) < S:
            sinks.append(f)
        else:
            window.append(f)
            if len(window) > W:
                window.popleft()
        states.append((list(sinks), list(window)))
    return states


@pytest.mark.parametrize("S,W", [(1, 2), (2, 3), (1, 6), (3, 4), (1, 1), (4, 8)])
def test_ring_matches_deque_simulation(S, W):
    states = _deque_sim(S, W, 5 * (S + W) + 3)
    for f, (sinks, window) in enumerate(states):
        held = slot_frames(f + 1, S, W)
        s_valid, w_valid = valid_slot_counts(f + 1, S, W)
        assert held[:S][:s_valid] == sinks
        assert s_valid == len(sinks) and w_valid == len(window)
        # valid slots form a prefix; the window holds exactly the deque's frames
        assert all(x >= 0 for x in held[:s_valid + w_valid])
        assert all(x == -1 for x in held[s_valid + w_valid:])
        assert sorted(held[S:S + w_valid]) == window
        assert held[slot_of_frame(f, S, W)] == f


@pytest.mark.parametrize("name,S,W", [("ring_S1_W2.txt", 1, 2), ("ring_S2_W3.txt", 2, 3)])
def test_ring_hand_table(name, S, W):
    for row in _rows(name):
        f, slot, sv, wv = (int(x) for x in row[:4])
        held = [int(x) for x in row[4:]]
        assert slot_of_frame(f, S, W) == slot
        assert valid_slot_counts(f + 1, S, W) == (sv, wv)
        assert slot_frames(f + 1, S, W) == held


def test_phase_reset():
    assert [rope_phase(f, 4) for f in range(10)] == [0, 1, 2, 3, 0, 1, 2, 3, 0, 1]
    assert [rope_phase(f, 0) for f in range(5)] == [0, 1, 2, 3, 4]
    assert rope_phase(256 + 17, 256) == 17
