"""Exhaustive check of the device E2M1 / E4M3 encoders against the oracle.

Every kernel encodes through the same two device functions (hardware
conversions).  Both they and the oracle's encoders are monotone step
functions of the input, so they are equal on all 2^32 binary32 inputs iff
(1) the device encoder is monotone over the whole range, and (2) it changes
code at exactly the same inputs as the oracle.  The sweep below checks (1) on
every finite input and (2) at every transition it finds, plus the sign rule
(R7: negative inputs, -0 included, carry the sign bit).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_video_dit_b200 import nvfp4 as nv

from .gpu_util import require_gpu

pytestmark = pytest.mark.gpu

CHUNK = 1 << 27
POS_END = 0x7F800000  # +inf bit pattern (exclusive): all finite non-negative floats


def _sweep(kind: str, sign: int):
    """Yield (magnitude codes, raw codes, first bits) for chunks of the range."""
    start = 0
    while start < POS_END:
        n = min(CHUNK, POS_END - start)
        bits = torch.arange(start, start + n, dtype=torch.int64, device="cuda")
        if sign:
            bits = bits | 0x80000000
        x = bits.to(torch.int64).bitwise_and(0xFFFFFFFF).to(torch.int64)
        x = torch.where(x >= 2 ** 31, x - 2 ** 32, x).to(torch.int32).view(torch.float32)
        e2, e4 = nv.test_encode(x, e2m1=(kind == "e2m1"), e4m3=(kind == "e4m3"))
        codes = e2 if kind == "e2m1" else e4
        yield start, codes
        start += n


def _bits_to_float(b: int) -> float:
    return float(np.array([b], np.uint32).view(np.float32)[0])


@pytest.mark.parametrize("kind,sign", [("e2m1", 0), ("e2m1", 1), ("e4m3", 0)])
def test_encoder_matches_oracle_on_all_inputs(kind, sign):
    require_gpu()
    enc = oracle.e2m1_encode if kind == "e2m1" else oracle.e4m3_encode
    mag_mask = 7 if kind == "e2m1" else 0x7F
    prev_last = None
    transitions = []
    for start, codes in _sweep(kind, sign):
        c = codes.to(torch.int32)
        if kind == "e2m1":
            signs = (c >> 3) & 1
            assert bool((signs == sign).all()), "sign bit rule broken"
        mag = c & mag_mask
        d = mag[1:] - mag[:-1]
        assert bool((d >= 0).all()), f"{kind} encoder not monotone in chunk at {start:#x}"
        idx = torch.nonzero(d).flatten().cpu().numpy()
        for i in idx:
            transitions.append((start + int(i), start + int(i) + 1))
        first = int(mag[0])
        if prev_last is not None:
            assert first >= prev_last[1]
            if first != prev_last[1]:
                transitions.append((prev_last[0], start))
        prev_last = (start + int(mag.numel()) - 1, int(mag[-1]))
    expected = 7 if kind == "e2m1" else 126
    assert len(transitions) == expected, len(transitions)
    for lo, hi in transitions:
        for b in (lo, hi):
            bits = b | (0x80000000 if sign else 0)
            x = _bits_to_float(bits)
            xt = torch.tensor([x], dtype=torch.float32, device="cuda")
            e2, e4 = nv.test_encode(xt)
            got = int((e2 if kind == "e2m1" else e4)[0])
            assert got == enc(x), (kind, hex(bits), got, enc(x))
    # endpoints
    for b in (0, POS_END - 1):
        bits = b | (0x80000000 if sign else 0)
        x = _bits_to_float(bits)
        e2, e4 = nv.test_encode(torch.tensor([x], dtype=torch.float32, device="cuda"))
        got = int((e2 if kind == "e2m1" else e4)[0])
        assert got == enc(x)
