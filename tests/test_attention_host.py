"""The library's host-side chunk set of the attention anchors (nvfp4_attention_chunks,
no GPU needed) against the hand-worked golden sets and the oracle's definition."""
import os

import numpy as np
import pytest

import oracle
from bit_video_dit_b200 import nvfp4 as nv

from .test_oracle_attention import _golden


@pytest.mark.parametrize("args,want", _golden())
def test_library_chunk_set_matches_the_golden_sets(args, want):
    assert nv.attention_chunks(*args) == want


def test_library_chunk_set_matches_the_oracle_on_random_arguments():
    rng = np.random.default_rng(0)
    for _ in range(2000):
        t = int(rng.integers(0, 80))
        args = (t, int(rng.integers(0, 6)), int(rng.integers(0, 90)), int(rng.integers(0, 6)), int(rng.integers(0, 12)))
        assert nv.attention_chunks(*args) == oracle.attention_chunks(*args), args


def test_library_chunk_set_rejects_bad_arguments():
    import ctypes
    buf = (ctypes.c_int32 * 4)()
    L = nv.lib()
    assert L.nvfp4_attention_chunks(10, -1, 0, 0, 2, buf, 4) == -1
    assert L.nvfp4_attention_chunks(10, 2, 0, 0, 8, buf, 4) == -1  # more than max_out chunks
