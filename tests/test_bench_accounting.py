"""bench.py's algorithmic-byte accounting, which sets roofline.achieved, against the per-vector
figures derived from the storage layout: packed words W = ceil(n_codes * b / 32) with 3G = 3 ceil(d/3)
RotorQuant codes (d = 128: 129 codes) or d TurboQuant codes, a 4-byte norm, fp16 in and out."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import kv_cache_vector_rq_b200 as kvrq  # noqa: E402


@pytest.mark.parametrize("d,words", [(128, (9, 13, 17)), (256, (17, 25, 33)), (1536, (96, 144, 192)),
                                     (4096, (257, 385, 513))])
def test_rotorquant_words_per_row(d, words):
    for b, w in zip((2, 3, 4), words):
        assert kvrq.packed_words(3 * kvrq.rq_groups(d), b) == w
        assert bench.rq_bytes_per_vector(d, b) == 2 * d + 4 * w + 4 + 2 * d


def test_headline_bytes():
    # fused roundtrip at d = 128, b = 3: 256 B in + 52 B codes + 4 B norm + 256 B out
    assert bench.rq_bytes_per_vector(128, 3) == 568
    # quantize-only / dequantize-only sides of the same row
    assert bench.rq_bytes_per_vector(128, 3, out_bytes=0) == 312
    assert bench.rq_bytes_per_vector(128, 3, in_bytes=0) == 312
    # TurboQuant-mse roundtrip: 128 codes of 3 bits = 12 words
    assert bench.tq_bytes_per_vector(128, 3) == 256 + 48 + 4 + 256
    assert bench.tq_bytes_per_vector(128, 3, out_bytes=0) == 308
