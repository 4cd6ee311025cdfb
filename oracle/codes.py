"""Nearest-centroid scalar quantization and the packed code layout.

"TurboQuant 论文解读", demo ("简单复现 demo"): each rotated coordinate gets the
index of the nearest codebook entry, argmin_i |y - c_i|. The arXiv summary page
("方法", Algorithm 1) says the same: quantization finds the nearest centroid of
each rotated coordinate. Ties go to the lower index (the first minimum, which is
what numpy's argmin returns); codes count up with the centroids.

Packed layout (the pages store "indices" but give no bit layout; this is the
plain reading): each row is one little-endian bit stream, code j occupies bits
[j*b, j*b + b) with its least significant bit first, and the stream is cut into
32-bit words, W = ceil(n_codes * b / 32) per row; unused high bits are zero.
"""

import numpy as np


def nearest(y, centroids):
    """Index of the nearest centroid for every entry of y (ties -> lower index)."""
    y = np.asarray(y, dtype=np.float64)
    c = np.asarray(centroids, dtype=np.float64)
    return np.abs(y[..., None] - c).argmin(axis=-1)


def n_words(n_codes, bits):
    """W = ceil(n_codes * bits / 32)."""
    return -(-(n_codes * bits) // 32)


def pack(codes, bits):
    """Pack integer codes [N, n] (each < 2^bits) into uint32 words [N, W]."""
    codes = np.asarray(codes, dtype=np.int64)
    N, n = codes.shape
    W = n_words(n, bits)
    stream = np.zeros((N, 32 * W), dtype=np.int64)
    for j in range(n):
        for i in range(bits):
            stream[:, j * bits + i] = (codes[:, j] >> i) & 1
    weights = np.array([1 << k for k in range(32)], dtype=np.int64)
    words = (stream.reshape(N, W, 32) * weights).sum(axis=2)
    return words.astype(np.uint32)


def unpack(words, n_codes, bits):
    """Inverse of ``pack``: uint32 words [N, W] -> codes [N, n_codes]."""
    words = np.asarray(words, dtype=np.uint32).astype(np.int64)
    N, W = words.shape
    stream = (words[:, :, None] >> np.arange(32)[None, None, :]) & 1
    stream = stream.reshape(N, 32 * W)
    codes = np.zeros((N, n_codes), dtype=np.int64)
    for i in range(bits):
        codes |= stream[:, i : n_codes * bits : bits][:, :n_codes] << i
    return codes
