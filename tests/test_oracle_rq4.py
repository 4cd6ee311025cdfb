"""Pins of the four-grade RotorQuant layout (oracle/rq4.py) against the page's storage table and
against the algebra: a unit-rotor sandwich of a vector has a zero trivector part, and the inverse
sandwich leaves a pseudoscalar unchanged, so the fourth code of a group never changes x_hat."""

import os

import numpy as np

from oracle import codebook, codes as ocodes, params, rq, rq4

D = 128
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _table():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "rq_tq_storage_table.txt"))
            if ln.strip() and not ln.startswith("#")]
    return {r[0]: (int(r[1]), float(r[2])) for r in rows}


def test_page_storage_table():
    t = _table()
    # RotorQuant: 4 indices per group of 43; 3-bit codes plus a 4-byte norm
    assert rq4.N_PER_GROUP * params.n_groups(D) == t["rotorquant"][0]
    assert round(2 * D / rq4.bytes_per_vector(D, 3), 1) == t["rotorquant"][1]
    # TurboQuant-mse: one index per coordinate, 48 bytes of 3-bit codes plus the norm
    assert D == t["turboquant"][0]
    assert round(2 * D / (ocodes.n_words(D, 3) * 4 + 4), 1) == t["turboquant"][1]
    # the three-component layout stored here would be 129 indices, 4.57x: not the page's layout
    assert round(2 * D / (ocodes.n_words(129, 3) * 4 + 4), 2) == 4.57


def test_codes_and_reconstruction():
    rot = params.rotors(D, 1)
    c = codebook.lloyd_max(D, 3)[0]
    x = np.random.default_rng(0).standard_normal((200, D))
    x[3] = 0
    q4 = rq4.quantize(x, rot, c, 3)
    q3 = rq.quantize(x, rot, c, 3)
    G = params.n_groups(D)
    codes4 = q4["codes"].reshape(200, G, 4)
    # trivector parts vanish for unit rotors and take the code of 0; vector codes as in the 3-code layout
    assert np.abs(q4["mv"][..., 7]).max() < 1e-12
    assert np.all(codes4[..., 3] == 3)  # the code of 0: the lower of the two middle centroids (ties low)
    assert ocodes.nearest(np.zeros(1), c)[0] == 3
    np.testing.assert_array_equal(codes4[..., :3].reshape(200, 3 * G), q3["codes"])
    assert q4["words"].shape[1] == ocodes.n_words(172, 3) == 17
    xh4 = rq4.dequantize(q4["words"], q4["norms"], rot, c, 3, D)
    xh3 = rq.dequantize(q3["words"], q3["norms"], rot, c, 3, D)
    np.testing.assert_allclose(xh4, xh3, rtol=0, atol=1e-12)
    # any trivector code gives the same x_hat (R~ e123 R = e123 has no vector part)
    codes4 = codes4.copy()
    codes4[..., 3] = np.random.default_rng(1).integers(0, 8, size=codes4[..., 3].shape)
    xh4b = rq4.dequantize(ocodes.pack(codes4.reshape(200, 4 * G), 3), q4["norms"], rot, c, 3, D)
    np.testing.assert_allclose(xh4b, xh3, rtol=0, atol=1e-12)
