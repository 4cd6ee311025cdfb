"""Counter-based random numbers for the method's own random draws (oracle side).

The method draws random parameters -- unit rotors ("TurboQuant + RotorQuant",
section "How RotorQuant Works"), the Gaussian matrix whose QR factor is Pi
("TurboQuant 论文解读", section "随机旋转（Lemma 1）" and its demo), and the
QJL Gaussian matrix (same blog, section "QJL 内积无偏估计（Theorem 2）"). The
pages do not fix a generator. Both this oracle and the library implement, each
on its own, the same published counter-based generator so that their draws can
be compared:

* splitmix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): the i-th output of the stream with seed ``s`` is
  ``mix64(s + (i + 1) * 0x9E3779B97F4A7C15 mod 2**64)`` with
  ``mix64(z) = z3 ^ (z3 >> 31)``, ``z3 = (z2 ^ (z2 >> 27)) * 0x94D049BB133111EB``,
  ``z2 = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9`` (all mod 2**64).
* uniform in (0, 1]: ``((out >> 11) + 1) * 2**-53``.
* Box-Muller (1958): normals 2j and 2j+1 come from uniforms u1 = U(2j),
  u2 = U(2j+1) as ``sqrt(-2 ln u1) * (cos(2 pi u2), sin(2 pi u2))``.
"""

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed, index):
    """Outputs ``index`` (array of stream positions, from 0) of the stream ``seed``."""
    idx = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed) + (idx + np.uint64(1)) * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform(seed, index):
    """Uniform doubles in (0, 1] at stream positions ``index``."""
    z = splitmix64(seed, index)
    return ((z >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def normals(seed, count):
    """The first ``count`` standard normals of stream ``seed`` (Box-Muller pairs)."""
    pairs = (count + 1) // 2
    j = np.arange(pairs, dtype=np.uint64)
    u1 = uniform(seed, 2 * j)
    u2 = uniform(seed, 2 * j + np.uint64(1))
    r = np.sqrt(-2.0 * np.log(u1))
    out = np.empty(2 * pairs, dtype=np.float64)
    out[0::2] = r * np.cos(2.0 * np.pi * u2)
    out[1::2] = r * np.sin(2.0 * np.pi * u2)
    return out[:count]
