"""Seeded synthetic KV-shaped inputs (no quantization arithmetic here).

The pages measure on real model caches (Qwen2.5-3B, Llama-3.1-8B) that are not
available; these generators stand in for them with the shapes and value
structure the workloads name:

* ``gaussian``   -- i.i.d. N(0, 1) rows.
* ``lognormal``  -- direction uniform on the sphere (normalised Gaussian), norm
  ~ LogNormal(0, 0.5), optionally a fixed set of outlier channels scaled x10.
* ``factor_keys``-- per (layer, head) a rank-r Gaussian factor model k = W z
  (W ~ N(0, 1/r), z ~ N(0, I_r)) plus outlier channels scaled x10.

All draw from ``torch.Generator`` seeded explicitly, on the CPU or directly on
a CUDA device for the large bench inputs.
"""

import torch

OUTLIER_CHANNELS = (3, 47, 88, 121)  # distinct rotor groups at d = 128
OUTLIER_SCALE = 10.0


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gaussian(n, d, seed=0, dtype=torch.float32, device="cpu"):
    g = _gen(seed, device)
    return torch.randn((n, d), generator=g, device=device, dtype=torch.float32).to(dtype)


def lognormal(n, d, seed=0, dtype=torch.float16, device="cpu", outliers=OUTLIER_CHANNELS, sigma=0.5,
              chunk=1 << 20):
    """Rows = (g / ||g||) * rho, rho ~ LogNormal(0, sigma); outlier channels (< d) x10."""
    out = torch.empty((n, d), dtype=dtype, device=device)
    g = _gen(seed, device)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        z = torch.randn((e - s, d), generator=g, device=device, dtype=torch.float32)
        rho = torch.exp(sigma * torch.randn((e - s, 1), generator=g, device=device, dtype=torch.float32))
        z = z / z.norm(dim=1, keepdim=True) * rho
        for c in outliers:
            if c < d:
                z[:, c] *= OUTLIER_SCALE
        out[s:e] = z.to(dtype)
    return out


def factor_keys(layers, heads, tokens, d, rank=16, seed=0, dtype=torch.bfloat16, device="cpu",
                outliers=OUTLIER_CHANNELS):
    """[layers, heads, tokens, d] keys from a rank-`rank` factor model per (layer, head)."""
    out = torch.empty((layers, heads, tokens, d), dtype=dtype, device=device)
    g = _gen(seed, device)
    for l in range(layers):
        for h in range(heads):
            W = torch.randn((d, rank), generator=g, device=device) / rank ** 0.5
            z = torch.randn((tokens, rank), generator=g, device=device)
            k = z @ W.T
            for c in outliers:
                if c < d:
                    k[:, c] *= OUTLIER_SCALE
            out[l, h] = k.to(dtype)
    return out
