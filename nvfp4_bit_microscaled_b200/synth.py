"""Seeded synthetic inputs shaped like a 12B hybrid Mamba-Transformer's linear layers.

This module only draws random numbers; it holds none of the quantization
arithmetic.  Tests feed the very same BF16 bytes to the CUDA path and to the CPU
oracle, and ``bench.py`` uses it for its timed workloads.

Distributions (all cast to BF16 at the end):
  activations  X  ~ N(0, 1) with 0.1 % of the channels (at least one) scaled x100
                    (outlier columns, the case the RHT and the E4M3 scales target)
  weights      W  ~ N(0, 0.02), optionally with a fraction of entries scaled
  gradients    dY ~ N(0, 1e-3) with a per-row log-normal(0, 1) factor
  heavy        X  ~ Student-t(3), built as Z / sqrt(chi2_3 / 3) from normals
Each tensor of one workload draws from its own generator (seed * 16 + slot),
so a tensor is the same bytes whichever workload asks for it.
"""
import torch

SLOT_X, SLOT_W, SLOT_DY, SLOT_TILE = 1, 2, 3, 4


def _gen(seed, slot, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 16 + slot)
    return g


def activations(T, C, seed, device="cpu", outlier_frac=1e-3, outlier_scale=100.0):
    g = _gen(seed, SLOT_X, device)
    x = torch.randn(T, C, generator=g, device=device, dtype=torch.float32)
    n_out = max(1, round(outlier_frac * C)) if outlier_frac > 0 else 0
    if n_out:
        cols = torch.randperm(C, generator=g, device=device)[:n_out]
        x[:, cols] *= outlier_scale
    return x.to(torch.bfloat16)


def heavy_activations(T, C, seed, device="cpu", nu=3):
    g = _gen(seed, SLOT_X, device)
    z = torch.randn(T, C, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros_like(z)
    for _ in range(nu):
        chi2 += torch.randn(T, C, generator=g, device=device, dtype=torch.float32).square()
    return (z / torch.sqrt(chi2 / nu)).to(torch.bfloat16)


def weights(N, K, seed, device="cpu", std=0.02, outlier_frac=0.0, outlier_scale=50.0):
    g = _gen(seed, SLOT_W, device)
    w = torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * std
    n_out = round(outlier_frac * N * K)
    if n_out:
        idx = torch.randperm(N * K, generator=g, device=device)[:n_out]
        w.view(-1)[idx] *= outlier_scale
    return w.to(torch.bfloat16)


def gradients(T, N, seed, device="cpu", std=1e-3, row_lognormal=True):
    g = _gen(seed, SLOT_DY, device)
    d = torch.randn(T, N, generator=g, device=device, dtype=torch.float32) * std
    if row_lognormal:
        d *= torch.exp(torch.randn(T, 1, generator=g, device=device, dtype=torch.float32))
    return d.to(torch.bfloat16)


def normal(R, C, seed, device="cpu", std=1.0, slot=SLOT_TILE):
    g = _gen(seed, slot, device)
    return (torch.randn(R, C, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


# --------------------------------------------------------------------------
# The five workloads.  Shapes follow the 12B model's linear layers
# (hidden 5120, FFN 20480) plus one large outlier-heavy case.
# --------------------------------------------------------------------------
WORKLOADS = {
    "tiny": dict(T=128, Cin=256, Cout=128, seed=0),
    "fprop": dict(T=8192, Cin=5120, Cout=20480, seed=1),
    "wgrad": dict(T=8192, Cin=5120, Cout=20480, seed=1),
    "full": dict(T=16384, Cin=5120, Cout=20480, seed=2),
    "large": dict(T=32768, Cin=8192, Cout=8192, seed=3),
}


def workload_inputs(name, device="cpu", scale_down=1):
    """X [T, Cin], W [Cout, Cin], dY [T, Cout] for a named workload.

    scale_down divides every dimension (keeping multiples of 128) so the same
    distributions can be checked at sizes the CPU oracle handles in seconds.
    """
    p = dict(WORKLOADS[name])

    def sd(v):
        return max(128, (v // scale_down) // 128 * 128)

    T, Cin, Cout, seed = sd(p["T"]), sd(p["Cin"]), sd(p["Cout"]), p["seed"]
    if name == "tiny":
        x = normal(T, Cin, seed, device, slot=SLOT_X)
        w = normal(Cout, Cin, seed, device, slot=SLOT_W)
        dy = normal(T, Cout, seed, device, std=1e-3, slot=SLOT_DY)
    elif name == "large":
        x = heavy_activations(T, Cin, seed, device)
        w = weights(Cout, Cin, seed, device, outlier_frac=1e-4, outlier_scale=50.0)
        dy = gradients(T, Cout, seed, device, row_lognormal=False)
    else:
        x = activations(T, Cin, seed, device)
        w = weights(Cout, Cin, seed, device)
        dy = gradients(T, Cout, seed, device)
    return x, w, dy
