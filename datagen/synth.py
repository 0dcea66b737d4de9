"""Seeded synthetic mixtures shaped like the workloads the e-means pages measure on.

Every generator takes an explicit seed and a torch device and returns
``(x_train, x_test)`` drawn from ONE mixture (test rows are fresh draws, never
training rows). Data is produced in fixed-size chunks from a single
``torch.Generator`` so that the bytes depend only on (seed, device type, sizes).

The datasets the pages use (DEEP1M, SIFT, SPACEV, DINO10B, the 1B runs) are not
available; these mixtures stand in for them. Nothing here implements any step of
the clustering method.
"""

from __future__ import annotations

import dataclasses

import torch

CHUNK_ROWS = 1 << 21  # rows generated per chunk (bounded temporary memory)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One benchmark configuration: sizes, clustering settings and data recipe."""

    name: str
    n_train: int
    n_test: int
    d: int
    k: int
    epochs: float
    storage: str  # "fp32" or "bf16": the dtype the data is handed over in
    recipe: str  # one-line description of the mixture

    def scaled(self, n_train: int, n_test: int, k: int | None = None) -> "Workload":
        return dataclasses.replace(self, n_train=n_train, n_test=n_test, k=self.k if k is None else k)


WORKLOADS = {
    "tiny": Workload("tiny", 10_000, 2_000, 32, 64, 5.0, "fp32",
                     "64-component isotropic Gaussian mixture, means ~N(0,4I), sigma=1, equal weights"),
    "emb768": Workload("emb768", 1_000_000, 100_000, 768, 4096, 5.0, "fp32",
                       "16384-component mixture, Zipf(1.1) weights, means ~N(0,I), sigma_c~U(0.3,1.0), L2-normalised"),
    "deep96": Workload("deep96", 1_000_000, 100_000, 96, 16384, 5.0, "fp32",
                       "50000-component mixture in a random 96-d basis with power-law(1.5) spectrum, L2-normalised"),
    "sift128": Workload("sift128", 10_000_000, 1_000_000, 128, 65536, 5.0, "bf16",
                        "131072-component integer mixture in [0,255]: round(mu+|N(0,30^2)|), mu~U[0,80], 30% zeros"),
    "stream128": Workload("stream128", 100_000_000, 1_000_000, 128, 262144, 3.0, "bf16",
                          "1e6-component mixture, Zipf(1.05) weights, means ~N(0,I), sigma_c~U(0.3,1.0), L2-normalised"),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _zipf_cdf(m: int, s: float, device) -> torch.Tensor:
    w = torch.arange(1, m + 1, dtype=torch.float64, device=device).pow(-s)
    c = torch.cumsum(w, 0)
    return c / c[-1]


def _draw_components(n: int, cdf: torch.Tensor | None, m: int, g, device) -> torch.Tensor:
    if cdf is None:
        return torch.randint(0, m, (n,), generator=g, device=device)
    u = torch.rand(n, generator=g, device=device, dtype=torch.float64)
    return torch.searchsorted(cdf, u).clamp_(max=m - 1)


def _finish(x: torch.Tensor, storage: str) -> torch.Tensor:
    return x.to(torch.bfloat16) if storage == "bf16" else x.to(torch.float32)


def isotropic_mixture(n_train, n_test, d, ncomp, mean_std, sigma, seed, device, storage="fp32"):
    """Equal-weight isotropic mixture: mu ~ N(0, mean_std^2 I), x = mu + sigma z."""
    g = _gen(seed, device)
    mu = torch.randn(ncomp, d, generator=g, device=device) * mean_std
    out = []
    for n in (n_train, n_test):
        rows = []
        for s in range(0, n, CHUNK_ROWS):
            m = min(CHUNK_ROWS, n - s)
            comp = _draw_components(m, None, ncomp, g, device)
            z = torch.randn(m, d, generator=g, device=device)
            rows.append(_finish(mu[comp] + sigma * z, storage))
        out.append(torch.cat(rows) if rows else torch.empty(0, d, device=device, dtype=torch.float32))
    return out[0], out[1]


def mixture_normalized(n_train, n_test, d, ncomp, zipf_s, seed, device, storage="fp32"):
    """Zipf-weighted mixture with per-component scale, every row L2-normalised.

    mu_c ~ N(0, I), sigma_c ~ U(0.3, 1.0), x = mu_c + sigma_c z, x <- x / |x|.
    """
    g = _gen(seed, device)
    mu = torch.randn(ncomp, d, generator=g, device=device)
    sig = 0.3 + 0.7 * torch.rand(ncomp, generator=g, device=device)
    cdf = _zipf_cdf(ncomp, zipf_s, device)
    out = []
    for n in (n_train, n_test):
        rows = []
        for s in range(0, n, CHUNK_ROWS):
            m = min(CHUNK_ROWS, n - s)
            comp = _draw_components(m, cdf, ncomp, g, device)
            x = mu[comp] + sig[comp, None] * torch.randn(m, d, generator=g, device=device)
            x = x / x.norm(dim=1, keepdim=True).clamp_min(1e-30)
            rows.append(_finish(x, storage))
        out.append(torch.cat(rows) if rows else torch.empty(0, d, device=device, dtype=torch.float32))
    return out[0], out[1]


def subspace_mixture(n_train, n_test, d, ncomp, spectrum_alpha, seed, device, storage="fp32", noise=0.5):
    """Mixture in a random orthonormal basis Q with power-law spectrum lambda_i ~ i^-alpha.

    mean = Q diag(sqrt(lambda)) g, x = mean + noise * Q diag(sqrt(lambda)) z, then L2-normalised.
    """
    g = _gen(seed, device)
    a = torch.randn(d, d, generator=g, device=device, dtype=torch.float64)
    q, r = torch.linalg.qr(a.cpu())
    q = (q * torch.sign(torch.diagonal(r))).to(device=device, dtype=torch.float32)
    lam = torch.arange(1, d + 1, dtype=torch.float32, device=device).pow(-spectrum_alpha)
    scale = lam.sqrt()
    mu = (torch.randn(ncomp, d, generator=g, device=device) * scale) @ q.T
    out = []
    for n in (n_train, n_test):
        rows = []
        for s in range(0, n, CHUNK_ROWS):
            m = min(CHUNK_ROWS, n - s)
            comp = _draw_components(m, None, ncomp, g, device)
            z = (torch.randn(m, d, generator=g, device=device) * scale) @ q.T
            x = mu[comp] + noise * z
            x = x / x.norm(dim=1, keepdim=True).clamp_min(1e-30)
            rows.append(_finish(x, storage))
        out.append(torch.cat(rows) if rows else torch.empty(0, d, device=device, dtype=torch.float32))
    return out[0], out[1]


def sift_like(n_train, n_test, d, ncomp, seed, device, storage="bf16"):
    """Non-negative integer vectors in [0, 255] (exact in bf16).

    mu ~ U[0, 80]^d per component (equal weights); x = clip(round(mu + |N(0, 30^2)|), 0, 255);
    each coordinate is zeroed with probability 0.3.
    """
    g = _gen(seed, device)
    mu = torch.rand(ncomp, d, generator=g, device=device) * 80.0
    out = []
    for n in (n_train, n_test):
        rows = []
        for s in range(0, n, CHUNK_ROWS):
            m = min(CHUNK_ROWS, n - s)
            comp = _draw_components(m, None, ncomp, g, device)
            x = (mu[comp] + (30.0 * torch.randn(m, d, generator=g, device=device)).abs()).round_().clamp_(0, 255)
            keep = torch.rand(m, d, generator=g, device=device) >= 0.3
            rows.append(_finish(x * keep, storage))
        out.append(torch.cat(rows))
    return out[0], out[1]


def make(name: str, device="cpu", seed: int = 0, n_train: int | None = None, n_test: int | None = None):
    """Build a named workload (optionally at reduced row counts). Returns (Workload, x_train, x_test)."""
    w = WORKLOADS[name]
    if n_train is not None or n_test is not None:
        w = w.scaled(n_train if n_train is not None else w.n_train, n_test if n_test is not None else w.n_test)
    if name == "tiny":
        xt, xs = isotropic_mixture(w.n_train, w.n_test, w.d, 64, 2.0, 1.0, seed, device, w.storage)
    elif name == "emb768":
        xt, xs = mixture_normalized(w.n_train, w.n_test, w.d, 16384, 1.1, seed, device, w.storage)
    elif name == "deep96":
        xt, xs = subspace_mixture(w.n_train, w.n_test, w.d, 50_000, 1.5, seed, device, w.storage)
    elif name == "sift128":
        xt, xs = sift_like(w.n_train, w.n_test, w.d, 131_072, seed, device, w.storage)
    elif name == "stream128":
        xt, xs = mixture_normalized(w.n_train, w.n_test, w.d, 1_000_000, 1.05, seed, device, w.storage)
    else:
        raise KeyError(name)
    return w, xt, xs


def hand_shape(n: int, d: int, ncomp: int, seed: int, device="cpu", storage="fp32", normalized=False):
    """Small mixtures for parity cases at arbitrary (n, d)."""
    if normalized:
        x, _ = mixture_normalized(n, 0, d, ncomp, 1.1, seed, device, storage)
    else:
        x, _ = isotropic_mixture(n, 0, d, ncomp, 2.0, 1.0, seed, device, storage)
    return x


def blobs3(seed: int = 7):
    """Three 2-D Gaussian blobs of 40 points each and a deliberately bad start.

    The start puts two centroids inside one blob and one midway between the
    other two, the situation the blog's own small simulation describes.
    Returns (x [120, 2] float64 tensor, start [3, 2] float64 tensor).
    """
    g = _gen(seed, "cpu")
    centers = torch.tensor([[0.0, 6.0], [-5.0, -3.0], [5.0, -3.0]], dtype=torch.float64)
    x = torch.cat([c + torch.randn(40, 2, generator=g, dtype=torch.float64) for c in centers])
    start = torch.tensor([[-0.6, 6.0], [0.6, 6.0], [0.0, -3.0]], dtype=torch.float64)
    return x, start


def zipf_cdf_for_tests(m: int, s: float):
    """Exposed for data-shape tests only."""
    return _zipf_cdf(m, s, "cpu")


def expected_tiny_noise_floor(d: int = 32, sigma: float = 1.0) -> float:
    """E|sigma z|^2 for the isotropic tiny mixture: the MSE of the true partition."""
    return d * sigma * sigma

