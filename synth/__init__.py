"""Seeded synthetic inputs for the Q-GaLore optimizer step.

Holds none of the method's arithmetic: it only draws gradients, weight codes and
weight scales with the shapes and value distributions of the workloads, for the
oracle and the GPU path alike.  Every draw is a deterministic function of its
seed.

Gradient model (low rank plus noise): G = U diag(s) V^T + sigma * E with U, V
Haar-distributed orthonormal columns (QR of a Gaussian with the diagonal sign of
R made positive), s_i = s0 * decay^i, E standard normal; G is rounded to bf16.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

# --------------------------------------------------------------------------
# Shapes of the workloads (LLaMA-style projection matrices)
# --------------------------------------------------------------------------

LLAMA_SHAPES = {
    "llama60m": dict(hidden=512, inter=1376, layers=8, r=128),
    "llama1b": dict(hidden=2048, inter=5461, layers=24, r=512),
    "llama7b": dict(hidden=4096, inter=11008, layers=32, r=1024),
}


def llama_layer_shapes(hidden, inter):
    """(name, m, n) of the seven matrices of one decoder layer, in stack order."""
    return [("q", hidden, hidden), ("k", hidden, hidden), ("v", hidden, hidden),
            ("o", hidden, hidden), ("gate", hidden, inter), ("up", hidden, inter),
            ("down", inter, hidden)]


def stack_shapes(name):
    d = LLAMA_SHAPES[name]
    out = []
    for _ in range(d["layers"]):
        out += [(m, n) for _, m, n in llama_layer_shapes(d["hidden"], d["inter"])]
    return out, d["r"]


# --------------------------------------------------------------------------
# CPU (numpy) generators: small and medium sizes, bit-identical everywhere
# --------------------------------------------------------------------------


def haar_columns(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    a = rng.standard_normal((n, k))
    q, r = np.linalg.qr(a)
    return q * np.sign(np.where(np.diag(r) == 0, 1.0, np.diag(r)))[None, :]


def to_bf16(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round to bf16 with torch; returns (float32 values, uint16 bit patterns)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    bits = t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.to(torch.float32).numpy(), bits


@dataclass
class LowRankGradient:
    U: np.ndarray
    V: np.ndarray
    s: np.ndarray
    sigma: float
    seed: int

    def draw(self, step: int) -> tuple[np.ndarray, np.ndarray]:
        """The gradient of step `step`: fixed signal, noise redrawn per step."""
        rng = np.random.default_rng([self.seed, 7, step])
        m, n = self.U.shape[0], self.V.shape[0]
        g = (self.U * self.s[None, :]) @ self.V.T + self.sigma * rng.standard_normal((m, n))
        return to_bf16(g)


def lowrank_gradient(m, n, rank, s0=1e-2, decay=0.8, sigma=1e-4, seed=0) -> LowRankGradient:
    rng = np.random.default_rng([seed, 1])
    rank = min(rank, m, n)
    U = haar_columns(rng, m, rank)
    V = haar_columns(rng, n, rank)
    s = s0 * decay ** np.arange(rank)
    return LowRankGradient(U, V, s, sigma, seed)


def gap_gradient(m, n, r, top=1.0, bottom=0.2, noise_edge_ratio=0.02, seed=0):
    """A matrix whose top r singular values lie in [bottom, top] and whose noise
    edge sigma*(sqrt(m)+sqrt(n)) is `noise_edge_ratio` * bottom: a clear gap
    after the r-th singular value.  Returns (float32 bf16 values, bits)."""
    rng = np.random.default_rng([seed, 3])
    U = haar_columns(rng, m, r)
    V = haar_columns(rng, n, r)
    s = np.linspace(top, bottom, r)
    sigma = noise_edge_ratio * bottom / (np.sqrt(m) + np.sqrt(n))
    g = (U * s[None, :]) @ V.T + sigma * rng.standard_normal((m, n))
    return to_bf16(g)


def weight_codes(m, n, seed=0) -> np.ndarray:
    rng = np.random.default_rng([seed, 11])
    return rng.integers(-127, 128, size=(m, n), dtype=np.int64).astype(np.int8)


def weight_scales(m, n, group=256, base=4.7e-4, seed=0) -> np.ndarray:
    rng = np.random.default_rng([seed, 13])
    ng = -(-(m * n) // group)
    return (base * rng.uniform(0.5, 1.5, size=ng)).astype(np.float32)


def orthonormal(m, r, seed=0) -> np.ndarray:
    return haar_columns(np.random.default_rng([seed, 17]), m, r)


# --------------------------------------------------------------------------
# GPU (torch) generators: full-size stacks, drawn on the device
# --------------------------------------------------------------------------


def device_lowrank_gradient(m, n, rank, s0, decay, sigma, seed, device, pad_to=8):
    """bf16 m x ld gradient on `device` (ld = n rounded up to `pad_to`, padding
    zero): U diag(s) V^T + sigma * E with Haar U, V drawn by torch on the device."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    rank = min(rank, m, n)
    a = torch.randn(m, rank, generator=g, device=device, dtype=torch.float32)
    b = torch.randn(n, rank, generator=g, device=device, dtype=torch.float32)
    qa, ra = torch.linalg.qr(a)
    qb, rb = torch.linalg.qr(b)
    qa = qa * torch.sign(torch.diagonal(ra))[None, :]
    qb = qb * torch.sign(torch.diagonal(rb))[None, :]
    s = s0 * decay ** torch.arange(rank, device=device, dtype=torch.float32)
    ld = -(-n // pad_to) * pad_to
    out = torch.zeros(m, ld, device=device, dtype=torch.bfloat16)
    full = (qa * s[None, :]) @ qb.T
    full += sigma * torch.randn(m, n, generator=g, device=device, dtype=torch.float32)
    out[:, :n] = full.to(torch.bfloat16)
    return out


def device_weight_codes(m, n, ldw, seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 7919 + 1)
    w = torch.zeros(m, ldw, device=device, dtype=torch.int8)
    w[:, :n] = torch.randint(-127, 128, (m, n), generator=g, device=device, dtype=torch.int16).to(torch.int8)
    return w


def device_weight_scales(m, n, seed, device, group=256, base=4.7e-4):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 7919 + 2)
    ng = -(-(m * n) // group)
    return base * (0.5 + torch.rand(ng, generator=g, device=device, dtype=torch.float32))


class DeviceDriftingGradient:
    """bf16 m x n gradients on the device whose signal subspace drifts.

    G_t = U_t diag(s) V^T + sigma E_t with s_i = s0 * decay^i (i < rank), Haar U_0,
    V and W (W orthonormal and orthogonal to U_0, drawn with them), and
    U_t = U_0 cos(theta_t) + W sin(theta_t): each left singular vector turns in
    its own plane (u_i, w_i) by theta_t = rate * min(t, freeze).  E_t is standard
    normal noise redrawn at every step from (seed, t)."""

    def __init__(self, m, n, rank, s0, decay, sigma, rate, freeze, seed, device, pad_to=8):
        g = torch.Generator(device=device)
        g.manual_seed(int(seed))
        self.m, self.n, self.rank = m, n, min(rank, m // 2, n)
        a = torch.randn(m, 2 * self.rank, generator=g, device=device, dtype=torch.float32)
        q, rr = torch.linalg.qr(a)
        q = q * torch.sign(torch.diagonal(rr))[None, :]
        self.U0, self.W = q[:, : self.rank].contiguous(), q[:, self.rank:].contiguous()
        b = torch.randn(n, self.rank, generator=g, device=device, dtype=torch.float32)
        qb, rb = torch.linalg.qr(b)
        s = s0 * decay ** torch.arange(self.rank, device=device, dtype=torch.float32)
        self.SVt = (s[:, None] * (qb * torch.sign(torch.diagonal(rb))[None, :]).T).contiguous()
        self.sigma, self.rate, self.freeze, self.seed = sigma, rate, freeze, int(seed)
        self.ld = -(-n // pad_to) * pad_to
        self.device = device
        self.out = torch.zeros(m, self.ld, device=device, dtype=torch.bfloat16)

    def draw(self, t):
        import math
        th = self.rate * min(t, self.freeze)
        U = self.U0 * math.cos(th) + self.W * math.sin(th)
        g = torch.Generator(device=self.device)
        g.manual_seed(self.seed * 1000003 + t + 1)
        full = U @ self.SVt
        full += self.sigma * torch.randn(self.m, self.n, generator=g, device=self.device, dtype=torch.float32)
        self.out[:, : self.n] = full.to(torch.bfloat16)
        return self.out


class DeviceLinearLayerBatch:
    """Activations and output gradients of one linear layer y = W x over a batch
    of B tokens, on the device, for gradients G = (1/B) D^T X (the weight-gradient
    model of the paper's Theorem 3.1: G lies in the principal subspaces of the
    inputs and of the output gradients).

    X_t = Z_t diag(s) A + sigma E_t                (B x n, bf16)
    D_t = (Z_t M diag(s) C_t + sigma F_t) / B      (B x m, bf16)

    A (k x n) has orthonormal rows, M is a Haar-random orthogonal k x k matrix
    (so the k directions of the output gradients stay well conditioned),
    s_i = decay^i; Z_t, E_t, F_t are standard normal and redrawn at every step
    from (seed, t).  The output-gradient subspace moves until the layer settles:
    C_t = cos(theta_t) C_0 + sin(theta_t) C_1, with C_0, C_1 (k x m) orthonormal
    rows, orthogonal to each other, so each row turns in its own plane by
    theta_t = rate * min(t, freeze) and then stays."""

    def __init__(self, m, n, B, k, decay, sigma, rate, freeze, seed, device, pad_to=8):
        g = torch.Generator(device=device)
        g.manual_seed(int(seed))
        self.m, self.n, self.B, self.k = m, n, B, min(k, m // 2)
        k = self.k
        qa, ra = torch.linalg.qr(torch.randn(n, k, generator=g, device=device))
        qc, rc = torch.linalg.qr(torch.randn(m, 2 * k, generator=g, device=device))
        qc = qc * torch.sign(torch.diagonal(rc))[None, :]
        s = decay ** torch.arange(k, device=device, dtype=torch.float32)
        self.SA = (s[:, None] * (qa * torch.sign(torch.diagonal(ra))[None, :]).T).contiguous()
        self.C0, self.C1 = qc[:, :k].T.contiguous(), qc[:, k:].T.contiguous()
        qm, rm = torch.linalg.qr(torch.randn(k, k, generator=g, device=device))
        self.SM = (qm * torch.sign(torch.diagonal(rm))[None, :]) * s[None, :]
        self.sigma, self.rate, self.freeze, self.seed = sigma, rate, freeze, int(seed)
        self.ldx = -(-n // pad_to) * pad_to
        self.ldd = -(-m // pad_to) * pad_to
        self.device = device
        self.X = torch.zeros(B, self.ldx, device=device, dtype=torch.bfloat16)
        self.D = torch.zeros(B, self.ldd, device=device, dtype=torch.bfloat16)

    def draw(self, t):
        """Fills and returns (X, D) for step t (bf16, row strides ldx and ldd)."""
        import math
        th = self.rate * min(t, self.freeze)
        C = self.C0 * math.cos(th) + self.C1 * math.sin(th)
        g = torch.Generator(device=self.device)
        g.manual_seed(self.seed * 1000003 + t + 1)
        Z = torch.randn(self.B, self.k, generator=g, device=self.device)
        x = Z @ self.SA
        x += self.sigma * torch.randn(self.B, self.n, generator=g, device=self.device)
        self.X[:, : self.n] = x.to(torch.bfloat16)
        d = (Z @ self.SM) @ C
        d += self.sigma * torch.randn(self.B, self.m, generator=g, device=self.device)
        self.D[:, : self.m] = (d / self.B).to(torch.bfloat16)
        return self.X, self.D
