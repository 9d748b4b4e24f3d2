"""Seeded synthetic inputs for the optimizer-step workloads.

This module only draws random numbers and lays them out; it holds none of the
optimizer arithmetic.  The tests hand the same arrays to the CUDA path and to the
float64 oracle, and the benchmark uses the device-side generators for the full
workloads.

Workloads (shapes read literally as rows x cols, m x n):
  muon_single   one 256x512 fp32 weight; W, G, M ~ N(0, 0.02^2) drawn in that order.
  soap_single   one 1024x1024 fp32 weight; G ~ N(0, 1e-3^2) plus a rank-16 spike
                0.05 * sum_k u_k v_k^T with u_k, v_k Gaussian vectors scaled to unit
                l2 norm; W ~ N(0, 0.02^2).
  gpt2_124m     12 x {768x2304, 768x768, 768x3072, 3072x768}; bf16 G ~ N(0, 0.02^2).
  gpt2_760m     24 x {1536x4608, 1536x1536, 1536x6144, 6144x1536}; fp32 G ~ N(0, 0.01^2).
  dense8b_moe   one 8B-style block {4096x4096, 4096x1024, 4096x1024, 4096x4096,
                4096x14336, 4096x14336, 14336x4096} plus 256 experts x
                {2048x768, 2048x768, 768x2048}; bf16 G ~ N(0, 0.01^2) * s_e with one
                log-uniform s_e in [0.1, 10] per expert (shared by its 3 matrices),
                s = 1 for the dense block.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np


@dataclass(frozen=True)
class MatSpec:
    m: int
    n: int
    g_std: float
    g_scale: float = 1.0
    name: str = ""


def bf16_round(x) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), kept as float32.

    A storage-format conversion: the result holds values exactly representable in
    bfloat16, so a later cast to torch.bfloat16 is lossless.
    """
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    bits = a.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    bits = ((bits + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return bits.view(np.float32).reshape(a.shape)


# ----------------------------------------------------------------------------
# Shape sets
# ----------------------------------------------------------------------------

def specs_muon_single() -> List[MatSpec]:
    return [MatSpec(256, 512, 0.02, name="w")]


def specs_gpt2_124m() -> List[MatSpec]:
    out = []
    for layer in range(12):
        for (m, n, nm) in ((768, 2304, "qkv"), (768, 768, "proj"), (768, 3072, "fc"), (3072, 768, "fc2")):
            out.append(MatSpec(m, n, 0.02, name=f"h{layer}.{nm}"))
    return out


def specs_gpt2_760m() -> List[MatSpec]:
    out = []
    for layer in range(24):
        for (m, n, nm) in ((1536, 4608, "qkv"), (1536, 1536, "proj"), (1536, 6144, "fc"), (6144, 1536, "fc2")):
            out.append(MatSpec(m, n, 0.01, name=f"h{layer}.{nm}"))
    return out


def expert_scales(n_experts: int, seed: int) -> np.ndarray:
    """One log-uniform scale in [0.1, 10] per expert."""
    rng = np.random.default_rng(seed)
    return np.exp(rng.uniform(np.log(0.1), np.log(10.0), size=n_experts))


def specs_dense8b_block() -> List[MatSpec]:
    shapes = ((4096, 4096, "q"), (4096, 1024, "k"), (4096, 1024, "v"), (4096, 4096, "o"),
              (4096, 14336, "gate"), (4096, 14336, "up"), (14336, 4096, "down"))
    return [MatSpec(m, n, 0.01, 1.0, name=nm) for (m, n, nm) in shapes]


def specs_moe_bank(n_experts: int = 256, seed: int = 0) -> List[MatSpec]:
    sc = expert_scales(n_experts, seed + 1000)
    out = []
    for e in range(n_experts):
        for (m, n, nm) in ((2048, 768, "gate"), (2048, 768, "up"), (768, 2048, "down")):
            out.append(MatSpec(m, n, 0.01, float(sc[e]), name=f"e{e}.{nm}"))
    return out


def specs_dense8b_moe(n_experts: int = 256, seed: int = 0) -> List[MatSpec]:
    return specs_dense8b_block() + specs_moe_bank(n_experts, seed)


WORKLOADS = {
    "muon_single": specs_muon_single,
    "gpt2_124m": specs_gpt2_124m,
    "gpt2_760m": specs_gpt2_760m,
    "dense8b_block": specs_dense8b_block,
    "moe_bank": specs_moe_bank,
    "dense8b_moe": specs_dense8b_moe,
}


# ----------------------------------------------------------------------------
# Host (NumPy) generators, for the sizes the oracle handles
# ----------------------------------------------------------------------------

def gaussian(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return (rng.standard_normal(shape) * std).astype(np.float32)


def muon_inputs(specs: Sequence[MatSpec], seed: int = 0, g_bf16: bool = False,
                w_std: float = 0.02, m_std: Optional[float] = None):
    """Per matrix: W ~ N(0, w_std^2), G ~ N(0, (g_std*g_scale)^2), M (zero, or N(0, m_std^2)).

    Draw order per matrix: W, G, M.  Returns a list of (W, G, M) float32 arrays;
    with g_bf16 the G values are bfloat16-exact.
    """
    rng = np.random.default_rng(seed)
    out = []
    for s in specs:
        W = gaussian(rng, (s.m, s.n), w_std)
        G = gaussian(rng, (s.m, s.n), s.g_std * s.g_scale)
        if g_bf16:
            G = bf16_round(G)
        M = gaussian(rng, (s.m, s.n), m_std) if m_std else np.zeros((s.m, s.n), np.float32)
        out.append((W, G, M))
    return out


def muon_single_inputs(seed: int = 0):
    """The 256x512 single-weight Muon case: W, G, M each N(0, 0.02^2), seed 0."""
    return muon_inputs(specs_muon_single(), seed, g_bf16=False, w_std=0.02, m_std=0.02)[0]


def spiked_gradient(rng: np.random.Generator, m: int, n: int, noise_std: float = 1e-3,
                    rank: int = 16, spike: float = 0.05) -> np.ndarray:
    """G = N(0, noise_std^2) + spike * sum_k u_k v_k^T, u_k, v_k unit-norm Gaussian vectors."""
    G = rng.standard_normal((m, n)) * noise_std
    U = rng.standard_normal((rank, m))
    V = rng.standard_normal((rank, n))
    U /= np.linalg.norm(U, axis=1, keepdims=True)
    V /= np.linalg.norm(V, axis=1, keepdims=True)
    G = G + spike * (U.T @ V)
    return G.astype(np.float32)


def soap_single_inputs(seed: int = 0, steps: int = 1, m: int = 1024, n: int = 1024):
    """The single-weight SOAP case: W ~ N(0, 0.02^2) then one spiked G per step.

    Step 1 uses `seed`; later steps use seeds seed+1, seed+2, ... (fresh G).
    """
    rng = np.random.default_rng(seed)
    W = gaussian(rng, (m, n), 0.02)
    Gs = [spiked_gradient(rng, m, n)]
    for s in range(1, steps):
        Gs.append(spiked_gradient(np.random.default_rng(seed + s), m, n))
    return W, Gs


def kronecker_gradients(rng: np.random.Generator, m: int, n: int, Q: np.ndarray, steps: int):
    """Gradients whose rotated square is rank one: G_s = k_s diag(sqrt a) E_s diag(sqrt b) Q^T.

    E_s is a random +-1 matrix, a in R^m and b in R^n are positive and fixed, k_s is a
    scalar per step.  Returns (list of G_s, a, b, k).
    """
    a = rng.uniform(0.5, 2.0, size=m)
    b = rng.uniform(0.5, 2.0, size=n)
    ks = rng.uniform(0.5, 1.5, size=steps)
    Gs = []
    for s in range(steps):
        E = np.where(rng.standard_normal((m, n)) >= 0, 1.0, -1.0)
        Gs.append(ks[s] * (np.sqrt(a)[:, None] * E * np.sqrt(b)[None, :]) @ Q.T)
    return Gs, a, b, ks


def drifting_spike_gradients(rng: np.random.Generator, m: int, n: int, steps: int, rank: int = 4,
                             spike: float = 0.05, noise_std: float = 1e-3, omega: float = 0.05):
    """A low-rank spike whose singular subspaces rotate slowly, plus noise, one G per step.

    Fixed orthonormal U0 (m x 2 rank) and V0 (n x 2 rank); at step t (1-based) the
    spike's k-th left vector is cos(omega t) U0[:, k] + sin(omega t) U0[:, rank + k]
    (the same for the right vectors with V0), its singular value spike * (1 + k / rank),
    and N(0, noise_std^2) noise is added.  Each direction turns by omega radians per
    step, a quarter turn in pi / (2 omega) steps: a basis computed from older
    gradients points away from the current ones.  Returns (list of float32 G_t,
    function t -> (U_t, V_t) of the spike's directions).
    """
    U0 = random_orthogonal(rng, m)[:, :2 * rank]
    V0 = random_orthogonal(rng, n)[:, :2 * rank]
    sv = spike * (1.0 + np.arange(rank) / rank)

    def dirs(t):
        c, s = np.cos(omega * t), np.sin(omega * t)
        return c * U0[:, :rank] + s * U0[:, rank:], c * V0[:, :rank] + s * V0[:, rank:]

    Gs = []
    for t in range(1, steps + 1):
        U, V = dirs(t)
        G = (U * sv[None, :]) @ V.T + rng.standard_normal((m, n)) * noise_std
        Gs.append(G.astype(np.float32))
    return Gs, dirs


def random_orthogonal(rng: np.random.Generator, n: int) -> np.ndarray:
    """Haar-like orthogonal matrix from the QR of a Gaussian matrix (sign-fixed)."""
    Z = rng.standard_normal((n, n))
    Q, R = np.linalg.qr(Z)
    return Q * np.sign(np.diag(R))[None, :]


def matrix_with_spectrum(rng: np.random.Generator, m: int, n: int, sv) -> np.ndarray:
    """m x n matrix U diag(sv) V^T with random orthonormal U, V."""
    k = len(sv)
    U = random_orthogonal(rng, m)[:, :k]
    V = random_orthogonal(rng, n)[:, :k]
    return (U * np.asarray(sv, dtype=np.float64)[None, :]) @ V.T


def symmetric_with_spectrum(rng: np.random.Generator, n: int, eig) -> np.ndarray:
    Q = random_orthogonal(rng, n)
    return (Q * np.asarray(eig, dtype=np.float64)[None, :]) @ Q.T


# ----------------------------------------------------------------------------
# Device (torch) generators, for the full-size workloads
# ----------------------------------------------------------------------------

def torch_gaussian(shape, std: float, gen, device, dtype):
    import torch
    return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std).to(dtype)


def torch_muon_inputs(specs: Sequence[MatSpec], seed: int, device, g_bf16: bool = True,
                      w_std: float = 0.02):
    """Device tensors per matrix, drawn W, G in order from one seeded CUDA generator; M = 0."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    gdt = torch.bfloat16 if g_bf16 else torch.float32
    out = []
    for s in specs:
        W = torch_gaussian((s.m, s.n), w_std, gen, device, torch.float32)
        G = torch_gaussian((s.m, s.n), s.g_std * s.g_scale, gen, device, gdt)
        M = torch.zeros((s.m, s.n), device=device, dtype=torch.float32)
        out.append((W, G, M))
    return out
