"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only draws random numbers with fixed shapes and distributions; it
holds none of the method's arithmetic (no encode, decode, RoPE or attention).

Workloads are shaped like the pages' models: Ouro-style T=4 loops, 16 heads of
width 128 at 4k context; a Huginn-style 32-loop model with d_head=96.  K/V
trajectories across loops follow a low-rank-plus-noise model,

    x_t = mu_t + sum_{i<R} a_i u_{i,t} + sigma * eps,

with a_i ~ N(0,1) per token, mu_t ~ N(0, 0.1^2), u_{i,t} random unit vectors
fixed per (layer, head, K/V) and sigma = 0.01.  In the deep-loop case the
directions converge geometrically toward the final loop:
u_{i,t} = normalise(b_i + gamma^t w_{i,t}), gamma = 0.85.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

MODE_PER_HEAD = 0
MODE_2D = 1


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    d: int
    r_k: int
    r_v: int
    mode: int
    B: int
    n: int
    R: int
    loops: tuple          # loops t at which decode attention runs
    encode_tokens: int    # tokens encoded per step (append or prefill)
    layers: int = 1
    gamma: float | None = None
    seed: int = 0


WORKLOADS = {
    "tiny_perhead_T4_H2_d64_r8_16_n128": Workload(
        "tiny_perhead_T4_H2_d64_r8_16_n128", T=4, H=2, d=64, r_k=8, r_v=16, mode=MODE_PER_HEAD,
        B=1, n=128, R=3, loops=(0, 1, 2, 3), encode_tokens=128, seed=1000),
    "perhead_4x_T4_H16_d128_r96_160_B8_n4096": Workload(
        "perhead_4x_T4_H16_d128_r96_160_B8_n4096", T=4, H=16, d=128, r_k=96, r_v=160,
        mode=MODE_PER_HEAD, B=8, n=4096, R=6, loops=(0, 1, 2, 3), encode_tokens=8, seed=1001),
    "perhead_21x_T4_H16_d128_r16_32_B256_n4096_L24": Workload(
        "perhead_21x_T4_H16_d128_r16_32_B256_n4096_L24", T=4, H=16, d=128, r_k=16, r_v=32,
        mode=MODE_PER_HEAD, B=256, n=4096, R=6, loops=(0, 1, 2, 3), encode_tokens=256,
        layers=24, seed=1002),
    "lla2d_T4_H16_d128_r64_128_B512_n4096": Workload(
        "lla2d_T4_H16_d128_r64_128_B512_n4096", T=4, H=16, d=128, r_k=64, r_v=128, mode=MODE_2D,
        B=512, n=4096, R=6, loops=(0, 1, 2, 3), encode_tokens=512, seed=1003),
    "deeploop_32x_T32_H8_d96_r64_128_B16_n32768": Workload(
        "deeploop_32x_T32_H8_d96_r64_128_B16_n32768", T=32, H=8, d=96, r_k=64, r_v=128,
        mode=MODE_PER_HEAD, B=16, n=32768, R=8, loops=(0, 15, 31), encode_tokens=16 * 32768,
        gamma=0.85, seed=1004),
}
WORKLOAD_ORDER = list(WORKLOADS)


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def unit_rows(g: np.random.Generator, shape) -> np.ndarray:
    v = g.standard_normal(shape)
    return v / np.linalg.norm(v, axis=-1, keepdims=True)


@dataclass
class TrajectoryModel:
    """Fixed parameters of one (layer, K or V) trajectory family.

    mu: [T, H, d]; U: [R, T, H, d] unit directions; shared: whether the
    coefficients a_i are shared by all heads of a token (LLA-2D workloads).
    """

    mu: np.ndarray
    U: np.ndarray
    sigma: float
    shared: bool


def trajectory_model(g, T, H, d, R, shared=False, gamma=None, sigma=0.01, mu_std=0.1):
    mu = mu_std * g.standard_normal((T, H, d))
    if gamma is None:
        U = unit_rows(g, (R, T, H, d))
    else:
        b = unit_rows(g, (R, 1, H, d))
        w = unit_rows(g, (R, T, H, d))
        # converge toward a common final state: the perturbation decays as gamma^t
        decay = gamma ** np.arange(T, dtype=np.float64)
        U = b + decay[None, :, None, None] * w
        U = U / np.linalg.norm(U, axis=-1, keepdims=True)
    return TrajectoryModel(mu, U, sigma, shared)


def sample_trajectories(g, model: TrajectoryModel, N: int) -> np.ndarray:
    """x [N, T, H, d] float64 drawn from ``model``."""
    R, T, H, d = model.U.shape
    if model.shared:
        a = g.standard_normal((N, R, 1))
        a = np.broadcast_to(a, (N, R, H))
    else:
        a = g.standard_normal((N, R, H))
    x = np.einsum("nrh,rthd->nthd", a, model.U)
    x += model.mu[None]
    x += model.sigma * g.standard_normal((N, T, H, d))
    return x


def queries(g, B, H, d) -> np.ndarray:
    """q ~ N(0, 1) / sqrt(d) per (b, h)."""
    return g.standard_normal((B, H, d)) / np.sqrt(d)


def random_matrix(g, shape, scale=1.0) -> np.ndarray:
    return scale * g.standard_normal(shape)


def random_orthonormal(g, rows: int, cols: int) -> np.ndarray:
    """[rows, cols] with orthonormal columns (QR of a Gaussian matrix)."""
    q, r = np.linalg.qr(g.standard_normal((rows, cols)))
    return q * np.sign(np.diag(r))[None, :]


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float values already representable in bf16 -> uint16 bit patterns."""
    f = np.ascontiguousarray(np.asarray(x, np.float32))
    bits = f.view(np.uint32)
    if np.any(bits & 0xFFFF):
        raise ValueError("values are not bf16-representable")
    return (bits >> 16).astype(np.uint16)


def from_bf16_bits(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Large inputs drawn on the GPU (torch Philox), for the full-size workloads.
# ---------------------------------------------------------------------------

def latents_lowrank_torch(gen, lead_shape, r, R, sigma, device, dtype):
    """Latents drawn directly in latent space: c = a Z + sigma N(0, I_r).

    With an orthonormal codec, projecting a rank-R-plus-noise trajectory gives
    exactly this distribution (Z = fixed R x r directions, a ~ N(0, 1)).
    Returns a tensor of shape lead_shape + (r,) in ``dtype``.
    """
    import torch

    Z = torch.randn((R, r), generator=gen, device=device)
    Z = Z / Z.norm(dim=-1, keepdim=True)
    out = torch.empty((*lead_shape, r), device=device, dtype=dtype)
    flat = out.view(-1, r)
    step = 1 << 22
    for s in range(0, flat.shape[0], step):
        e = min(flat.shape[0], s + step)
        a = torch.randn((e - s, R), generator=gen, device=device)
        c = a @ Z + sigma * torch.randn((e - s, r), generator=gen, device=device)
        flat[s:e] = c.to(dtype)
    return out


def workload_codec(w: Workload, seed_offset: int = 0):
    """fp32 codec arrays for a workload: random orthonormal W_down, W_up,t = its loop rows.

    Returns a dict of float32 numpy arrays in the library's input layouts
    (per head: W_down [H, T*d, r], W_up [H, T, d, r], mu [H, T*d]; LLA-2D:
    W_down [T*H*d, r], W_up [T, H, d, r], mu [T*H*d]).
    """
    g = rng(w.seed * 7919 + seed_offset)
    T, H, d = w.T, w.H, w.d
    out = {}
    for key, r in (("k", w.r_k), ("v", w.r_v)):
        if w.mode == MODE_PER_HEAD:
            Wd = np.stack([random_orthonormal(g, T * d, r) for _ in range(H)])
            Wu = Wd.reshape(H, T, d, r)
            mu = 0.1 * g.standard_normal((H, T * d))
        else:
            Wd = random_orthonormal(g, T * H * d, r)
            Wu = Wd.reshape(T, H, d, r)
            mu = 0.1 * g.standard_normal(T * H * d)
        out["W_down_" + key] = Wd.astype(np.float32)
        out["W_up_" + key] = np.ascontiguousarray(Wu).astype(np.float32)
        out["mu_" + key] = mu.astype(np.float32)
    return out


def workload_tensors(w: Workload, device, seed_offset: int = 0, B: int | None = None,
                     n: int | None = None):
    """Device tensors of one decode step of workload ``w`` (one layer).

    Latents are drawn directly in latent space (rank-R plus noise, bf16);
    positions are 0..n-1 with the in-flight token at n; q ~ N(0,1)/sqrt(d);
    k_self, v_self ~ N(0, 0.2^2).
    """
    import torch

    B = w.B if B is None else B
    n = w.n if n is None else n
    tg = torch.Generator(device=device)
    tg.manual_seed(w.seed * 104729 + seed_offset)
    lead = (B, n, w.H) if w.mode == MODE_PER_HEAD else (B, n)
    t = {
        "c_k": latents_lowrank_torch(tg, lead, w.r_k, w.R, 0.01, device, torch.bfloat16),
        "c_v": latents_lowrank_torch(tg, lead, w.r_v, w.R, 0.01, device, torch.bfloat16),
        "positions": torch.arange(n, device=device, dtype=torch.int32).repeat(B, 1).contiguous(),
        "q_pos": torch.full((B,), n, device=device, dtype=torch.int32),
        "ctx_len": torch.full((B,), n, device=device, dtype=torch.int32),
        "q": torch.randn((B, w.H, w.d), generator=tg, device=device) / float(np.sqrt(w.d)),
        "k_self": 0.2 * torch.randn((B, w.H, w.d), generator=tg, device=device),
        "v_self": 0.2 * torch.randn((B, w.H, w.d), generator=tg, device=device),
    }
    return t


def encode_inputs(w: Workload, device, n_tok: int, seed_offset: int = 0):
    """bf16 per-loop K/V rows [n_tok, T, H, d] for encode, trajectory-shaped magnitudes."""
    import torch

    tg = torch.Generator(device=device)
    tg.manual_seed(w.seed * 15485863 + seed_offset)
    shape = (n_tok, w.T, w.H, w.d)
    xk = (0.3 * torch.randn(shape, generator=tg, device=device)).to(torch.bfloat16)
    xv = (0.3 * torch.randn(shape, generator=tg, device=device)).to(torch.bfloat16)
    return xk, xv
