"""Seeded synthetic inputs for the ParisKV retrieval path.

This module is the only code shared by the tests, the benchmark and the
oracle checks: it draws inputs and holds none of the method's arithmetic.
Every tensor is drawn from a ``torch.Generator`` seeded per (config seed,
sequence x KV-head), on the device the caller asks for, so a given device and
seed always give the same inputs.

The pages measure on LongBench-v2, AIME25, GPQA-Diamond, MATH500 and RULER
with Llama3.1-8B / Qwen3 weights; none of those are available here, so these
generators stand in for them with the workload shapes the pages use (contexts
32K-1M, head_dim 128, 8 KV heads / 32 query heads, Top-100).

Readings (the configs leave these open):
  * outlier channels of the tiny config are channels 0-3;
  * "N(0,0.5)" query noise means standard deviation 0.5;
  * Llama-shaped keys: K_c = N(0,1) * sigma_c, sigma_c ~ LogNormal(0, 0.5) per
    (sequence, KV head, channel); RoPE rotate-half layout, theta = 500000, no
    long-context scaling, positions 0..n-1; V = N(0,1) * sigma'_c, no RoPE;
  * Llama-shaped queries: q_{h,g} = K_h[j] + 0.5 * sigma_h (.) N(0,1), j uniform;
  * drift stream: K ~ N(mu_t, diag sigma^2), mu_1 = mu_0 + 2 * RMS(sigma) * d
    with d a random unit vector, mu_t moving linearly from mu_0 to mu_1.
"""
from __future__ import annotations

import math

import torch

ROPE_THETA = 500000.0


def _gen(device, seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + int(stream) * 7919 + 17) % (2**63 - 1))
    return g


def rope_rotate_half(x: torch.Tensor, pos0: int = 0, theta: float = ROPE_THETA) -> torch.Tensor:
    """Apply rotate-half RoPE to x[n][D] at positions pos0..pos0+n-1."""
    n, D = x.shape
    half = D // 2
    inv = theta ** (-torch.arange(half, device=x.device, dtype=torch.float64) * 2.0 / D)
    pos = torch.arange(pos0, pos0 + n, device=x.device, dtype=torch.float64)
    ang = pos[:, None] * inv[None, :]
    cos = torch.cos(ang).to(torch.float32)
    sin = torch.sin(ang).to(torch.float32)
    x1, x2 = x[:, :half], x[:, half:]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=1)


# --------------------------------------------------------------------------
def tiny(seed: int = 0, device="cpu", n: int = 4096, D: int = 128, n_queries: int = 16,
         outliers: int = 4, outlier_scale: float = 8.0, noise: float = 0.5):
    """Tiny single-head retrieval: 1 KV head, fp32 K/V ~ N(0,1), K channels
    0..outliers-1 scaled by outlier_scale; queries q = K[j] + noise*N(0,1).

    Returns K, V [1][1][n][D] fp32 and q [n_queries][1][1][D] fp32."""
    g = _gen(device, seed, 0)
    K = torch.randn(n, D, generator=g, device=device)
    K[:, :outliers] *= outlier_scale
    V = torch.randn(n, D, generator=g, device=device)
    j = torch.randint(0, n, (n_queries,), generator=g, device=device)
    q = K[j] + noise * torch.randn(n_queries, D, generator=g, device=device)
    return dict(K=K.view(1, 1, n, D).contiguous(), V=V.view(1, 1, n, D).contiguous(),
                q=q.view(n_queries, 1, 1, D).contiguous(), qsrc=j)


def llama_pair(b: int, h: int, n: int, H: int = 8, G: int = 4, D: int = 128, seed: int = 0,
               device="cpu", n_queries: int = 1, dtype=torch.bfloat16, noise: float = 0.5,
               rope: bool = True):
    """One (sequence b, KV head h) pair of the Llama-shaped layer: K, V [n][D]
    and its G query heads q [n_queries][G][D].  Drawn from the pair's own
    generator, so any pair can be regenerated alone."""
    g = _gen(device, seed, b * H + h)
    sig = torch.exp(0.5 * torch.randn(D, generator=g, device=device))
    sigv = torch.exp(0.5 * torch.randn(D, generator=g, device=device))
    k = torch.randn(n, D, generator=g, device=device) * sig
    if rope:
        k = rope_rotate_half(k)
    K = k.to(dtype)
    del k
    V = (torch.randn(n, D, generator=g, device=device) * sigv).to(dtype)
    j = torch.randint(0, n, (n_queries, G), generator=g, device=device)
    kq = K.float()[j.reshape(-1)].reshape(n_queries, G, D)
    q = (kq + noise * sig * torch.randn(n_queries, G, D, generator=g, device=device)).to(dtype)
    return K, V, q


def llama_layer(batch: int, n: int, H: int = 8, G: int = 4, D: int = 128, seed: int = 0,
                device="cpu", n_queries: int = 1, dtype=torch.bfloat16, noise: float = 0.5,
                rope: bool = True):
    """Llama3.1-8B-shaped decode layer with per-channel LogNormal(0,0.5) scales
    and RoPE on the keys.

    Returns K, V [batch][H][n][D] (dtype) and q [n_queries][batch][H*G][D]."""
    K = torch.empty(batch, H, n, D, dtype=dtype, device=device)
    V = torch.empty(batch, H, n, D, dtype=dtype, device=device)
    q = torch.empty(n_queries, batch, H * G, D, dtype=dtype, device=device)
    for b in range(batch):
        for h in range(H):
            k_, v_, q_ = llama_pair(b, h, n, H=H, G=G, D=D, seed=seed, device=device,
                                    n_queries=n_queries, dtype=dtype, noise=noise, rope=rope)
            K[b, h] = k_
            V[b, h] = v_
            q[:, b, h * G:(h + 1) * G] = q_
            del k_, v_, q_
    return dict(K=K, V=V, q=q)


def drift_stream(n_prefill: int, n_steps: int, H: int = 8, D: int = 128, seed: int = 0,
                 device="cpu", dtype=torch.bfloat16, shift_sigmas: float = 2.0):
    """Drift stream: prefill keys ~ N(mu_0, diag sigma^2); decode step t
    (t = 1..n_steps) draws one key/value and one query per KV head from
    N(mu_0 + (t/n_steps)(mu_1 - mu_0), diag sigma^2).

    Returns K0, V0 [1][H][n_prefill][D]; k_new, v_new [n_steps][1][H][1][D];
    q [n_steps][1][H][D] (G = 1)."""
    g = _gen(device, seed, 0)
    sig = torch.exp(0.5 * torch.randn(H, 1, D, generator=g, device=device))
    mu0 = torch.randn(H, 1, D, generator=g, device=device)
    d = torch.randn(H, 1, D, generator=g, device=device)
    d = d / d.norm(dim=-1, keepdim=True)
    rms = sig.pow(2).mean(dim=-1, keepdim=True).sqrt()
    mu1 = mu0 + shift_sigmas * rms * d
    K0 = mu0 + sig * torch.randn(H, n_prefill, D, generator=g, device=device)
    V0 = torch.randn(H, n_prefill, D, generator=g, device=device)
    t = torch.arange(1, n_steps + 1, device=device, dtype=torch.float32) / float(n_steps)
    mut = mu0[None] + t[:, None, None, None] * (mu1 - mu0)[None]        # [T][H][1][D]
    kn = mut + sig[None] * torch.randn(n_steps, H, 1, D, generator=g, device=device)
    vn = torch.randn(n_steps, H, 1, D, generator=g, device=device)
    qn = mut[:, :, 0] + sig[None, :, 0] * torch.randn(n_steps, H, D, generator=g, device=device)
    return dict(K=K0.unsqueeze(0).to(dtype).contiguous(), V=V0.unsqueeze(0).to(dtype).contiguous(),
                k_new=kn.unsqueeze(1).to(dtype).contiguous(),
                v_new=vn.unsqueeze(1).to(dtype).contiguous(),
                q=qn.unsqueeze(1).to(dtype).contiguous())


def to_np_f32(t: torch.Tensor):
    """Exact fp32 copy on the host (bf16 widens exactly)."""
    return t.detach().to("cpu", torch.float32).contiguous().numpy()


def default_scale(D: int = 128) -> float:
    return 1.0 / math.sqrt(D)
