"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and bench.py.

This module draws random numbers and builds tensors of the shapes the workloads
use.  It holds none of the method's arithmetic: no projection, reconstruction,
score, softmax or mixing.  The one linear-algebra step here is the QR
factorisation that turns a Gaussian matrix into an orthonormal basis, which is
how the pages obtain the bases themselves (StiefAttention technical summary,
"Mecanismo Central" item 3, "Ortonormalizacao"/"Orthonormalisierung": A = QR and
Q is the basis); the bases are inputs to the decode path.

Recipe (per (layer, sequence, KV head), all seeded):
  * keys and values: bf16(Z . W + 0.1 . N),  Z ~ N(0,1) of shape L x 32,
    W ~ N(0, 1/32) of shape 32 x dim, N ~ N(0,1) of shape L x dim, independent
    draws for K and V;
  * queries: bf16(N(0,1));
  * bases: P = Q of the QR factorisation of an N(0,1) d x r matrix, columns
    signed so diag(R) > 0, float64, then rounded to bf16 for both the GPU path
    and the oracle.
A latent cache drawn directly with dim = r has the same distribution as the
projection of full-dimension rows from the recipe, because W . P and N . P are
again i.i.d. Gaussians of the same variances when P has orthonormal columns.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple

import numpy as np
import torch

LOW_RANK = 32
NOISE = 0.1


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one decode workload (a single layer unless ``layers`` > 1)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    L: int
    rK: int
    rV: int
    layers: int = 1
    seed: int = 0
    # per-layer ranks for heterogeneous profiles (layers > 1); None = (rK, rV) everywhere
    ranks: Optional[Tuple[Tuple[int, int], ...]] = None

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def layer_ranks(self) -> List[Tuple[int, int]]:
        if self.ranks is not None:
            return list(self.ranks)
        return [(self.rK, self.rV)] * self.layers

    def latent_bytes(self) -> int:
        """Algorithmic decode bytes per step: the bf16 latent cache read once per KV head."""
        return sum(2 * (rk + rv) * self.B * self.Hkv * self.L for rk, rv in self.layer_ranks())


RANK_SET = (32, 48, 64, 96)


def heterogeneous_ranks(layers: int = 32, seed: int = 1003) -> Tuple[Tuple[int, int], ...]:
    """Per-layer (r_K, r_V) drawn from {32,48,64,96} with r_V != r_K (seeded schedule)."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(layers):
        rk = int(rng.choice(RANK_SET))
        rv = int(rng.choice([r for r in RANK_SET if r != rk]))
        out.append((rk, rv))
    return tuple(out)


WORKLOADS: Dict[str, Workload] = {
    # tiny single layer: one decode step
    "tiny": Workload("tiny", B=1, Hq=4, Hkv=1, d=128, L=1024, rK=64, rV=64, seed=1001),
    # Llama-3-8B-shaped single layer, 32k context, 50% compression
    "llama3_8b_32k": Workload("llama3_8b_32k", B=1, Hq=32, Hkv=8, d=128, L=32768,
                              rK=64, rV=64, seed=1002),
    # 32 layers, batch 16, context 8192, heterogeneous per-layer ranks
    "llama3_8b_32layer_b16": Workload("llama3_8b_32layer_b16", B=16, Hq=32, Hkv=8, d=128,
                                      L=8192, rK=64, rV=64, layers=32, seed=1003,
                                      ranks=heterogeneous_ranks(32, 1003)),
    # Llama-3.1-8B long context, aggressive compression
    "llama31_8b_128k": Workload("llama31_8b_128k", B=1, Hq=32, Hkv=8, d=128, L=131072,
                                rK=32, rV=48, seed=1004),
    # batched decode after a 4096-token prefill compress (decode part)
    "prefill_b64": Workload("prefill_b64", B=64, Hq=32, Hkv=8, d=128, L=4096,
                            rK=64, rV=64, layers=32, seed=1005),
}

# the prefill-compress part of the last workload: one 4096-token chunk per layer
PREFILL_CHUNK = dict(B=1, Hkv=8, T=4096, d=128, rK=64, rV=64, layers=32, seed=1005)


def sub_seed(base: int, *keys: int) -> int:
    """Deterministic child seed for (layer, sequence, head, ...) keys."""
    ss = np.random.SeedSequence([int(base)] + [int(k) for k in keys])
    return int(ss.generate_state(1, dtype=np.uint32)[0])


# ----------------------------------------------------------------------------- numpy (CPU)

def stiefel_basis(rng: np.random.Generator, d: int, r: int) -> np.ndarray:
    """Orthonormal d x r basis: Q of QR(N(0,1)^{d x r}) with diag(R) > 0 (float64)."""
    a = rng.standard_normal((d, r))
    q, rr = np.linalg.qr(a, mode="reduced")
    signs = np.sign(np.diag(rr))
    signs[signs == 0] = 1.0
    return q * signs[None, :]


def bases(seed: int, Hkv: int, d: int, r: int) -> np.ndarray:
    """[Hkv][d][r] float64 per-KV-head bases."""
    return np.stack([stiefel_basis(np.random.default_rng(sub_seed(seed, 7, h, r)), d, r)
                     for h in range(Hkv)])


def low_rank_rows(rng: np.random.Generator, n: int, dim: int,
                  rank: int = LOW_RANK, noise: float = NOISE) -> np.ndarray:
    """n x dim rows Z.W + noise.N (float64) with Z ~ N(0,1), W ~ N(0, 1/rank)."""
    z = rng.standard_normal((n, rank))
    w = rng.standard_normal((rank, dim)) / np.sqrt(rank)
    return z @ w + noise * rng.standard_normal((n, dim))


def to_bf16(x) -> torch.Tensor:
    """Round an array to a bf16 CPU tensor (input rounding, same values for both sides)."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32))
    return t.to(torch.bfloat16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def full_kv(seed: int, B: int, Hkv: int, T: int, d: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """Full-dimension k, v rows [B][Hkv][T][d] as bf16 CPU tensors."""
    ks, vs = [], []
    for b in range(B):
        for h in range(Hkv):
            ks.append(low_rank_rows(np.random.default_rng(sub_seed(seed, 1, b, h)), T, d))
            vs.append(low_rank_rows(np.random.default_rng(sub_seed(seed, 2, b, h)), T, d))
    k = np.stack(ks).reshape(B, Hkv, T, d)
    v = np.stack(vs).reshape(B, Hkv, T, d)
    return to_bf16(k), to_bf16(v)


def latent_cache(seed: int, B: int, Hkv: int, L_max: int, r: int, which: int) -> torch.Tensor:
    """Latent cache [B][Hkv][L_max][r] drawn directly from the low-rank-plus-noise recipe."""
    rows = [low_rank_rows(np.random.default_rng(sub_seed(seed, 3 + which, b, h, r)), L_max, r)
            for b in range(B) for h in range(Hkv)]
    return to_bf16(np.stack(rows).reshape(B, Hkv, L_max, r))


def queries(seed: int, B: int, Hq: int, d: int, scale: float = 1.0) -> torch.Tensor:
    rng = np.random.default_rng(sub_seed(seed, 5))
    return to_bf16(scale * rng.standard_normal((B, Hq, d)))


def bases_bf16(seed: int, Hkv: int, d: int, rK: int, rV: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """(P_K, P_V) as bf16 CPU tensors [Hkv][d][r]."""
    return to_bf16(bases(seed, Hkv, d, rK)), to_bf16(bases(seed + 1, Hkv, d, rV))


# ----------------------------------------------------------------------------- torch (GPU-sized)

def _torch_gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def low_rank_rows_torch(seed: int, n_mat: int, n: int, dim: int, device,
                        rank: int = LOW_RANK, noise: float = NOISE,
                        chunk: int = 8) -> torch.Tensor:
    """[n_mat][n][dim] bf16 rows from the recipe, generated on ``device`` with a seeded generator."""
    g = _torch_gen(seed, device)
    out = torch.empty((n_mat, n, dim), dtype=torch.bfloat16, device=device)
    for m0 in range(0, n_mat, chunk):
        m1 = min(n_mat, m0 + chunk)
        z = torch.randn((m1 - m0, n, rank), generator=g, device=device)
        w = torch.randn((m1 - m0, rank, dim), generator=g, device=device) / rank ** 0.5
        x = torch.bmm(z, w)
        x.add_(torch.randn(x.shape, generator=g, device=device), alpha=noise)
        out[m0:m1] = x.to(torch.bfloat16)
    return out


def latent_cache_torch(seed: int, B: int, Hkv: int, L_max: int, r: int, which: int,
                       device) -> torch.Tensor:
    """Latent cache [B][Hkv][L_max][r] (bf16) generated on ``device``."""
    x = low_rank_rows_torch(sub_seed(seed, 3 + which, r), B * Hkv, L_max, r, device)
    return x.view(B, Hkv, L_max, r)


def queries_torch(seed: int, B: int, Hq: int, d: int, device, scale: float = 1.0) -> torch.Tensor:
    g = _torch_gen(sub_seed(seed, 5), device)
    return (scale * torch.randn((B, Hq, d), generator=g, device=device)).to(torch.bfloat16)
