"""Seeded synthetic workloads for the ReplaySSM decode path.

This module is shared by the fp64 oracle and by the CUDA path (tests, bench,
smoke).  It draws token inputs, layer parameters, initial checkpoints and
speculative acceptance counts, and it holds none of the method's arithmetic.

Every tensor is drawn from its own torch CPU generator, keyed by
(seed, tensor name, step), so any step of any workload can be regenerated on
its own without replaying the ones before it.

Recipes (the distributions of the layers the pages evaluate, synthetic and
seeded; no trained weights and no dataset are used):

* Mamba-2: x, B, C ~ N(0, 1); dt = softplus(N(-1, 0.5)) per (batch, head);
  A = -exp(U(ln 1, ln 16)) and D ~ N(0, 1) per head; checkpoint h ~ N(0, std)
  with std 0.1 (or zeros).  Token tensors are rounded to the layer's input
  dtype (fp32 or bf16); A, D and the checkpoint are fp32.
* Gated DeltaNet: q, k ~ N(0, 1) L2-normalised in fp32 and then rounded to the
  input dtype; v ~ N(0, 1); alpha = exp(-0.1 * softplus(N(0, 1))) and
  beta = sigmoid(N(0, 1)) in fp32; checkpoint S ~ N(0, 0.05) in fp32.
* Speculative rounds: k drafts drawn from the same token recipe, and an
  accepted-prefix length a ~ U{0..k} per sequence and round.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, replace

import torch
import torch.nn.functional as F

__all__ = [
    "Mamba2Layer", "GDNLayer", "MAMBA2_TINY_F32", "MAMBA2_SERVING",
    "GDN_SERVING", "mamba2_params", "mamba2_checkpoint", "mamba2_tokens",
    "mamba2_drafts", "gdn_checkpoint", "gdn_tokens", "gdn_drafts",
    "accept_counts", "torch_dtype", "kda_checkpoint", "kda_tokens", "kda_drafts",
]


def _generator(seed: int, *key) -> torch.Generator:
    digest = hashlib.blake2b(repr((int(seed),) + tuple(key)).encode(),
                             digest_size=8).digest()
    return torch.Generator().manual_seed(
        int.from_bytes(digest, "little") & ((1 << 63) - 1))


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


@dataclass(frozen=True)
class Mamba2Layer:
    """Shape of one Mamba-2 SSM layer at decode time."""
    batch: int
    nheads: int
    headdim: int      # P
    dstate: int       # N
    ngroups: int      # G; head h reads group h // (nheads // ngroups)
    window: int = 16  # L
    dtype: str = "bf16"
    state_std: float = 0.1
    max_draft: int = 4

    def with_(self, **kw) -> "Mamba2Layer":
        return replace(self, **kw)


@dataclass(frozen=True)
class GDNLayer:
    """Shape of one Gated DeltaNet layer at decode time."""
    batch: int
    nheads: int
    dk: int
    dv: int
    window: int = 16
    dtype: str = "bf16"
    state_std: float = 0.05
    max_draft: int = 4

    def with_(self, **kw) -> "GDNLayer":
        return replace(self, **kw)


@dataclass(frozen=True)
class KDALayer:
    """Shape of one Kimi Delta Attention layer at decode time (per-channel gates)."""
    batch: int
    nheads: int
    dk: int
    dv: int
    window: int = 16
    dtype: str = "bf16"
    state_std: float = 0.05

    def with_(self, **kw) -> "KDALayer":
        return replace(self, **kw)


# Mamba-2, fp32 throughout, 64 steps from a zero checkpoint (parity workload).
MAMBA2_TINY_F32 = Mamba2Layer(batch=4, nheads=8, headdim=64, dstate=64,
                              ngroups=1, window=16, dtype="f32", state_std=0.0)
# Mamba-2 decode layer at serving batch 256 (1 GiB fp32 checkpoint).
MAMBA2_SERVING = Mamba2Layer(batch=256, nheads=128, headdim=64, dstate=128,
                             ngroups=8, window=16, dtype="bf16", state_std=0.1)
# Gated DeltaNet decode layer at serving batch 256 (512 MiB fp32 checkpoint).
GDN_SERVING = GDNLayer(batch=256, nheads=32, dk=128, dv=128, window=16,
                       dtype="bf16", state_std=0.05)
# KDA decode layer of the same shape as the GDN one.
KDA_SERVING = KDALayer(batch=256, nheads=32, dk=128, dv=128, window=16,
                       dtype="bf16", state_std=0.05)


# ----------------------------------------------------------------- Mamba-2
def mamba2_params(layer: Mamba2Layer, seed: int = 0):
    """A[H] = -exp(U(ln 1, ln 16)), D[H] ~ N(0, 1), both fp32."""
    g = _generator(seed, "m2.A")
    u = torch.rand(layer.nheads, generator=g, dtype=torch.float64)
    A = (-torch.exp(u * torch.log(torch.tensor(16.0, dtype=torch.float64)))).float()
    D = torch.randn(layer.nheads, generator=_generator(seed, "m2.D"))
    return A, D


def mamba2_checkpoint(layer: Mamba2Layer, seed: int = 0, rows=None) -> torch.Tensor:
    """Initial fp32 checkpoint [B, H, P, N] ~ N(0, state_std) (zeros if std 0).

    ``rows`` selects batch rows of the full tensor (the full tensor is drawn).
    """
    shape = (layer.batch, layer.nheads, layer.headdim, layer.dstate)
    if layer.state_std == 0.0:
        h = torch.zeros(shape)
    else:
        h = torch.randn(shape, generator=_generator(seed, "m2.h0")) * layer.state_std
    return h if rows is None else h[rows].contiguous()


def _m2_draw(layer: Mamba2Layer, gen_key, lead):
    B, H, P, N, G = (layer.batch, layer.nheads, layer.headdim, layer.dstate,
                     layer.ngroups)
    dt_ = torch_dtype(layer.dtype)
    x = torch.randn((B,) + lead + (H, P), generator=_generator(*gen_key, "x"))
    Bm = torch.randn((B,) + lead + (G, N), generator=_generator(*gen_key, "B"))
    C = torch.randn((B,) + lead + (G, N), generator=_generator(*gen_key, "C"))
    z = torch.randn((B,) + lead + (H,), generator=_generator(*gen_key, "dt"))
    dt = F.softplus(-1.0 + 0.5 * z)
    return {"x": x.to(dt_), "B": Bm.to(dt_), "C": C.to(dt_), "dt": dt.to(dt_)}


def mamba2_tokens(layer: Mamba2Layer, step: int, seed: int = 0):
    """One decode token per sequence: x[B,H,P], B[B,G,N], C[B,G,N], dt[B,H]."""
    return _m2_draw(layer, (seed, "m2.tok", int(step)), ())


def mamba2_drafts(layer: Mamba2Layer, rnd: int, k: int, seed: int = 0):
    """k draft tokens per sequence: x[B,k,H,P], B/C[B,k,G,N], dt[B,k,H]."""
    return _m2_draw(layer, (seed, "m2.draft", int(rnd), int(k)), (k,))


# ---------------------------------------------------------- Gated DeltaNet
def gdn_checkpoint(layer: GDNLayer, seed: int = 0, rows=None) -> torch.Tensor:
    """Initial fp32 checkpoint S[B, H, dv, dk] ~ N(0, state_std)."""
    shape = (layer.batch, layer.nheads, layer.dv, layer.dk)
    if layer.state_std == 0.0:
        S = torch.zeros(shape)
    else:
        S = torch.randn(shape, generator=_generator(seed, "gdn.S0")) * layer.state_std
    return S if rows is None else S[rows].contiguous()


def _gdn_draw(layer: GDNLayer, gen_key, lead):
    B, H, dk, dv = layer.batch, layer.nheads, layer.dk, layer.dv
    dt_ = torch_dtype(layer.dtype)
    q = torch.randn((B,) + lead + (H, dk), generator=_generator(*gen_key, "q"))
    k = torch.randn((B,) + lead + (H, dk), generator=_generator(*gen_key, "k"))
    q = q / torch.linalg.vector_norm(q, dim=-1, keepdim=True)
    k = k / torch.linalg.vector_norm(k, dim=-1, keepdim=True)
    v = torch.randn((B,) + lead + (H, dv), generator=_generator(*gen_key, "v"))
    za = torch.randn((B,) + lead + (H,), generator=_generator(*gen_key, "alpha"))
    zb = torch.randn((B,) + lead + (H,), generator=_generator(*gen_key, "beta"))
    alpha = torch.exp(-0.1 * F.softplus(za))
    beta = torch.sigmoid(zb)
    return {"q": q.to(dt_), "k": k.to(dt_), "v": v.to(dt_),
            "alpha": alpha.float(), "beta": beta.float()}


def gdn_tokens(layer: GDNLayer, step: int, seed: int = 0):
    """One decode token: q,k[B,H,dk], v[B,H,dv] (input dtype), alpha,beta[B,H] fp32."""
    return _gdn_draw(layer, (seed, "gdn.tok", int(step)), ())


def gdn_drafts(layer: GDNLayer, rnd: int, k: int, seed: int = 0):
    """k draft tokens: q,k[B,k,H,dk], v[B,k,H,dv], alpha,beta[B,k,H]."""
    return _gdn_draw(layer, (seed, "gdn.draft", int(rnd), int(k)), (k,))


# -------------------------------------------------------------- speculation
def accept_counts(batch: int, rnd: int, k: int, seed: int = 0) -> torch.Tensor:
    """Accepted draft-prefix length per sequence, uniform on {0, ..., k}, int32."""
    return torch.randint(0, k + 1, (batch,), generator=_generator(seed, "accept", int(rnd), int(k)),
                         dtype=torch.int32)


# ------------------------------------------------------------------- KDA
def kda_checkpoint(layer: KDALayer, seed: int = 0) -> torch.Tensor:
    """Initial fp32 checkpoint S[B, H, dv, dk] ~ N(0, state_std)."""
    shape = (layer.batch, layer.nheads, layer.dv, layer.dk)
    if layer.state_std == 0.0:
        return torch.zeros(shape)
    return torch.randn(shape, generator=_generator(seed, "kda.S0")) * layer.state_std


def _kda_draw(layer: KDALayer, key, extra):
    """q,k[B,*extra,H,dk], v[B,*extra,H,dv] (input dtype), alpha[B,*extra,H,dk] fp32
    (one gate per key channel, the GDN recipe drawn per channel), beta[B,*extra,H] fp32."""
    B, H, dk, dv = layer.batch, layer.nheads, layer.dk, layer.dv
    dt_ = torch_dtype(layer.dtype)
    q = torch.randn((B, *extra, H, dk), generator=_generator(*key, "q"))
    k = torch.randn((B, *extra, H, dk), generator=_generator(*key, "k"))
    q = q / torch.linalg.vector_norm(q, dim=-1, keepdim=True)
    k = k / torch.linalg.vector_norm(k, dim=-1, keepdim=True)
    v = torch.randn((B, *extra, H, dv), generator=_generator(*key, "v"))
    za = torch.randn((B, *extra, H, dk), generator=_generator(*key, "alpha"))
    zb = torch.randn((B, *extra, H), generator=_generator(*key, "beta"))
    return {"q": q.to(dt_), "k": k.to(dt_), "v": v.to(dt_),
            "alpha": torch.exp(-0.1 * F.softplus(za)).float(), "beta": torch.sigmoid(zb).float()}


def kda_tokens(layer: KDALayer, step: int, seed: int = 0):
    """One decode token: q,k[B,H,dk], v[B,H,dv] (input dtype), alpha[B,H,dk] fp32 (one
    gate per key channel, the GDN recipe drawn per channel), beta[B,H] fp32."""
    return _kda_draw(layer, (seed, "kda.tok", int(step)), ())


def kda_drafts(layer: KDALayer, rnd: int, k: int, seed: int = 0):
    """k draft tokens: q,k[B,k,H,dk], v[B,k,H,dv], alpha[B,k,H,dk], beta[B,k,H]."""
    return _kda_draw(layer, (seed, "kda.draft", int(rnd), int(k)), (k,))


# ------------------------------------------------------------------ branching
def branch_parents(batch: int, step: int, seed: int = 0, keep: float = 0.5) -> torch.Tensor:
    """A beam-search-like parent map, int32 [batch]: each row keeps its own history
    with probability ``keep``, else continues from a uniformly drawn row."""
    g = _generator(seed, "branch", int(step))
    own = torch.rand(batch, generator=g, dtype=torch.float64) < keep
    other = torch.randint(0, batch, (batch,), generator=g, dtype=torch.int64)
    return torch.where(own, torch.arange(batch), other).to(torch.int32)
