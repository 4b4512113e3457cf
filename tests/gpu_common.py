"""Shared helpers for the GPU parity tests (CUDA path vs the fp64 oracle)."""
import numpy as np
import torch

import seeded_inputs as si
from hybrid_ssm_decode_replayssm_b200 import rssm

DEV = "cuda:0"
M2_KEYS = ("x", "B", "C", "dt")
GDN_KEYS = ("q", "k", "v", "alpha", "beta")


def to64(t) -> np.ndarray:
    """Exact widening of the values the GPU sees (bf16/fp32) to fp64."""
    return t.detach().to("cpu", torch.float64).numpy()


def tok64(tok):
    return {k: to64(v) for k, v in tok.items()}


def dev_inputs(tok, keys):
    return [tok[k].to(DEV).contiguous() for k in keys]


def rel_err(got, want):
    """Elementwise |g - o| / (|o| + rms(o)); the parity tolerance is a bound on its max."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    rms = np.sqrt(np.mean(want ** 2)) if want.size else 0.0
    return float(np.max(np.abs(got - want) / (np.abs(want) + rms + 1e-300))) if want.size else 0.0


def assert_close(got, want, tol, what=""):
    e = rel_err(got, want)
    assert e <= tol, f"{what}: max scaled error {e:.3e} > {tol:.1e}"
    return e


def _ckpt(h0, branching):
    """The device checkpoint: h0 itself, or for a branching layer 2B slots whose
    first B hold h0."""
    if not branching:
        return h0.to(DEV).contiguous()
    c = torch.zeros((2 * h0.shape[0],) + tuple(h0.shape[1:]), dtype=torch.float32, device=DEV)
    c[: h0.shape[0]] = h0.to(DEV)
    return c


def m2_layer(shape: si.Mamba2Layer, read_fmt=rssm.RSSM_READ_FP32, auto_flush=True, seed=0, max_draft=None,
             branching=False):
    A, D = si.mamba2_params(shape, seed)
    h0 = si.mamba2_checkpoint(shape, seed)
    desc = rssm.make_desc(rssm.RSSM_MAMBA2, shape.batch, shape.nheads, shape.headdim, shape.dstate,
                          ngroups=shape.ngroups, window=shape.window,
                          max_draft=shape.max_draft if max_draft is None else max_draft,
                          in_dtype=rssm.RSSM_BF16 if shape.dtype == "bf16" else rssm.RSSM_F32,
                          read_fmt=read_fmt, auto_flush=auto_flush, branching=branching)
    layer = rssm.ReplayLayer(desc, _ckpt(h0, branching), A.to(DEV), D.to(DEV))
    return layer, A.double().numpy(), D.double().numpy(), h0


def gdn_layer(shape: si.GDNLayer, read_fmt=rssm.RSSM_READ_FP32, auto_flush=True, seed=0, out_scale=1.0,
              max_draft=None, branching=False):
    S0 = si.gdn_checkpoint(shape, seed)
    desc = rssm.make_desc(rssm.RSSM_GDN, shape.batch, shape.nheads, shape.dv, shape.dk,
                          window=shape.window,
                          max_draft=shape.max_draft if max_draft is None else max_draft,
                          in_dtype=rssm.RSSM_BF16 if shape.dtype == "bf16" else rssm.RSSM_F32,
                          read_fmt=read_fmt, auto_flush=auto_flush, out_scale=out_scale,
                          branching=branching)
    layer = rssm.ReplayLayer(desc, _ckpt(S0, branching))
    return layer, S0


KDA_KEYS = ("q", "k", "v", "alpha", "beta")


def kda_layer(shape, auto_flush=True, seed=0, out_scale=1.0, branching=False, max_draft=0,
              read_fmt=rssm.RSSM_READ_FP32):
    S0 = si.kda_checkpoint(shape, seed)
    desc = rssm.make_desc(rssm.RSSM_KDA, shape.batch, shape.nheads, shape.dv, shape.dk, window=shape.window,
                          max_draft=max_draft, in_dtype=rssm.RSSM_BF16 if shape.dtype == "bf16" else rssm.RSSM_F32,
                          auto_flush=auto_flush, out_scale=out_scale, branching=branching, read_fmt=read_fmt)
    layer = rssm.ReplayLayer(desc, _ckpt(S0, branching))
    return layer, S0
