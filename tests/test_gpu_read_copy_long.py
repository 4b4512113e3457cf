"""Read-copy output error at the serving shapes, against the fp64 oracle, with
a stated bound, over 2048 decode steps for L in {1, 4, 8, 16, 32}.

"ReplaySSM: Rethinking State Storage for Faster Hybrid-Model Decoding"
(deskofai.com summary, paragraph 4): the recurrence stays in high precision
while a low-precision copy serves the reads, so the copy's rounding does not
compound over the decode.  Layers: Mamba-2 (batch 256, 128 heads, P 64,
N 128, G 8) and Gated DeltaNet (batch 256, 32 heads, d 128), bf16 inputs, fp32
checkpoint, FP8 E4M3 row copy and NVFP4 copy.  Four sequences spread over the
batch are compared every step with the oracle (worker processes); tokens cycle
through 64 seeded steps.

The bound.  Between folds a read-copy layer computes exactly the recurrence
started from the copy C = deq(copy) instead of the fp32 checkpoint S_c (its
replay form is that recurrence unrolled), so with dS = C - S_c, taken from
the GPU's own checkpoint and read copy (its codes equal the oracle's encoders
bit for bit, which the code tests pin; they are decoded here with the
oracle's code tables):
  * Mamba-2: the output is affine in the checkpoint with coefficient
    e^{G_t} C_t, so |dy_t[p]| <= e^{G_t} sum_n |dS[p, n]| |C_t[n]|;
  * gated delta rule: a row r of the state evolves as r <- alpha r (I - beta k k^T)
    and ||I - beta k k^T||_2 = 1 for 0 <= beta ||k||^2 <= 2, so
    |do_t[i]| <= out_scale e^{G_t} ||dS[i, :]||_2 ||q_t||_2,
with G_t the log-decay summed over the window entries since the last fold.
Every output element must satisfy it, plus 1e-4 (|o| + rms(o)) for the fp32
arithmetic and checkpoint.  Also: the fp32 checkpoint tracks the fp64 state
(2e-3, after every 32nd token) and the error of the last 256 steps is no larger than twice that of
the first 256 (no compounding).  The bound's arithmetic runs in fp64 on the
device (torch), the exact outputs in the oracle.  `pytest -s` prints the
per-case errors.
"""
import numpy as np
import pytest
import torch

import seeded_inputs as si
from gpu_common import DEV, GDN_KEYS, M2_KEYS, dev_inputs, gdn_layer, m2_layer
from hybrid_ssm_decode_replayssm_b200 import rssm
from oracle import codecs as oc
from oracle import mamba2 as om
from oracle_workers import OracleWorkers

pytestmark = pytest.mark.gpu

STEPS = 2048
EDGE = 256
POOL = 64
ROWS = [5, 70, 141, 250]
SLACK = 1e-4
FMT_NAME = {rssm.RSSM_READ_FP8_E4M3_ROW: "fp8_e4m3_row", rssm.RSSM_READ_NVFP4: "nvfp4"}


def _copy_error(layer, fmt, rows):
    """deq(read copy) - checkpoint for the sequences `rows`, fp64 on the device."""
    codes, scales = layer.read_copy_views()
    codes, scales = codes[rows].long(), scales[rows]
    e4m3 = torch.tensor(oc.E4M3_VALUES, dtype=torch.float64, device=DEV)
    e4m3 = torch.cat([e4m3, torch.tensor([float("nan")], dtype=torch.float64, device=DEV)])
    signed8 = torch.cat([e4m3, -e4m3])                                  # code -> value, 256 entries
    if fmt == rssm.RSSM_READ_FP8_E4M3_ROW:
        deq = signed8[codes] * scales.double()[..., None]
    else:
        e2m1 = torch.tensor(oc.E2M1_VALUES, dtype=torch.float64, device=DEV)
        signed4 = torch.cat([e2m1, -e2m1])
        q = torch.stack([codes & 0xF, codes >> 4], dim=-1).flatten(-2)  # element 2i in the low nibble
        blk = signed4[q].unflatten(-1, (-1, 16)) * signed8[scales.long()][..., None]
        deq = blk.flatten(-2)
    return deq - layer.ckpt[rows].double()


def _run(kind, fmt, L):
    if kind == "mamba2":
        shape = si.MAMBA2_SERVING.with_(window=L, max_draft=1)
        layer, A, D, h0 = m2_layer(shape, read_fmt=fmt)
        keys, params = M2_KEYS, {"A": A, "D": D}
        toks = [si.mamba2_tokens(shape, t, seed=3) for t in range(POOL)]
        groups = om.head_groups(shape.nheads, shape.ngroups)
        out = torch.empty(256, 128, 64, device=DEV)
    else:
        shape = si.GDN_SERVING.with_(window=L, max_draft=1)
        layer, h0 = gdn_layer(shape, read_fmt=fmt)
        keys, params = GDN_KEYS, None
        toks = [si.gdn_tokens(shape, t, seed=3) for t in range(POOL)]
        out = torch.empty(256, 32, 128, device=DEV)
    dev_toks = [dev_inputs(t, keys) for t in toks]
    np_toks = [{k: v[ROWS].float().numpy() for k, v in t.items()} for t in toks]
    workers = OracleWorkers(kind, h0[ROWS].numpy(), nblocks=len(ROWS), params=params)
    dS = _copy_error(layer, fmt, ROWS)                           # [rows, H, R, C]
    adS, dS_norm = dS.abs(), dS.square().sum(-1).sqrt()
    G = torch.zeros((len(ROWS), shape.nheads), dtype=torch.float64, device=DEV)   # log-decay since the fold
    if kind == "mamba2":
        A_dev = torch.tensor(A, device=DEV)
        groups_dev = torch.tensor(groups, device=DEV)
    try:
        for t in range(STEPS):
            tk, dt_ = np_toks[t % POOL], dev_toks[t % POOL]
            layer.decode_step(dt_, out)
            if kind == "mamba2":
                G += dt_[3][ROWS].double() * A_dev[None, :]
                Ct = dt_[2][ROWS].double().abs()[:, groups_dev, :]                  # [rows, H, N]
                bound = torch.exp(G)[..., None] * torch.matmul(adS, Ct[..., None])[..., 0]
            else:
                G += torch.log(dt_[3][ROWS].double())
                qn = dt_[0][ROWS].double().square().sum(-1).sqrt()                  # [rows, H]
                bound = (torch.exp(G) * qn)[..., None] * dS_norm
            folded = (t + 1) % L == 0
            ck = layer.ckpt[ROWS].cpu().numpy() if (t + 1) % 32 == 0 else None   # after every 32nd token (a fold)
            workers.decode_bound(f"step {t}", tk, out[ROWS].cpu().numpy(), bound.cpu().numpy(), SLACK, ck, 2e-3)
            if folded:   # the window was folded after this output: a new checkpoint and copy
                dS = _copy_error(layer, fmt, ROWS)
                adS, dS_norm = dS.abs(), dS.square().sum(-1).sqrt()
                G.zero_()
        assert layer.get_status() == 0
    finally:
        worst, failures = workers.finish()
    series = np.array(workers.series)                 # [rows, steps, (max, mean square)]
    emax = series[:, :, 0].max(axis=0)
    erms = np.sqrt(series[:, :, 1].mean(axis=0))
    return worst, failures, emax, erms


@pytest.mark.parametrize("L", [1, 4, 8, 16, 32])
@pytest.mark.parametrize("fmt", [rssm.RSSM_READ_FP8_E4M3_ROW, rssm.RSSM_READ_NVFP4])
@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
def test_read_copy_error_bounded_and_not_compounding(kind, fmt, L):
    worst, failures, emax, erms = _run(kind, fmt, L)
    first, last = emax[:EDGE].max(), emax[-EDGE:].max()
    print(f"\n{kind} {FMT_NAME[fmt]} L={L}: per-step max |err|/rms(o) first {EDGE} {first:.3e}, "
          f"last {EDGE} {last:.3e}; rms over {STEPS} steps {np.sqrt(np.mean(erms ** 2)):.3e}; "
          f"worst error / bound {worst.get('bound ratio', 0):.3f}; "
          f"fp32 checkpoint vs fp64 {worst.get('checkpoint', 0):.2e}")
    assert not failures, failures
    assert worst["checkpoint"] < 2e-3
    assert last <= 2.0 * first, f"error grew: first {first:.3e}, last {last:.3e}"
    assert np.sqrt(np.mean(erms[-EDGE:] ** 2)) <= 1.5 * np.sqrt(np.mean(erms[:EDGE] ** 2)) + 1e-6
