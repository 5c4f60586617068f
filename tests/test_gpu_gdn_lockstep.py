"""Lockstep error propagation through the delta-rule recurrence, on random
weights: a synthetic analogue of the pages' recurrence study (Paper summary
page (ai.info), "Main Findings", recurrence bullet: the state error of the
4-bit model against the full-precision one stays flat over 32K tokens, and a
one-off 1% state impulse is erased within hundreds to a few thousand steps,
much sooner than the decay alone would; fused-GEMM bullet: one common global
scale for the fused b/a gate projections corrupts the gates).

Setup (no trained weights exist here, so the gates are set up to decay slowly,
as the pages' layers do): X is the GDN prefill activation (32768 tokens, 5120
channels, 0.5% outlier channels x100); q, k, v weights N(0, 0.02); the b and a
gate weights N(0, 0.02) divided by the RMS of X (so a ~ N(0, 1)), with b's
weights also divided by 2.75 (the pages' b/a scale ratio, so that the shared
scale of the pair is b's and the decay gate is the one it distorts);
A_log ~ U(-1, 1) and dt_bias = -10 + N(0, 0.5), which puts the decay-implied
horizons at thousands of tokens.  Three projections feed the same recurrence kernel:
  * exact: FP64 products of the BF16 X and W, gates in FP64;
  * NVFP4 W4A4 with each module's own global scale (the library's fused GEMM);
  * NVFP4 W4A4 with the b/a pair sharing one scale (the serving bug).
The test prints the relative state error |S - S_exact|_F / |S_exact|_F (mean
over the 32 heads) at checkpoints, and, for a 1% impulse added to the exact
state at token 1024, the steps until its norm falls to 1/e and 1/10 next to the
decay-implied horizon (the steps until the summed log decay reaches -1).
"""
import numpy as np
import pytest
import torch

from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
from bit_quantized_linear_nvfp4_b200 import workloads as wl

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda:0"
H, DK, DV = wl.GDN_HEADS, wl.GDN_DK, wl.GDN_DV
CHECKPOINTS = (256, 1024, 4096, 8192, 16384, 32768)


def _setup(T):
    w = wl.GDN
    x = wl.make_x(w, rows=T)
    segs = wl.make_w_segments(w)
    rms = float(np.sqrt(np.mean(x.astype(np.float64) ** 2)))
    wq, wk, wv = segs[0], segs[1], segs[2]
    wb = wl.round_to_bf16((segs[4] / (2.75 * rms)).astype(np.float32))
    wa = wl.round_to_bf16((segs[5] / rms).astype(np.float32))
    a_log, dt = wl.make_gate_params(w)
    dt = (dt - 10.0).astype(np.float32)
    return x, [wq, wk, wv, wb, wa], a_log, dt


def _exact(x, ws, a_log, dt):
    xd = torch.from_numpy(x).to(DEV).double()
    outs = [xd @ torch.from_numpy(wm).to(DEV).double().T for wm in ws]
    beta = torch.sigmoid(outs[3])
    al = torch.from_numpy(a_log).to(DEV).double()
    dtb = torch.from_numpy(dt).to(DEV).double()
    g = -torch.exp(al) * torch.nn.functional.softplus(outs[4] + dtb)
    return [outs[0].float(), outs[1].float(), outs[2].float(), beta.float(), g.float()]


def _nvfp4(x, ws, a_log, dt, bug):
    T = x.shape[0]
    A, ga = nv.nvfp4_quantize(torch.from_numpy(x).to(DEV).to(torch.bfloat16))
    bounds = np.concatenate([[0], np.cumsum([wm.shape[0] for wm in ws])])
    W, gw = nv.nvfp4_quantize_segments(torch.from_numpy(np.concatenate(ws)).to(DEV).to(torch.bfloat16), bounds)
    if bug:  # b and a share the smaller (dequantisation-direction) scale of the pair
        gw = gw.clone()
        gw[3:5] = torch.minimum(gw[3], gw[4])
    q = torch.empty((T, H * DK), dtype=torch.bfloat16, device=DEV)
    k = torch.empty_like(q)
    v = torch.empty((T, H * DV), dtype=torch.bfloat16, device=DEV)
    beta = torch.empty((T, H), dtype=torch.float32, device=DEV)
    g = torch.empty_like(beta)
    b = [int(t) for t in bounds]
    nv.nvfp4_fused_proj(A, ga, W, gw, [
        nv.Segment(b[0], b[1], "identity_bf16", q), nv.Segment(b[1], b[2], "identity_bf16", k),
        nv.Segment(b[2], b[3], "identity_bf16", v), nv.Segment(b[3], b[4], "sigmoid", beta),
        nv.Segment(b[4], b[5], "gdn_decay", g, A_log=torch.from_numpy(a_log).to(DEV),
                   dt_bias=torch.from_numpy(dt).to(DEV))])
    return [q, k, v, beta, g]


def _run(inp, h0, t0, t1):
    h = torch.empty((H, DV, DK), dtype=torch.float32, device=DEV)
    nv.nvfp4_gdn_recurrence(*(t[t0:t1] for t in inp), h0, h_out=h, out_dtype=torch.float32)
    return h


def _states(inp):
    states, h, t = {}, None, 0
    for c in CHECKPOINTS:
        h = _run(inp, h, t, c)
        states[c] = h.clone()
        t = c
    return states


def _rel(a, b):
    d = (a - b).double().flatten(1).norm(dim=1)
    return (d / b.double().flatten(1).norm(dim=1)).mean().item()


def test_lockstep_state_error_and_impulse():
    T = CHECKPOINTS[-1]
    x, ws, a_log, dt = _setup(T)
    ex = _exact(x, ws, a_log, dt)
    q4 = _nvfp4(x, ws, a_log, dt, bug=False)
    bad = _nvfp4(x, ws, a_log, dt, bug=True)
    s_ex, s_q4, s_bad = _states(ex), _states(q4), _states(bad)
    torch.cuda.synchronize()
    rel = {c: _rel(s_q4[c], s_ex[c]) for c in CHECKPOINTS}
    rel_bad = {c: _rel(s_bad[c], s_ex[c]) for c in CHECKPOINTS}
    g_err = ((q4[4] - ex[4]).abs().sum() / ex[4].abs().sum()).item()
    g_err_bad = ((bad[4] - ex[4]).abs().sum() / ex[4].abs().sum()).item()
    print("\ntoken   relS (per-module scales)   relS (common b/a scale)")
    for c in CHECKPOINTS:
        print(f"{c:6d}   {rel[c]:.4f}                     {rel_bad[c]:.4f}")
    print(f"decay gate relative error: per-module {g_err:.4f}, common scale {g_err_bad:.4f}")

    # impulse: 1% of each head's state norm, in a random direction, at token 1024
    t0, span, step = 1024, 16384, 32
    base = s_ex[t0]
    rng = np.random.default_rng(5)
    d = torch.from_numpy(rng.standard_normal((H, DV, DK)).astype(np.float32)).to(DEV)
    d *= 0.01 * base.flatten(1).norm(dim=1)[:, None, None] / d.flatten(1).norm(dim=1)[:, None, None]
    a, b = base.clone(), base + d
    n0 = d.flatten(1).norm(dim=1)
    ratio = []
    for t in range(t0, t0 + span, step):
        a = _run(ex, a, t, t + step)
        b = _run(ex, b, t, t + step)
        ratio.append(((b - a).flatten(1).norm(dim=1) / n0).cpu().numpy())
    ratio = np.stack(ratio)  # [steps, H]
    ts = step * (1 + np.arange(ratio.shape[0]))
    neg_g = -ex[4][t0:t0 + span].double().cpu().numpy()
    horizon = np.array([np.searchsorted(np.cumsum(neg_g[:, h]), 1.0) + 1 for h in range(H)])

    def first_below(level):
        out = np.full(H, np.inf)
        for h in range(H):
            idx = np.nonzero(ratio[:, h] <= level)[0]
            if idx.size:
                out[h] = ts[idx[0]]
        return out
    e1, e10 = first_below(np.exp(-1.0)), first_below(0.1)
    print(f"impulse at token {t0}: steps to 1/e median {np.median(e1):.0f} (range {e1.min():.0f}-{e1.max():.0f}), "
          f"to 1/10 median {np.median(e10):.0f} (range {e10.min():.0f}-{e10.max():.0f}); "
          f"decay-implied horizon median {np.median(horizon):.0f} (range {horizon.min()}-{horizon.max()})")

    # the state error stays flat (no accumulation) and is set by the projection
    assert rel[CHECKPOINTS[-1]] <= 2.0 * rel[1024]
    assert 0.0 < rel[CHECKPOINTS[-1]] < 0.5
    # the common scale corrupts the decay gate, and the state with it
    assert g_err_bad > 2.0 * g_err and rel_bad[CHECKPOINTS[-1]] > rel[CHECKPOINTS[-1]]
    # the delta rule erases the impulse well before the decay alone would
    assert np.mean(e1 < horizon) >= 0.75
