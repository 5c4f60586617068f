"""GPU parity of the chunked delta-rule recurrence with the oracle's token loop.

Tolerance, derived from the arithmetic.  The kernels round every product
operand to TF32 (nearest: relative error <= 2^-11) and accumulate and keep the
state in FP32; the triangular inverse is FP32 substitution plus 3xTF32 block
products (about FP32).  A rounded product sum_k a_k b_k is off by at most
2^-10 sum_k |a_k b_k|; between the inputs and an output sit four such
products in sequence (W and U~ through L, then M, N, R and Y, then S M and
S R^T), each amplified by at most |L| = |(I + A)^-1|, which stays below 2 for
unit keys and beta in [0, 1] on these inputs (checked on CPU for every chunk
of every case here; the largest value is 1.64).  So every output is held to
    |o_gpu - o| <= 4 * 2 * 2^-10 |S_t[i, :]|_2 |q_t|_2 = 2^-7 |S_t[i, :]|_2 |q_t|_2,
the right-hand side being the natural size of o_t[i] (|o_t[i]| <= |S_t[i,:]| |q_t|),
plus half a BF16 ulp for BF16 outputs; the final state to
|S_gpu - S| <= 2^-7 |S[i, :]|_2 per row.  The largest error / bound ratio is
printed for every case.
"""
import numpy as np
import pytest
import torch

from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
from bit_quantized_linear_nvfp4_b200 import workloads as wl
from oracle import nvfp4_oracle as o

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TAU = 2.0 ** -7
DK, DV = 64, 128


def _t(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x)).to(DEV)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _reference(q, k, v, beta, g, H, Hk, h0, scale, heads=None):
    T = v.shape[0]
    q3, k3, v3 = q.reshape(T, Hk, DK), k.reshape(T, Hk, DK), v.reshape(T, H, DV)
    if heads is not None:  # a subset of value heads with their query/key heads
        rep = H // Hk
        qk = [h // rep for h in heads]
        q3, k3, v3 = q3[:, qk], k3[:, qk], v3[:, heads]
        beta, g = beta[:, heads], g[:, heads]
        h0 = None if h0 is None else h0[heads]
    ref_o, ref_s, rn = o.gdn_recurrence(q3, k3, v3, beta, g, h0=h0, scale=None if scale == 0 else scale,
                                        row_norms=True)
    qn = np.linalg.norm(o.l2_normalise(q3) * (DK ** -0.5 if scale == 0 else scale), axis=2)
    if heads is None:
        qn = np.repeat(qn, H // Hk, axis=1)  # per value head
    return ref_o, ref_s, rn * qn[:, :, None]


def _check_out(got, ref, mag, bf16, what):
    bound = TAU * mag + 1e-30
    if bf16:
        bound = bound + 0.5 * o.bf16_ulp(np.abs(ref) + bound)
    err = np.abs(got - ref)
    ratio = float((err / bound).max()) if err.size else 0.0
    print(f"{what}: max error / bound = {ratio:.3g}, max |error| = {float(err.max()) if err.size else 0:.3g}")
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"{what}: {len(bad)} outside the bound, first {bad[:4].tolist()}"
    return ratio


def _check_state(got, ref, what):
    bound = TAU * np.linalg.norm(ref, axis=2, keepdims=True) + 1e-30
    err = np.abs(got - ref)
    print(f"{what}: state max error / bound = {float((err / bound).max()):.3g}")
    assert np.all(err <= bound)


def _run(T, H, Hk, seed, dtype="bf16", out_dtype="f32", with_h0=True, slow=False, scale=0.0):
    q, k, v, beta, g = wl.make_recurrence_inputs(T, H, Hk, seed, dtype, slow)
    rng = np.random.default_rng(seed + 1)
    h0 = (0.3 * rng.standard_normal((H, DV, DK))).astype(np.float32) if with_h0 else None
    h0_d = None if h0 is None else torch.from_numpy(h0).to(DEV)
    h_out = torch.empty((H, DV, DK), dtype=torch.float32, device=DEV)
    out = nv.nvfp4_gdn_recurrence(_t(q, dtype), _t(k, dtype), _t(v, dtype), _t(beta, "f32"), _t(g, "f32"), h0_d,
                                  scale, out_dtype=torch.bfloat16 if out_dtype == "bf16" else torch.float32,
                                  h_out=h_out)
    torch.cuda.synchronize()
    nv.nvfp4_check()
    ref_o, ref_s, mag = _reference(q, k, v, beta, g, H, Hk, h0, scale)
    got = out.to(torch.float64).cpu().numpy().reshape(T, H, DV)
    _check_out(got, ref_o, mag, out_dtype == "bf16", f"T={T} H={H}/{Hk} {dtype}->{out_dtype}")
    _check_state(h_out.cpu().numpy().astype(np.float64), ref_s, f"T={T}")
    return q, k, v, beta, g, h0, out, h_out


@pytest.mark.parametrize("T,H,Hk,dtype,out_dtype,with_h0", [
    (150, 4, 2, "f32", "f32", True),     # two chunks and a ragged tail, shared query/key heads
    (321, 2, 2, "bf16", "bf16", False),  # five chunks and one token, zero entering state
    (64, 3, 3, "f32", "bf16", True),     # exactly one chunk
    (1, 2, 1, "bf16", "f32", True),      # a single token
    (40, 8, 2, "bf16", "f32", True),     # one partial chunk, four value heads per query/key head
])
def test_recurrence_matches_oracle(T, H, Hk, dtype, out_dtype, with_h0):
    _run(T, H, Hk, seed=T + 17 * H, dtype=dtype, out_dtype=out_dtype, with_h0=with_h0)


def test_slow_decay_long_sequence():
    # alpha close to 1: the state carries information across many chunks
    _run(2000, 2, 2, seed=5, dtype="bf16", out_dtype="f32", slow=True)


def test_explicit_query_scale():
    _run(200, 2, 2, seed=6, dtype="f32", out_dtype="f32", scale=0.3)


def test_state_carries_across_calls_and_in_place_state():
    T1, T2, H = 130, 95, 2
    q, k, v, beta, g = wl.make_recurrence_inputs(T1 + T2, H, H, 7, "bf16")
    rng = np.random.default_rng(8)
    h0 = torch.from_numpy((0.3 * rng.standard_normal((H, DV, DK))).astype(np.float32)).to(DEV)
    whole_s = torch.empty_like(h0)
    whole = nv.nvfp4_gdn_recurrence(_t(q, "bf16"), _t(k, "bf16"), _t(v, "bf16"), _t(beta, "f32"), _t(g, "f32"), h0,
                                    out_dtype=torch.float32, h_out=whole_s)
    state = h0.clone()
    parts = []
    for a, b in ((0, T1), (T1, T1 + T2)):
        parts.append(nv.nvfp4_gdn_recurrence(_t(q[a:b], "bf16"), _t(k[a:b], "bf16"), _t(v[a:b], "bf16"),
                                             _t(beta[a:b], "f32"), _t(g[a:b], "f32"), state,
                                             out_dtype=torch.float32, h_out=state))  # in place
    torch.cuda.synchronize()
    ref_o, ref_s, mag = _reference(q, k, v, beta, g, H, H, h0.cpu().numpy(), 0.0)
    split = torch.cat(parts).double().cpu().numpy().reshape(-1, H, DV)
    _check_out(split, ref_o, mag, False, "two calls")
    _check_out(whole.double().cpu().numpy().reshape(-1, H, DV), ref_o, mag, False, "one call")
    _check_state(state.cpu().numpy().astype(np.float64), ref_s, "in place")
    _check_state(whole_s.cpu().numpy().astype(np.float64), ref_s, "whole")


def test_strided_inputs_and_output():
    T, H = 100, 2
    q, k, v, beta, g = wl.make_recurrence_inputs(T, H, H, 9, "bf16")
    # q, k, v as column ranges of one wide buffer (as a fused projection lays them out)
    wide = torch.zeros((T, 2 * H * DK + H * DV + 64), dtype=torch.bfloat16, device=DEV)
    wide[:, :H * DK] = _t(q, "bf16")
    wide[:, H * DK:2 * H * DK] = _t(k, "bf16")
    wide[:, 2 * H * DK:2 * H * DK + H * DV] = _t(v, "bf16")
    gates = torch.zeros((T, 4 * H), dtype=torch.float32, device=DEV)
    gates[:, :H] = _t(beta, "f32")
    gates[:, 2 * H:3 * H] = _t(g, "f32")
    out = torch.full((T, H * DV + 32), 7.0, dtype=torch.bfloat16, device=DEV)
    nv.nvfp4_gdn_recurrence(wide[:, :H * DK], wide[:, H * DK:2 * H * DK], wide[:, 2 * H * DK:2 * H * DK + H * DV],
                            gates[:, :H], gates[:, 2 * H:3 * H], out=out[:, :H * DV])
    torch.cuda.synchronize()
    ref_o, _, mag = _reference(q, k, v, beta, g, H, H, None, 0.0)
    _check_out(out[:, :H * DV].double().cpu().numpy().reshape(T, H, DV), ref_o, mag, True, "strided")
    assert torch.all(out[:, H * DV:] == 7.0)


def test_empty_sequence_copies_the_state():
    H = 3
    h0 = torch.randn((H, DV, DK), device=DEV)
    h_out = torch.empty_like(h0)
    z = torch.empty((0, H * DK), dtype=torch.bfloat16, device=DEV)
    nv.nvfp4_gdn_recurrence(z, z, torch.empty((0, H * DV), dtype=torch.bfloat16, device=DEV),
                            torch.empty((0, H), device=DEV), torch.empty((0, H), device=DEV), h0, h_out=h_out)
    torch.cuda.synchronize()
    assert torch.equal(h_out, h0)


@pytest.mark.slow
def test_full_length_sampled_heads():
    """32768 tokens, 32 heads (the GDN projection's layout), BF16 in and out:
    every token of three sampled heads against the oracle."""
    T, H = 32768, wl.GDN_HEADS
    q, k, v, beta, g = wl.make_recurrence_inputs(T, H, H, 11, "bf16")
    h_out = torch.empty((H, DV, DK), dtype=torch.float32, device=DEV)
    out = nv.nvfp4_gdn_recurrence(_t(q, "bf16"), _t(k, "bf16"), _t(v, "bf16"), _t(beta, "f32"), _t(g, "f32"),
                                  h_out=h_out)
    torch.cuda.synchronize()
    heads = [0, 13, 31]
    ref_o, ref_s, mag = _reference(q, k, v, beta, g, H, H, None, 0.0, heads=heads)
    got = out.double().cpu().numpy().reshape(T, H, DV)[:, heads]
    _check_out(got, ref_o, mag, True, "full length")
    _check_state(h_out.cpu().numpy().astype(np.float64)[heads], ref_s, "full length")
