"""The package docstring's usage example runs as written and gives the same
outputs as the two steps called on their own."""
import textwrap

import pytest
import torch

import bit_quantized_linear_nvfp4_b200 as pkg
from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv

pytestmark = pytest.mark.gpu


def _example_code():
    doc = pkg.__doc__
    start = doc.index("::\n") + 3
    end = doc.index("\n\nSegments may")
    return textwrap.dedent(doc[start:end])


def test_docstring_example_runs_and_matches_the_two_steps():
    gen = torch.Generator(device="cuda").manual_seed(5)
    M, K = 96, 512
    env = {
        "M": M,
        "x": torch.randn((M, K), generator=gen, device="cuda").to(torch.bfloat16),
        "w_q": (torch.randn((256, K), generator=gen, device="cuda") * 0.02).to(torch.bfloat16),
        "w_k": (torch.randn((128, K), generator=gen, device="cuda") * 0.5).to(torch.bfloat16),
    }
    exec(compile(_example_code(), "package docstring", "exec"), env)
    torch.cuda.synchronize()
    A, g_a = nv.nvfp4_quantize(env["x"])
    q2 = torch.empty_like(env["q"])
    k2 = torch.empty_like(env["k"])
    segs = [nv.Segment(0, 256, "identity", q2), nv.Segment(256, 384, "identity", k2)]
    nv.nvfp4_fused_proj(A, g_a, env["W"], env["g_w"], segs)
    torch.cuda.synchronize()
    assert torch.equal(env["q"], q2)
    assert torch.equal(env["k"], k2)
    assert env["g_w"].shape == (2,) and bool(env["g_w"][0] != env["g_w"][1])
