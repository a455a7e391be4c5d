"""GPU parity of the CUDA-core backward (fp32 I/O, head dims of 64) against the fp64 oracle's token
adjoint, through the C ABI: all six gradients, packed and grouped inputs, partial blocks, empty
sequences; bit-reproducible across calls."""
import pytest
import torch

import gated_deltanet_chunked_prefill_b200 as gdn
from gated_deltanet_chunked_prefill_b200.workloads import CONFIGS, make_inputs
from oracle import bwd_token

from _helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dg", "dbeta", "dh0")
CASES = {
    # name: (B, T, Hqk, Hv, dk, dv, dtype, h0_std, lengths)
    "fp32_d64": (1, 256, 2, 2, 64, 64, "f32", None, None),
    "fp32_d128_ragged": (2, 150, 1, 1, 128, 128, "f32", 0.1, None),
    "bf16_d64_gqa": (1, 200, 1, 2, 64, 64, "bf16", 0.1, None),
    "fp32_mixed_dims": (1, 131, 1, 1, 64, 128, "f32", 0.1, None),
    "fp32_d64_varlen": (1, 0, 1, 2, 64, 64, "f32", 0.1, [70, 0, 1, 129, 64, 33]),
}


def _run(x, **kw):
    d = to_dev(x)
    gr = gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["scale"], d["h0"], d["dhT"],
                           d["cu_seqlens"], **kw)
    torch.cuda.synchronize()
    return {k: (v.cpu() if v is not None else None) for k, v in gr.items()}


@pytest.mark.parametrize("name", list(CASES))
def test_cuda_core_backward_parity(name):
    B, T, Hqk, Hv, dk, dv, dtype, h0, lengths = CASES[name]
    x = make_inputs(B, T, Hqk, Hv, dk, dv, dtype, seed=900 + len(name), h0_std=h0, lengths=lengths, backward=True)
    got = _run(x)
    ref = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"], x["dhT"],
                    x["cu_seqlens"])
    tol = "f32" if dtype == "f32" else "bf16"
    for n in GRADS:
        assert got[n].dtype == (torch.float32 if n in ("dg", "dh0") or dtype == "f32" else torch.bfloat16), n
        assert_close(got[n], ref[n], tol, f"{name} {n}")


@pytest.mark.parametrize("name", ["fp32_d64", "bf16_d64_gqa", "fp32_d64_varlen"])
def test_cuda_core_backward_weak_decay(name):
    """g x 0.01: the adjoint carried back across many tokens keeps its weight (with the recipe's
    decay it fades within a chunk), so every term of the reverse pass is exercised."""
    B, T, Hqk, Hv, dk, dv, dtype, h0, lengths = CASES[name]
    x = make_inputs(B, T, Hqk, Hv, dk, dv, dtype, seed=960 + len(name), h0_std=h0, lengths=lengths, backward=True)
    x["g"] = x["g"] * 0.01
    got = _run(x)
    ref = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"], x["dhT"],
                    x["cu_seqlens"])
    tol = "f32" if dtype == "f32" else "bf16"
    for n in GRADS:
        assert_close(got[n], ref[n], tol, f"{name} weak decay {n}")


def test_cuda_core_backward_tiny_fp32_config_and_reproducible():
    """The tiny fp32 workload (B1 H2 T256 d64) end to end, twice: bit-identical results (every
    reduction in a fixed order)."""
    w = CONFIGS["tiny_fp32"]
    x = make_inputs(w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.dtype, w.seed, h0_std=w.h0_std, backward=True)
    a, b = _run(x), _run(x)
    for n in GRADS:
        assert torch.equal(a[n], b[n]), n
    ref = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"], x["dhT"],
                    x["cu_seqlens"])
    for n in GRADS:
        assert_close(a[n], ref[n], "f32", f"tiny fp32 {n}")


def test_cuda_core_backward_refuses_a_cache():
    """The chunk-state cache belongs to the tensor-core path: refused here before anything runs."""
    x = make_inputs(1, 64, 1, 1, 64, 64, "f32", seed=950, backward=True)
    d = to_dev(x)
    states = torch.zeros(1 << 20, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gdn.GdnError):
        gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], None, states=states)
