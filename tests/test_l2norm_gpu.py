"""GPU parity of the in-kernel q/k L2 normalisation (gdn_options.qk_l2norm): raw q, k ~ N(0, 1)
go in, every row is divided by sqrt(|x|^2 + 1e-6) inside the kernels, and the forward outputs and
all six gradients (dq, dk with respect to the raw rows) match the fp64 oracle with the same
normalisation, through the C ABI and through the autograd entry point."""
import zlib

import pytest
import torch

import gated_deltanet_chunked_prefill_b200 as gdn
from gated_deltanet_chunked_prefill_b200.workloads import make_inputs
from oracle import bwd_token, fwd_chunk

from _helpers import assert_close, rel_l2, to_dev

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dg", "dbeta", "dh0")

CASES = {
    # name: (B, T, Hqk, Hv, h0_std, lengths, cp_segment_chunks, cp_exact)
    "ragged": (2, 300, 2, 2, 0.1, None, -1, False),
    "gqa": (1, 257, 2, 4, None, None, -1, False),
    "varlen": (1, 0, 2, 2, 0.1, [1, 64, 65, 130, 7, 200], 0, False),
    "cp_gate": (1, 900, 1, 2, 0.1, None, 3, False),
    "cp_exact": (1, 0, 1, 2, 0.1, [700, 64, 333], 2, True),
}


def _inputs(name, backward=False):
    B, T, Hqk, Hv, h0, lengths, _, _ = CASES[name]
    return make_inputs(B, T, Hqk, Hv, 128, 128, "bf16", seed=zlib.crc32(name.encode()) % 1000 + 500,
                       h0_std=h0, lengths=lengths, backward=backward, qk_unit=False)


@pytest.mark.parametrize("name", list(CASES))
def test_l2norm_forward_parity(name):
    *_, cp, exact = CASES[name]
    x = _inputs(name)
    d = to_dev(x)
    o, hT = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], d["cu_seqlens"],
                              cp_segment_chunks=cp, cp_exact=exact, qk_l2norm=True)
    torch.cuda.synchronize()
    ro, rh = fwd_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"], x["cu_seqlens"],
                       qk_l2norm=True)
    assert_close(o.cpu(), ro, "bf16", f"{name} o")
    assert_close(hT.cpu(), rh, "bf16", f"{name} hT")
    # without the normalisation the same raw inputs give a different operator (with beta |k|^2 far
    # above 2 the unnormalised recurrence grows without bound, so its result may not even be finite)
    o2, _ = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], d["cu_seqlens"],
                              cp_segment_chunks=cp, cp_exact=exact)
    assert not rel_l2(o2.cpu(), ro) <= 0.1


@pytest.mark.parametrize("name", ["ragged", "gqa", "varlen", "cp_gate"])
def test_l2norm_backward_parity(name):
    *_, cp, _exact = CASES[name]
    x = _inputs(name, backward=True)
    d = to_dev(x)
    gr = gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["scale"], d["h0"], d["dhT"],
                           d["cu_seqlens"], cp_segment_chunks=cp, qk_l2norm=True)
    torch.cuda.synchronize()
    ref = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"], x["dhT"],
                    x["cu_seqlens"], qk_l2norm=True)
    for n in GRADS:
        assert_close(gr[n].cpu(), ref[n], "bf16", f"{name} {n}")


def test_l2norm_cached_states_match_recompute():
    """The forward's chunk-state cache (written with the normalisation) gives the backward the same
    gradients, bit for bit, as the backward's own forward pass."""
    x = _inputs("varlen", backward=True)
    d = to_dev(x)
    states = gdn.chunk_states(d["q"], d["v"], d["cu_seqlens"])
    gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], d["cu_seqlens"],
                      states=states, qk_l2norm=True)
    args = (d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["scale"], d["h0"], d["dhT"], d["cu_seqlens"])
    cached = gdn.gdn_chunk_bwd(*args, states=states, qk_l2norm=True)
    recomputed = gdn.gdn_chunk_bwd(*args, qk_l2norm=True)
    torch.cuda.synchronize()
    for n in GRADS:
        assert torch.equal(cached[n], recomputed[n]), n


def test_l2norm_unit_rows_match_plain_path():
    """On rows that are already of unit norm the normalisation changes the result only at eps and
    rounding level."""
    x = make_inputs(1, 500, 2, 2, 128, 128, "bf16", seed=71, h0_std=0.1, backward=True)
    d = to_dev(x)
    o1, h1 = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], qk_l2norm=True)
    o0, h0 = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"])
    torch.cuda.synchronize()
    assert rel_l2(o1.cpu(), o0.cpu()) < 5e-3 and rel_l2(h1.cpu(), h0.cpu()) < 5e-3


def test_l2norm_autograd_entry():
    """chunk_gated_delta_rule(use_qk_l2norm_in_kernel=True): output and gradients of raw q, k."""
    x = _inputs("gqa", backward=True)
    d = to_dev(x)
    leaves = {n: d[n].clone().requires_grad_(True) for n in ("q", "k", "v", "g", "beta")}
    o, hT = gdn.chunk_gated_delta_rule(leaves["q"], leaves["k"], leaves["v"], leaves["g"], leaves["beta"],
                                       scale=d["scale"], output_final_state=True, use_qk_l2norm_in_kernel=True)
    (o.float() * d["dO"].float()).sum().add((hT * d["dhT"]).sum()).backward()
    ref = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], None, x["dhT"],
                    qk_l2norm=True)
    ro, _ = fwd_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], None, qk_l2norm=True)
    assert_close(o.detach().cpu(), ro, "bf16", "o")
    for n, gname in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("beta", "dbeta")):
        assert_close(leaves[n].grad.cpu(), ref[gname], "bf16", f"autograd {gname}")
