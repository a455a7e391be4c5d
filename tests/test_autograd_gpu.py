"""The autograd entry point (flash-linear-attention call signature) on the GPU: its forward and
gradients are those of the same C-ABI calls (forward filling the chunk-state cache, backward
reading it), bit for bit, and match the fp64 oracle."""
import pytest
import torch

import gated_deltanet_chunked_prefill_b200 as gdn
from gated_deltanet_chunked_prefill_b200.workloads import make_inputs
from oracle import bwd_token, fwd_token

from _helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu

INPUTS = ("q", "k", "v", "g", "beta")


def _leaves(d, with_h0=True):
    out = {n: d[n].clone().requires_grad_(True) for n in INPUTS}
    out["h0"] = d["h0"].clone().requires_grad_(True) if with_h0 and d["h0"] is not None else d["h0"]
    return out


def _autograd(d, leaves, cu=None, final_state=True):
    o, hT = gdn.chunk_gated_delta_rule(leaves["q"], leaves["k"], leaves["v"], leaves["g"], leaves["beta"],
                                       scale=d["scale"], initial_state=leaves["h0"],
                                       output_final_state=final_state, cu_seqlens=cu)
    with_h0 = leaves["h0"] is not None and leaves["h0"].requires_grad
    wrt = [leaves[n] for n in INPUTS] + ([leaves["h0"]] if with_h0 else [])
    outs, grads_out = [o], [d["dO"]]
    if final_state:
        outs.append(hT)
        grads_out.append(d["dhT"])
    gr = torch.autograd.grad(outs, wrt, grads_out)
    torch.cuda.synchronize()
    names = list(INPUTS) + (["h0"] if with_h0 else [])
    return o, hT, dict(zip(names, gr))


def test_autograd_equals_c_abi():
    """Forward and every gradient equal the direct gdn_chunk_fwd / gdn_chunk_bwd results."""
    x = make_inputs(2, 300, 2, 2, 128, 128, "bf16", seed=71, h0_std=0.1, backward=True)
    d = to_dev(x)
    o, hT, gr = _autograd(d, _leaves(d))
    states = gdn.chunk_states(d["q"], d["v"])
    o_ref, hT_ref = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"],
                                      states=states)
    ref = gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["scale"], d["h0"], d["dhT"],
                            states=states)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(hT, hT_ref)
    for n, r in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("beta", "dbeta"), ("h0", "dh0")):
        assert torch.equal(gr[n], ref[r]), n


def test_autograd_gqa_packed_int64_oracle():
    """Grouped values on a packed batch with int64 cu_seqlens, against the oracle's token adjoint."""
    x = make_inputs(1, 0, 2, 4, 128, 128, "bf16", seed=72, h0_std=0.1, backward=True,
                    lengths=[130, 1, 64, 250])
    d = to_dev(x)
    o, hT, gr = _autograd(d, _leaves(d), cu=d["cu_seqlens"].to(torch.int64))
    o_ref, hT_ref = fwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"], x["cu_seqlens"])
    assert_close(o.cpu(), o_ref, "bf16", "o")
    assert_close(hT.cpu(), hT_ref, "bf16", "hT")
    ref = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"], x["dhT"],
                    x["cu_seqlens"])
    for n, r in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("beta", "dbeta"), ("h0", "dh0")):
        assert_close(gr[n].cpu(), ref[r], "bf16", n)


def test_autograd_without_final_state_or_h0_grad():
    """No final state requested (its gradient is absent) and an initial state that needs no grad."""
    x = make_inputs(1, 200, 1, 1, 128, 128, "bf16", seed=73, h0_std=0.1, backward=True)
    d = to_dev(x)
    leaves = _leaves(d, with_h0=False)
    o, hT, gr = _autograd(d, leaves, final_state=False)
    assert hT is None and "h0" not in gr
    states = gdn.chunk_states(d["q"], d["v"])
    gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], output_final_state=False,
                      states=states)
    ref = gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["scale"], d["h0"], None,
                            want_dh0=False, states=states)
    torch.cuda.synchronize()
    for n, r in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("beta", "dbeta")):
        assert torch.equal(gr[n], ref[r]), n


def test_autograd_cuda_core_paths():
    """fp32 and head dim 64: the forward equals the C ABI, and the gradients (CUDA-core backward)
    equal gdn_chunk_bwd's and match the oracle."""
    x = make_inputs(1, 100, 1, 1, 64, 64, "f32", seed=74, h0_std=0.1, backward=True)
    d = to_dev(x)
    with torch.no_grad():
        o, hT = gdn.chunk_gated_delta_rule(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d["h0"],
                                           output_final_state=True)
    o_ref, hT_ref = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None, d["h0"])
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(hT, hT_ref)
    leaves = {n: d[n].clone().requires_grad_(True) for n in ("q", "k", "v", "g", "beta", "h0")}
    o, hT = gdn.chunk_gated_delta_rule(leaves["q"], leaves["k"], leaves["v"], leaves["g"], leaves["beta"],
                                       initial_state=leaves["h0"], output_final_state=True)
    (o * d["dO"]).sum().add((hT * d["dhT"]).sum()).backward()
    gr = gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], None, d["h0"], d["dhT"])
    ref = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"], x["dhT"])
    torch.cuda.synchronize()
    for n, gname in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("beta", "dbeta"), ("h0", "dh0")):
        assert torch.equal(leaves[n].grad, gr[gname]), gname
        assert_close(leaves[n].grad.cpu(), ref[gname], "f32", f"autograd fp32 {gname}")