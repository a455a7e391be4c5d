"""GPU parity of the recurrent decode step (gdn_recurrent_step) against the fp64 oracle's token
form, and continuity with the chunked prefill: prefill T tokens, then step the next one."""
import zlib

import pytest
import torch

import gated_deltanet_chunked_prefill_b200 as gdn
from gated_deltanet_chunked_prefill_b200.workloads import make_inputs
from oracle import fwd_token

from _helpers import assert_close

pytestmark = pytest.mark.gpu

CASES = {
    # name: (N, Hqk, Hv, dk, dv, dtype)
    "bf16_d128": (5, 2, 2, 128, 128, "bf16"),
    "bf16_gqa": (3, 2, 4, 128, 128, "bf16"),
    "f32_d64": (4, 1, 2, 64, 64, "f32"),
    "f32_dk128_dv64": (2, 1, 1, 128, 64, "f32"),
    "f32_dk64_dv128": (2, 1, 1, 64, 128, "f32"),
    "bf16_d256": (3, 1, 2, 256, 256, "bf16"),
    "f32_d256": (2, 1, 1, 256, 256, "f32"),
    "f32_dk256_dv64": (2, 1, 1, 256, 64, "f32"),
    "bf16_dk64_dv256_gqa": (2, 1, 2, 64, 256, "bf16"),
}


def _step_inputs(x, t):
    """Token t of every sequence as [N, H, d] tensors on the GPU."""
    return {n: x[n][:, t].contiguous().cuda() for n in ("q", "k", "v", "g", "beta")}


@pytest.mark.parametrize("name", list(CASES))
def test_step_parity(name):
    N, Hqk, Hv, dk, dv, dt = CASES[name]
    x = make_inputs(N, 1, Hqk, Hv, dk, dv, dt, seed=zlib.crc32(name.encode()) % 1000, h0_std=0.5)
    s = _step_inputs(x, 0)
    state = x["h0"].clone().cuda()
    o = gdn.gdn_recurrent_step(s["q"], s["k"], s["v"], s["g"], s["beta"], state, x["scale"])
    torch.cuda.synchronize()
    o_ref, h_ref = fwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"])
    assert_close(o.cpu(), o_ref[:, 0], dt, f"{name} o")
    assert_close(state.cpu(), h_ref, "f32", f"{name} state")


def test_prefill_then_decode():
    """Chunked prefill over 300 tokens, then 3 decode steps from its hT: the same outputs and final
    state as the oracle over all 303 tokens."""
    B, T, steps = 2, 303, 3
    x = make_inputs(B, T, 2, 2, 128, 128, "bf16", seed=77, h0_std=0.1)
    pre = {n: x[n][:, :T - steps].contiguous().cuda() for n in ("q", "k", "v", "g", "beta")}
    _, state = gdn.gdn_chunk_fwd(pre["q"], pre["k"], pre["v"], pre["g"], pre["beta"], x["scale"],
                                 x["h0"].cuda())
    outs = []
    for t in range(T - steps, T):
        s = _step_inputs(x, t)
        outs.append(gdn.gdn_recurrent_step(s["q"], s["k"], s["v"], s["g"], s["beta"], state, x["scale"]))
    torch.cuda.synchronize()
    o_ref, h_ref = fwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"])
    for i, t in enumerate(range(T - steps, T)):
        assert_close(outs[i].cpu(), o_ref[:, t], "bf16", f"o[{t}]")
    assert_close(state.cpu(), h_ref, "bf16", "state")


def test_step_zero_decay_identity():
    """g = 0, beta = 0: the state is unchanged (bit for bit) and o = scale h^T q."""
    x = make_inputs(3, 1, 1, 1, 128, 128, "f32", seed=78, h0_std=0.3)
    s = _step_inputs(x, 0)
    s["g"].zero_()
    s["beta"].zero_()
    state = x["h0"].clone().cuda()
    o = gdn.gdn_recurrent_step(s["q"], s["k"], s["v"], s["g"], s["beta"], state, x["scale"])
    torch.cuda.synchronize()
    assert torch.equal(state.cpu(), x["h0"])
    ref = x["scale"] * torch.einsum("nhdr,nhd->nhr", x["h0"].double(), x["q"][:, 0].double())
    assert_close(o.cpu(), ref, "f32", "o")
