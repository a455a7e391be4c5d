"""CUDA-graph capture of the C-ABI calls (the way a serving or training loop removes launch
overhead): a forward + backward step and a run of decode steps are captured once, then replayed on
new data copied into the captured buffers; every replay equals the eager calls bit for bit."""
import pytest
import torch

import gated_deltanet_chunked_prefill_b200 as gdn
from gated_deltanet_chunked_prefill_b200.workloads import make_inputs

from _helpers import to_dev

pytestmark = pytest.mark.gpu


def _fwdbwd(d, states, ws_f, ws_b, o, hT):
    gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], d["cu_seqlens"],
                      states=states, workspace=ws_f, o=o, hT=hT, check_status=False)
    return gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["scale"], d["h0"], d["dhT"],
                             d["cu_seqlens"], states=states, workspace=ws_b, check_status=False)


def test_graph_replay_forward_backward():
    lengths = [300, 129, 64, 507]
    xs = [make_inputs(1, 0, 2, 4, 128, 128, "bf16", seed=800 + i, h0_std=0.1, lengths=lengths, backward=True)
          for i in range(3)]
    static = to_dev(xs[0])
    B, T, Hqk, Hv, N = 1, sum(lengths), 2, 4, len(lengths)
    states = gdn.chunk_states(static["q"], static["v"], static["cu_seqlens"])
    ws_f = torch.zeros(gdn.fwd_workspace_size(B, T, Hqk, Hv, 128, 128, N), dtype=torch.uint8, device="cuda")
    ws_b = torch.zeros(gdn.bwd_workspace_size(B, T, Hqk, Hv, 128, 128, N, states=states), dtype=torch.uint8,
                       device="cuda")
    o = torch.empty_like(static["v"])
    hT = torch.empty((N, Hv, 128, 128), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):                      # warm-up outside the capture (module load, attributes)
        _fwdbwd(static, states, ws_f, ws_b, o, hT)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        grads = _fwdbwd(static, states, ws_f, ws_b, o, hT)
    for x in xs[1:]:
        for key, t in static.items():
            if isinstance(t, torch.Tensor):
                t.copy_(x[key].to(t.device))
        graph.replay()
        torch.cuda.synchronize()
        got = {"o": o.clone(), "hT": hT.clone(), **{k: v.clone() for k, v in grads.items() if v is not None}}
        d = to_dev(x)
        ref_o, ref_hT = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"],
                                          d["cu_seqlens"])
        ref = gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["scale"], d["h0"], d["dhT"],
                                d["cu_seqlens"])
        torch.cuda.synchronize()
        assert torch.equal(got["o"], ref_o) and torch.equal(got["hT"], ref_hT)
        for k, v in ref.items():
            if v is not None:
                assert torch.equal(got[k], v), k
    assert gdn.check_device_error() == 0


def test_graph_replay_decode_steps():
    """Eight decode steps captured once (state updated in place), replayed: the same state and
    outputs as eight eager steps from the same start."""
    N, H, d = 32, 4, 128
    toks = [make_inputs(N, 1, H, H, d, d, "bf16", seed=850 + i, h0_std=0.1) for i in range(8)]
    start = toks[0]["h0"].cuda()
    state = start.clone()
    inputs = [{n: t[n][:, 0].contiguous().cuda() for n in ("q", "k", "v", "g", "beta")} for t in toks]
    outs = [torch.empty((N, H, d), dtype=torch.bfloat16, device="cuda") for _ in range(8)]
    scale = d ** -0.5
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        gdn.gdn_recurrent_step(inputs[0]["q"], inputs[0]["k"], inputs[0]["v"], inputs[0]["g"], inputs[0]["beta"],
                               state.clone(), scale, o=outs[0])
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(8):
            t = inputs[i]
            gdn.gdn_recurrent_step(t["q"], t["k"], t["v"], t["g"], t["beta"], state, scale, o=outs[i])
    state.copy_(start)
    graph.replay()
    torch.cuda.synchronize()
    ref_state = start.clone()
    for i in range(8):
        t = inputs[i]
        ref_o = gdn.gdn_recurrent_step(t["q"], t["k"], t["v"], t["g"], t["beta"], ref_state, scale)
        torch.cuda.synchronize()
        assert torch.equal(outs[i], ref_o), i
    assert torch.equal(state, ref_state)
