"""GPU tests of the host-buffer entry point (gdn_chunk_host): host arrays in, host arrays out,
through the C ABI. Its kernels are those of gdn_chunk_fwd / gdn_chunk_bwd, so every output must
equal, bit for bit, the device-buffer calls on the same inputs; one case is also checked against
the fp64 oracle. The asynchronous mode (three streams, two scratch buffers used in turn) must give
every call its own inputs' results."""
import pytest
import torch

import gated_deltanet_chunked_prefill_b200 as gdn
from gated_deltanet_chunked_prefill_b200.workloads import make_inputs
from oracle import bwd_token, fwd_chunk

from _helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dg", "dbeta", "dh0")
CASES = {
    # name: (B, T, Hqk, Hv, h0_std, lengths)
    "ragged": (2, 300, 2, 2, 0.1, None),
    "gqa": (1, 257, 2, 4, None, None),
    "varlen": (1, 0, 2, 2, 0.1, [1, 64, 65, 130, 7, 200]),
}


def _inputs(name, seed, backward=True):
    B, T, Hqk, Hv, h0, lengths = CASES[name]
    return make_inputs(B, T, Hqk, Hv, 128, 128, "bf16", seed=seed, h0_std=h0, lengths=lengths, backward=backward)


def _host_args(x, pin=True):
    keys = ("q", "k", "v", "g", "beta", "h0", "cu_seqlens", "dO", "dhT")
    h = {k: (x[k].contiguous().pin_memory() if pin else x[k].contiguous()) if isinstance(x.get(k), torch.Tensor)
         else None for k in keys}
    h["scale"] = x["scale"]
    return h


def _device_results(x, mode):
    d = to_dev(x)
    out = {}
    if mode in ("fwd", "fwdbwd"):
        states = gdn.chunk_states(d["q"], d["v"], d["cu_seqlens"]) if mode == "fwdbwd" else None
        o, hT = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], d["cu_seqlens"],
                                  states=states)
        out.update(o=o, hT=hT)
    if mode in ("bwd", "fwdbwd"):
        gr = gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["scale"], d["h0"], d["dhT"],
                               d["cu_seqlens"], states=states if mode == "fwdbwd" else None)
        out.update(gr)
    torch.cuda.synchronize()
    return {k: v.cpu() for k, v in out.items() if v is not None}


def _host_call(h, mode, **kw):
    return gdn.gdn_chunk_host(h["q"], h["k"], h["v"], h["g"], h["beta"], h["scale"], h["h0"], h["cu_seqlens"],
                              dO=h["dO"] if mode != "fwd" else None, dhT=h["dhT"] if mode != "fwd" else None,
                              mode=mode, **kw)


@pytest.mark.parametrize("mode", ["fwd", "bwd", "fwdbwd"])
@pytest.mark.parametrize("name", list(CASES))
def test_host_call_equals_device_calls(name, mode):
    x = _inputs(name, seed=300 + len(name))
    got = _host_call(_host_args(x), mode)
    ref = _device_results(x, mode)
    assert set(ref) <= set(got)
    for k, v in ref.items():
        assert not got[k].is_cuda
        assert torch.equal(got[k], v), f"{name} {mode} {k}"


def test_host_call_pageable_memory_and_oracle():
    """Pageable host arrays work too (each copy then blocks the thread); the forward + backward
    step matches the oracle."""
    x = _inputs("varlen", seed=311)
    got = _host_call(_host_args(x, pin=False), "fwdbwd")
    ro, rh = fwd_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"], x["cu_seqlens"])
    assert_close(got["o"], ro, "bf16", "o")
    assert_close(got["hT"], rh, "bf16", "hT")
    ref = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"], x["dhT"],
                    x["cu_seqlens"])
    for n in GRADS:
        assert_close(got[n], ref[n], "bf16", n)


def test_host_calls_overlap_with_two_scratch_buffers():
    """Six calls on three streams with two scratch buffers and two output sets used in turn, none
    synchronised until the end: the third call reuses the first call's scratch while the second
    runs, so the library's per-scratch events must order its copies after the first call's
    kernels and its kernels after the first call's output copies. Every call gets exactly the
    device-call results of its own inputs."""
    dev = torch.device("cuda", torch.cuda.current_device())
    compute, h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    xs = [_inputs("ragged", seed=400 + i) for i in range(6)]
    hosts = [_host_args(x) for x in xs]
    B, T, Hqk, Hv, _, _ = CASES["ragged"]
    need = gdn.host_scratch_size("fwdbwd", torch.bfloat16, B, T, Hqk, Hv, 128, 128, B)
    scratch = [torch.empty(need, dtype=torch.uint8, device=dev) for _ in range(2)]
    results = []
    for i, h in enumerate(hosts):
        out = _host_call(h, "fwdbwd", scratch=scratch[i % 2], stream=compute, h2d_stream=h2d, d2h_stream=d2h,
                         synchronize=False)
        results.append(out)                   # a fresh output set per call
    d2h.synchronize()
    torch.cuda.synchronize()
    for i, x in enumerate(xs):
        ref = _device_results(x, "fwdbwd")
        for k, v in ref.items():
            assert torch.equal(results[i][k], v), f"call {i} {k}"


def test_host_call_reuses_output_buffers():
    """outputs= reuses a previous call's host buffers (no new allocation) and overwrites them."""
    x1, x2 = _inputs("gqa", seed=501), _inputs("gqa", seed=502)
    out = _host_call(_host_args(x1), "fwdbwd")
    ptrs = {k: v.data_ptr() for k, v in out.items()}
    out2 = _host_call(_host_args(x2), "fwdbwd", outputs=out)
    assert {k: v.data_ptr() for k, v in out2.items()} == ptrs
    ref = _device_results(x2, "fwdbwd")
    for k, v in ref.items():
        assert torch.equal(out2[k], v), k


def test_host_call_passes_options():
    """Options reach the kernels unchanged: q/k normalisation and an explicit segment length give
    the device calls' results bit for bit."""
    x = make_inputs(1, 900, 2, 2, 128, 128, "bf16", seed=601, h0_std=0.1, backward=True, qk_unit=False)
    h = _host_args(x)
    got = _host_call(h, "fwdbwd", qk_l2norm=True, cp_segment_chunks=3)
    d = to_dev(x)
    states = gdn.chunk_states(d["q"], d["v"], d["cu_seqlens"])
    o, hT = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], d["cu_seqlens"],
                              states=states, qk_l2norm=True, cp_segment_chunks=3)
    gr = gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["scale"], d["h0"], d["dhT"],
                           d["cu_seqlens"], states=states, qk_l2norm=True, cp_segment_chunks=3)
    torch.cuda.synchronize()
    ref = dict(o=o, hT=hT, **gr)
    for k, v in ref.items():
        if v is not None:
            assert torch.equal(got[k], v.cpu()), k


def test_host_call_cuda_core_sizes():
    """fp32 with head dims 64 through the host entry: the CUDA-core forward and backward."""
    x = make_inputs(1, 0, 1, 2, 64, 64, "f32", seed=611, h0_std=0.1, lengths=[100, 1, 64], backward=True)
    got = _host_call(_host_args(x), "fwdbwd")
    d = to_dev(x)
    o, hT = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], d["cu_seqlens"])
    gr = gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["scale"], d["h0"], d["dhT"],
                           d["cu_seqlens"])
    torch.cuda.synchronize()
    ref = dict(o=o, hT=hT, **gr)
    for k, v in ref.items():
        assert torch.equal(got[k], v.cpu()), k


def test_host_call_many_scratch_buffers():
    """A new scratch buffer per call (80 of them, all kept alive so their addresses differ): the
    library's event table releases the idle ones past 64 addresses, and calls keep giving the
    device calls' results, including one reusing the first buffer."""
    x = make_inputs(1, 64, 1, 1, 128, 128, "bf16", seed=701, backward=True)
    h = _host_args(x)
    need = gdn.host_scratch_size("fwdbwd", torch.bfloat16, 1, 64, 1, 1, 128, 128, 1)
    bufs = [torch.empty(need, dtype=torch.uint8, device="cuda") for _ in range(80)]
    outs = [_host_call(h, "fwdbwd", scratch=b) for b in bufs]
    outs.append(_host_call(h, "fwdbwd", scratch=bufs[0]))
    ref = _device_results(x, "fwdbwd")
    for out in (outs[0], outs[70], outs[-1]):
        for k, v in ref.items():
            assert torch.equal(out[k], v), k
