"""The allocation-free forward entry point, for callers that cannot allocate device
memory where they run the operator: its output must match gdn_chunk_fwd's on two calls
in a row (the library-held scratch is shared and keeps the previous call's contents).
Named to run last: a failure here leaves every other test already run."""
import ctypes

import pytest
import torch

import gated_deltanet_chunked_prefill_b200 as gdn
from gated_deltanet_chunked_prefill_b200.workloads import make_inputs

from _helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu

CASES = {
    # packed sequences long enough for automatic segments: the segment table lives in the scratch
    "packed_segments": dict(B=1, T=0, Hqk=2, Hv=4, lengths=[3000, 64, 1, 2333, 129, 2700], cp=0),
    "dense": dict(B=2, T=700, Hqk=2, Hv=2, lengths=None, cp=-1),
}


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_forward_matches_workspace_forward(name):
    c = CASES[name]
    x = make_inputs(c["B"], c["T"], c["Hqk"], c["Hv"], 128, 128, "bf16", seed=404, h0_std=0.1,
                    lengths=c["lengths"])
    d = to_dev(x)
    ref_o, ref_h = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"],
                                     d["cu_seqlens"], cp_segment_chunks=c["cp"])
    torch.cuda.synchronize()
    for call in range(2):
        o, h = gdn.gdn_chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"],
                                         d["cu_seqlens"], cp_segment_chunks=c["cp"])
        torch.cuda.synchronize()
        assert_close(o.cpu(), ref_o.cpu(), "bf16", f"{name} call {call} o")
        assert_close(h.cpu(), ref_h.cpu(), "bf16", f"{name} call {call} hT")


def test_noalloc_rejects_scratch_beyond_its_limit():
    # the exact affine stitch keeps two 64 KB maps per segment: far more than the 1 MiB array
    x = make_inputs(1, 8192, 1, 8, 128, 128, "bf16", seed=5, h0_std=None)
    d = to_dev(x)
    with pytest.raises(gdn.GdnError) as e:
        L = gdn.lib()
        opt = gdn.Options()
        opt.cp_segment_chunks = 2
        opt.cp_exact = 1
        o = torch.empty_like(d["v"])
        st = L.gdn_chunk_fwd_noalloc(1, 1, 8192, 1, 8, 128, 128, ctypes.c_void_p(d["q"].data_ptr()),
                                     ctypes.c_void_p(d["k"].data_ptr()), ctypes.c_void_p(d["v"].data_ptr()),
                                     ctypes.c_void_p(d["g"].data_ptr()), ctypes.c_void_p(d["beta"].data_ptr()),
                                     d["scale"], None, None, 1, ctypes.c_void_p(o.data_ptr()), None,
                                     ctypes.byref(opt), None)
        if st != 0:
            raise gdn.GdnError(st, "gdn_chunk_fwd_noalloc")
    assert e.value.code == 3
    assert b"static array holds" in gdn.lib().gdn_last_error()
