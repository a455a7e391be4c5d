"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
entry point include/gdn.h declares, and rejects invalid calls before launching
anything. Only calls that fail host validation are made here (no kernel runs).
"""
import ctypes
import os
import re

import pytest
import torch

import gated_deltanet_chunked_prefill_b200 as gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")

FAKE = 0x7F0000000000        # 16-byte aligned address that is never dereferenced
MISALIGNED = FAKE + 8


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = gdn.lib()
    names = declared_functions()
    assert "gdn_chunk_fwd" in names and "gdn_chunk_bwd" in names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version():
    L = gdn.lib()
    for code in range(7):
        assert L.gdn_status_string(code)
    assert L.gdn_version() >= 100


def test_workspace_size_has_status_head():
    for dims in [(1, 256, 2, 2, 64, 64, 1), (4, 4096, 16, 16, 128, 128, 4),
                 (1, 32768, 16, 32, 128, 128, 1), (1, 65536, 16, 16, 128, 128, 24)]:
        assert gdn.fwd_workspace_size(*dims) >= 256
        assert gdn.bwd_workspace_size(*dims) >= 256
        assert gdn.fwd_workspace_size(*dims) % 256 == 0


def _fwd(dtype=1, B=1, T=64, Hqk=1, Hv=1, dk=128, dv=128, q=FAKE, k=FAKE, v=FAKE, g=FAKE,
         beta=FAKE, h0=None, cu=None, N=1, o=FAKE, hT=None, ws=FAKE, wsb=1 << 20, opt=None):
    L = gdn.lib()
    vp = ctypes.c_void_p
    o_ = gdn.Options() if opt is None else opt
    return L.gdn_chunk_fwd(dtype, B, T, Hqk, Hv, dk, dv, vp(q), vp(k), vp(v), vp(g), vp(beta),
                           0.1, vp(h0) if h0 else None, vp(cu) if cu else None, N, vp(o),
                           vp(hT) if hT else None, vp(ws) if ws else None, wsb, ctypes.byref(o_),
                           None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), 1), (dict(T=-1), 1), (dict(Hqk=3, Hv=4), 1), (dict(Hqk=0), 1),
    (dict(dk=96), 2), (dict(dv=32), 2), (dict(dtype=7), 1),
    (dict(q=None), 1), (dict(o=None), 1), (dict(g=MISALIGNED), 1), (dict(h0=MISALIGNED), 1),
    (dict(ws=None), 3), (dict(wsb=16), 3), (dict(ws=MISALIGNED), 3),
    (dict(cu=FAKE, B=2, N=2), 1), (dict(cu=FAKE, N=0), 1),
])
def test_forward_rejects_invalid_arguments(kw, code):
    assert _fwd(**kw) == code


def test_forward_rejects_reserved_options():
    o = gdn.Options()
    o.reserved[1] = 1
    assert _fwd(opt=o) == 1


@pytest.mark.parametrize("field,value", [("deterministic", 2), ("qk_l2norm", -1), ("test_stall", 3),
                                         ("cp_mode", -2), ("cp_exact", 3), ("cp_exact", -1)])
def test_forward_rejects_option_values_out_of_range(field, value):
    o = gdn.Options()
    setattr(o, field, value)
    assert _fwd(opt=o) == 1


def test_deterministic_option_accepted():
    """deterministic = 1 is accepted (every path already reduces in a fixed order): the call gets
    past option validation to the workspace check."""
    o = gdn.Options()
    o.deterministic = 1
    assert _fwd(opt=o, ws=None) == 3


def test_cp_mode_gives_the_segment_count():
    """cp_mode = n asks for at most n segments: the plan matches cp_segment_chunks of
    ceil(chunks / n) (visible in the exact stitch's workspace, which holds per-segment maps)."""
    dims = (1, 4096, 1, 1, 128, 128, 1)           # 64 chunks
    for n, seg in ((4, 16), (3, 22), (64, 1)):
        assert gdn.fwd_workspace_size(*dims, cp_mode=n, cp_exact=True) == \
            gdn.fwd_workspace_size(*dims, cp_segment_chunks=seg, cp_exact=True)
    assert gdn.fwd_workspace_size(*dims, cp_mode=-1, cp_exact=True) == \
        gdn.fwd_workspace_size(*dims, cp_segment_chunks=-1, cp_exact=True) < \
        gdn.fwd_workspace_size(*dims, cp_mode=2, cp_exact=True)
    # cp_segment_chunks, when set, wins over cp_mode
    assert gdn.fwd_workspace_size(*dims, cp_mode=4, cp_segment_chunks=8, cp_exact=True) == \
        gdn.fwd_workspace_size(*dims, cp_segment_chunks=8, cp_exact=True)


def test_context_parallel_modes_workspace():
    """The exact fallback (mode 2) keeps per-segment maps and window records only once a sequence can
    have 3 or more segments; the restart mode (0) needs none; the exact stitch (1) always has maps."""
    dims = (1, 8192, 1, 8, 128, 128, 1)             # 128 chunks
    ws = lambda **kw: gdn.fwd_workspace_size(*dims, **kw)
    maps = 2 * 4 * 8 * 128 * 128 * 4               # 4 segments x 8 v-heads x (M, b), fp32
    assert ws(cp_segment_chunks=32, cp_exact=0) + maps <= ws(cp_segment_chunks=32, cp_exact=2)
    assert ws(cp_segment_chunks=32, cp_exact=1) + 4 * 8 * 4 <= ws(cp_segment_chunks=32, cp_exact=2) + 256
    assert ws(cp_segment_chunks=64, cp_exact=2) == ws(cp_segment_chunks=64, cp_exact=0)   # 2 segments


def test_interface_names():
    """The calls and option fields of the interface exist under their names."""
    L = gdn.lib()
    for name in ("gdn_chunk_fwd", "gdn_chunk_bwd", "gdn_chunk_fwd_workspace_size", "gdn_chunk_bwd_workspace_size",
                 "gdn_status_string", "gdn_check_device_error", "gdn_read_device_status"):
        assert hasattr(L, name), name
    fields = [f[0] for f in gdn.Options._fields_]
    assert fields[:2] == ["cp_mode", "deterministic"]
    for code in range(8):
        assert L.gdn_status_string(code) != b"unknown status"


def test_state_rows_beyond_32_bit_coordinates_refused():
    """Chunk-state rows (slots x Hv x 128) are 32-bit TMA coordinates: sizes whose rows do not fit
    are refused on the host, for a forward that caches states and for the backward."""
    T = 1 << 26                                   # B * T * H = 2^30 fits; 2^20 slots * 16 * 128 = 2^31 does not
    o = gdn.Options()
    o.states = FAKE
    assert _fwd(T=T, Hqk=16, Hv=16, opt=o) == 2
    assert _fwd(T=T, Hqk=16, Hv=16, opt=o, ws=None) == 2     # refused before the workspace check
    L = gdn.lib()
    vp = ctypes.c_void_p
    f = vp(FAKE)
    st = L.gdn_chunk_bwd(1, 1, T, 16, 16, 128, 128, f, f, f, f, f, 0.1, None, None, 1, f, None, f, f, f, f, f,
                         None, f, 1 << 40, ctypes.byref(gdn.Options()), None)
    assert st == 2


def test_binding_refuses_a_states_cache_that_does_not_fit():
    """The C ABI takes the chunk-state cache as a bare pointer; the binding checks its size and
    device against the inputs first."""
    from gated_deltanet_chunked_prefill_b200 import _check_states
    q = torch.zeros(1, 256, 2, 128, dtype=torch.bfloat16)
    v = torch.zeros(1, 256, 2, 128, dtype=torch.bfloat16)
    need = gdn.lib().gdn_chunk_states_size(1, 256, 2, 2, 128, 128, 1)
    _check_states(torch.zeros(need // 2, dtype=torch.bfloat16), q, v, None)
    with pytest.raises(ValueError, match="bytes"):
        _check_states(torch.zeros(need // 2 - 1, dtype=torch.bfloat16), q, v, None)
    with pytest.raises(ValueError, match="device"):
        _check_states(torch.zeros(need // 2, dtype=torch.bfloat16, device="meta"), q, v, None)


def test_python_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 64, 1, 128, dtype=torch.bfloat16)
    g = torch.zeros(1, 64, 1)
    with pytest.raises(ValueError):
        gdn.gdn_chunk_fwd(x, x, x, g, torch.zeros(1, 64, 1, dtype=torch.bfloat16))


def test_options_struct_layout():
    # int cp_mode, deterministic, cp_segment_chunks, cp_exact; pointer; int qk_l2norm, test_stall,
    # reserved[2]: 40 bytes with the pointer at offset 16
    assert ctypes.sizeof(gdn.Options) == 40
    assert gdn.Options.states.offset == 16
    assert gdn.Options.qk_l2norm.offset == 24


def test_chunk_states_size():
    L = gdn.lib()
    per = 128 * 128 * 2 + 64 * 64 * 4 + 64 * 64 * 2   # bf16 start state, fp32 A, bf16 P per chunk slot
    # independent sequences: N * ceil(T / 64) slots per v-head
    assert L.gdn_chunk_states_size(2, 8192, 16, 16, 128, 128, 0) == 2 * 128 * 16 * per
    assert L.gdn_chunk_states_size(3, 100, 2, 4, 128, 128, 0) == 3 * 2 * 4 * per
    # packed: ceil(T / 64) + N slots bound the chunks of any split of T tokens into N sequences
    assert L.gdn_chunk_states_size(1, 65536, 16, 16, 128, 128, 24) == (1024 + 24) * 16 * per
    assert L.gdn_chunk_states_size(0, 64, 1, 1, 128, 128, 0) == 0


def test_states_option_checks():
    o = gdn.Options()
    o.states = FAKE
    assert _fwd(dtype=0, dk=64, dv=64, opt=o) == 2        # fp32 / CUDA-core path: unsupported
    n = gdn.Options()
    n.qk_l2norm = 1
    assert _fwd(dtype=0, dk=64, dv=64, opt=n) == 2        # the normalisation: tensor-core path only
    assert _fwd(dtype=1, dk=64, dv=64, opt=n) == 2
    o.states = MISALIGNED
    assert _fwd(opt=o) == 1


def test_autograd_entry_host_checks():
    """The autograd entry point refuses what it does not do before touching the GPU."""
    x = torch.zeros(1, 64, 1, 128)
    g = torch.zeros(1, 64, 1)
    with pytest.raises(ValueError):
        gdn.chunk_gated_delta_rule(x, x, x, g, g)
    from gated_deltanet_chunked_prefill_b200.autograd import _host_cu_seqlens
    _host_cu_seqlens(torch.tensor([0, 3, 3, 10]), 10)
    for bad in ([0, 5, 3, 10], [1, 10], [0, 9]):
        with pytest.raises(ValueError, match="cu_seqlens"):
            _host_cu_seqlens(torch.tensor(bad), 10)
    from gated_deltanet_chunked_prefill_b200.autograd import backward_supported
    assert backward_supported(x.to(torch.bfloat16), x)
    assert backward_supported(x, x)                                       # fp32: CUDA-core backward
    assert backward_supported(torch.zeros(1, 64, 1, 64, dtype=torch.bfloat16), x)       # dk = 64
    assert not backward_supported(x.double(), x)
    assert not backward_supported(torch.zeros(1, 64, 1, 96), x)           # dk = 96


def test_recurrent_step_host_validation():
    """gdn_recurrent_step rejects bad arguments on the host (no GPU call is reached)."""
    L = gdn.lib()
    p = ctypes.c_void_p(16)                   # never dereferenced: validation fails first
    call = lambda dtype, N, Hqk, Hv, dk, dv, ptr: L.gdn_recurrent_step(dtype, N, Hqk, Hv, dk, dv, ptr, ptr, ptr,
                                                                        ptr, ptr, 1.0, ptr, ptr, None)
    assert call(7, 1, 1, 1, 128, 128, p) == 1                # unknown dtype
    assert call(1, 1, 2, 3, 128, 128, p) == 1                # Hv not a multiple of Hqk
    assert call(1, -1, 1, 1, 128, 128, p) == 1               # negative N
    assert call(1, 1, 1, 1, 96, 128, p) == 2                 # unsupported head dim
    assert call(1, 1, 1, 1, 128, 512, p) == 2
    assert call(1, 1 << 28, 1, 2, 256, 256, p) == 2          # grid of N * Hv * dv / 64 blocks beyond 2^31 - 1
    assert call(1, 1, 1, 1, 128, 128, None) == 1             # null pointers
    assert call(1, 1, 1, 1, 128, 128, ctypes.c_void_p(24)) == 1   # misaligned
    assert call(1, 0, 1, 1, 128, 128, None) == 0             # N = 0: nothing to do


def test_binding_refuses_mismatched_shapes():
    """Shapes that disagree with q and v are refused on the host (the C ABI would trust them)."""
    from gated_deltanet_chunked_prefill_b200.workloads import make_inputs
    x = make_inputs(2, 70, 2, 4, 64, 64, "f32", seed=3, h0_std=0.1, backward=True)
    args = lambda **kw: {**{n: x[n] for n in ("q", "k", "v", "g", "beta")}, "h0": x["h0"], **kw}
    fwd = lambda a: gdn.gdn_chunk_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], None, a["h0"])
    with pytest.raises(ValueError, match="CUDA"):           # consistent shapes reach the device check
        fwd(args())
    bad = {"k": x["k"][:, :, :1], "g": x["g"][:, :, :2], "beta": x["beta"][:1], "h0": x["h0"][:1],
           "v": x["v"][:, :69]}
    for name, t in bad.items():
        with pytest.raises(ValueError, match=name):
            fwd(args(**{name: t}))
    with pytest.raises(ValueError, match="dO"):
        gdn.gdn_chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["dO"][:, :, :1], None, x["h0"], x["dhT"])
    with pytest.raises(ValueError, match="dhT"):
        gdn.gdn_chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["dO"], None, x["h0"], x["dhT"][:1])
    # the decode step: q, k [N,Hqk,dk], v [N,Hv,dv], g, beta [N,Hv], state [N,Hv,dk,dv]
    t = {n: x[n][:, 0].contiguous() for n in ("q", "k", "v", "g", "beta")}
    step = lambda **kw: gdn.gdn_recurrent_step(**{**t, "state": x["h0"], **kw})
    with pytest.raises(ValueError, match="CUDA"):
        step()
    for name, bad_t in (("state", x["h0"][:, :1]), ("g", t["g"][:, :1]), ("k", t["k"][:1])):
        with pytest.raises(ValueError, match=name):
            step(**{name: bad_t})


def _host(mode=3, dtype=1, B=1, T=64, Hqk=1, Hv=1, dk=128, dv=128, q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE,
          h0=None, cu=None, N=1, dO=FAKE, dhT=None, o=FAKE, hT=None, dq=FAKE, dk_=FAKE, dv_=FAKE, dg=FAKE, db=FAKE,
          dh0=None, scratch=FAKE, nbytes=1 << 40, opt=None):
    L = gdn.lib()
    o_ = gdn.Options() if opt is None else opt

    def n(p):
        return ctypes.c_void_p(p) if p else None
    return L.gdn_chunk_host(mode, dtype, B, T, Hqk, Hv, dk, dv, n(q), n(k), n(v), n(g), n(beta), 0.1, n(h0), n(cu),
                            N, n(dO), n(dhT), n(o), n(hT), n(dq), n(dk_), n(dv_), n(dg), n(db), n(dh0), n(scratch),
                            nbytes, ctypes.byref(o_), None, None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(mode=0), 1), (dict(mode=4), 1), (dict(dtype=7), 1), (dict(B=0), 1), (dict(Hqk=3, Hv=4), 1),
    (dict(dk=96), 2), (dict(q=None), 1), (dict(g=None), 1), (dict(mode=1, o=None), 1),
    (dict(mode=2, dO=None), 1), (dict(mode=3, dq=None), 1), (dict(mode=2, dbeta_absent=True), 1),
    (dict(mode=2, dtype=0, opt_l2=True), 2), (dict(mode=1, dk=64, dv=64, opt_l2=True), 2),
    (dict(scratch=None), 3), (dict(scratch=FAKE + 16), 3), (dict(nbytes=1024), 3),
    (dict(cu=FAKE, B=2, N=2), 1),
])
def test_host_call_rejects_invalid_arguments(kw, code):
    """gdn_chunk_host validates everything before its first copy: these calls return at once
    (a call that passed would need a GPU)."""
    if kw.pop("dbeta_absent", False):
        kw["db"] = None
    if kw.pop("opt_l2", False):                # the normalisation: tensor-core sizes only
        kw["opt"] = gdn.Options()
        kw["opt"].qk_l2norm = 1
    assert _host(**kw) == code


def test_host_call_refuses_a_states_option():
    o = gdn.Options()
    o.states = FAKE                  # the host call keeps its own chunk-state cache in the scratch
    assert _host(opt=o) == 1
    o = gdn.Options()
    o.reserved[0] = 1
    assert _host(opt=o) == 1


def test_host_scratch_size():
    """The scratch holds a device copy of every array of the mode (and, for forward + backward, the
    chunk-state cache): it grows with the mode's arrays, covers the packed reading of B == 1, and is
    0 for invalid sizes."""
    L = gdn.lib()
    opt = gdn.Options()

    def size(mode, dims, dtype=1):
        return int(L.gdn_chunk_host_scratch_size(mode, dtype, *dims, ctypes.byref(opt)))
    dims = (2, 1024, 2, 4, 128, 128, 2)
    B, T, Hqk, Hv, dk, dv, N = dims
    inputs = 2 * B * T * Hqk * dk * 2 + B * T * Hv * dv * 2 + B * T * Hv * 6
    f, b, fb = size(1, dims), size(2, dims), size(3, dims)
    assert f >= inputs + B * T * Hv * dv * 2 and f % 256 == 0
    assert b >= inputs + B * T * Hv * dv * 2 + inputs          # dO in, the gradients out
    assert fb > f and fb > b - gdn.bwd_workspace_size(*dims)
    states = int(L.gdn_chunk_states_size(*dims))
    assert fb >= f + states
    # B == 1 with num_seqs: covers 24 packed sequences as well as one unpacked one
    packed = (1, 65536, 16, 16, 128, 128, 24)
    assert size(3, packed) >= size(3, packed[:6] + (0,))
    assert size(3, (0, 64, 1, 1, 128, 128, 1)) == 0
    assert size(5, dims) == 0
    assert size(1, dims, dtype=0) > 0 and size(2, dims, dtype=0) > 0


def test_host_binding_checks():
    """The binding refuses non-host, mistyped or misshapen arrays before calling the C ABI."""
    q = torch.zeros(1, 64, 1, 128, dtype=torch.bfloat16)
    v = torch.zeros(1, 64, 1, 128, dtype=torch.bfloat16)
    g = torch.zeros(1, 64, 1)
    beta = torch.zeros(1, 64, 1, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        gdn.gdn_chunk_host(q, q, v, g.double(), beta)
    with pytest.raises(ValueError):
        gdn.gdn_chunk_host(q, q, v, g, beta, mode="bwd")            # no dO
    with pytest.raises(ValueError):
        gdn.gdn_chunk_host(q, q, v, g, beta, mode="sideways")
    with pytest.raises(ValueError):
        gdn.gdn_chunk_host(q[:, ::2], q[:, ::2], v[:, ::2], g[:, ::2], beta[:, ::2])   # not contiguous
    with pytest.raises(ValueError):
        gdn.gdn_chunk_host(q, q, v, g, beta, dO=torch.zeros(1, 64, 2, 128, dtype=torch.bfloat16))


def _bwd(dtype=1, B=1, T=64, Hqk=1, Hv=1, dk=128, dv=128, ws=FAKE, wsb=1 << 40, opt=None):
    L = gdn.lib()
    vp = ctypes.c_void_p
    o_ = gdn.Options() if opt is None else opt
    f = vp(FAKE)
    return L.gdn_chunk_bwd(dtype, B, T, Hqk, Hv, dk, dv, f, f, f, f, f, 0.1, None, None, 1, f, None, f, f, f, f, f,
                           None, vp(ws) if ws else None, wsb, ctypes.byref(o_), None)


def test_backward_cuda_core_path_host_checks():
    """fp32 or head dims 64 take the CUDA-core backward, which has neither the chunk-state cache nor
    the in-kernel q/k normalisation; its workspace is checked against its own plan."""
    o = gdn.Options()
    o.states = FAKE
    assert _bwd(dtype=0, opt=o) == 2
    assert _bwd(dtype=1, dk=64, dv=64, opt=o) == 2
    n = gdn.Options()
    n.qk_l2norm = 1
    assert _bwd(dtype=0, dk=64, dv=64, opt=n) == 2
    assert _bwd(dtype=0, dk=64, dv=64, ws=None) == 3
    assert _bwd(dtype=0, dk=64, dv=64, wsb=1024) == 3
    assert _bwd(dtype=0, dk=96, dv=64) == 2
    # the size query (no dtype) covers the CUDA-core plan: fp32 checkpoints every 64 tokens
    per = 64 * 64 * 4
    assert gdn.bwd_workspace_size(1, 256, 2, 2, 64, 64, 1) >= 4 * 2 * per
    assert gdn.bwd_workspace_size(2, 8192, 16, 16, 128, 128, 2) >= 2 * 128 * 16 * 128 * 128 * 4


def test_empty_inputs_succeed_before_any_device_work():
    """T = 0 is a valid call that does nothing: the host-buffer entry and the CUDA-core backward
    return GDN_OK after validation, before any device query or launch (this runs without a GPU)."""
    assert _host(T=0) == 0
    assert _host(mode=1, T=0, dtype=0, dk=64, dv=64) == 0
    assert _bwd(dtype=0, dk=64, dv=64, T=0) == 0
    assert _bwd(dtype=0, dk=64, dv=64, T=0, ws=None) == 3      # the workspace is still checked


@pytest.mark.skipif(torch.cuda.is_available(), reason="the probe calls pass validation and would then run")
@pytest.mark.parametrize("dims,packed", [((2, 300, 2, 4, 128, 128, 2), False), ((1, 700, 1, 2, 128, 128, 5), True),
                                         ((1, 256, 2, 2, 64, 64, 1), False), ((1, 500, 1, 1, 64, 128, 3), True),
                                         ((1, 1 << 20, 16, 16, 128, 128, 1), False),     # tens of GiB of scratch
                                         ((1, 300000, 4, 8, 64, 128, 1000), True)])
def test_size_queries_cover_their_calls(dims, packed):
    """Every size query covers its call: given exactly the queried bytes, a call passes all of its
    host checks and stops only at its first CUDA call (status GDN_ERR_CUDA here, on a machine
    without a GPU), while one byte less is refused as GDN_ERR_WORKSPACE."""
    L = gdn.lib()
    B, T, Hqk, Hv, dk, dv, N = dims
    cu = FAKE if packed else None
    opt = gdn.Options()
    for dtype in (0, 1):
        for mode in (1, 2, 3):
            need = int(L.gdn_chunk_host_scratch_size(mode, dtype, B, T, Hqk, Hv, dk, dv, N if packed else 0,
                                                     ctypes.byref(opt)))
            assert need > 0
            assert _host(mode=mode, dtype=dtype, B=B, T=T, Hqk=Hqk, Hv=Hv, dk=dk, dv=dv, cu=cu, N=N,
                         nbytes=need) == 4, (dtype, mode)
            assert _host(mode=mode, dtype=dtype, B=B, T=T, Hqk=Hqk, Hv=Hv, dk=dk, dv=dv, cu=cu, N=N,
                         nbytes=need - 1) == 3, (dtype, mode)
        wsb = gdn.bwd_workspace_size(B, T, Hqk, Hv, dk, dv, N if packed else 0)
        f = ctypes.c_void_p(FAKE)
        args = lambda ws_bytes: (dtype, B, T, Hqk, Hv, dk, dv, f, f, f, f, f, 0.1, None, ctypes.c_void_p(cu) if cu else None,
                                 N, f, None, f, f, f, f, f, None, f, ws_bytes, ctypes.byref(opt), None)
        assert L.gdn_chunk_bwd(*args(wsb)) == 4, dtype
        assert L.gdn_chunk_bwd(*args(16)) == 3, dtype
        if dtype == 0 or dk != 128 or dv != 128:      # the query takes no dtype: it covers both backward plans
            assert L.gdn_chunk_bwd(*args(wsb // 2)) == 3, dtype


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without the built library every entry point raises: there is no CPU path to fall back to,
    not even for the host-buffer entry, whose inputs are CPU tensors."""
    from gated_deltanet_chunked_prefill_b200.workloads import make_inputs
    monkeypatch.setattr(gdn, "LIB_PATH", str(tmp_path / "libgdn.so"))
    monkeypatch.setattr(gdn, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        gdn.lib()
    x = make_inputs(1, 64, 1, 1, 128, 128, "bf16", seed=1, backward=True)
    with pytest.raises(RuntimeError, match="not built|NVIDIA driver"):   # whichever it meets first
        gdn.gdn_chunk_host(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], None, None, mode="fwd")
    with pytest.raises(Exception):
        gdn.chunk_gated_delta_rule(x["q"], x["k"], x["v"], x["g"], x["beta"], scale=x["scale"])
