"""GPU parity of gdn_chunk_fwd against the fp64 oracle, through the C ABI."""
import zlib

import numpy as np
import pytest
import torch

import gated_deltanet_chunked_prefill_b200 as gdn
from gated_deltanet_chunked_prefill_b200.workloads import CONFIGS, config_inputs, make_inputs
from oracle import fwd_chunk, fwd_token

from _helpers import assert_close, oracle_unit_fwd, to_dev

pytestmark = pytest.mark.gpu

SMALL = {
    # name: (B, T, Hqk, Hv, dk, dv, dtype, h0_std, lengths)
    "tiny_fp32_full": (1, 256, 2, 2, 64, 64, "f32", None, None),
    "f32_d128_ragged": (2, 200, 2, 2, 128, 128, "f32", 0.1, None),
    "f32_d64_gqa_varlen": (1, 0, 1, 2, 64, 64, "f32", 0.1, [1, 63, 64, 65, 130]),
    "bf16_d128_ragged": (2, 300, 2, 2, 128, 128, "bf16", 0.1, None),
    "bf16_d128_gqa": (1, 257, 2, 4, 128, 128, "bf16", None, None),
    "bf16_d128_varlen": (1, 0, 2, 2, 128, 128, "bf16", 0.1, [1, 64, 65, 130, 7, 200]),
    "bf16_d64": (1, 190, 2, 2, 64, 64, "bf16", 0.1, None),
    "bf16_d128_long": (1, 1100, 1, 1, 128, 128, "bf16", 0.1, None),
}


def run_gpu(x, **kw):
    d = to_dev(x)
    o, hT = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"],
                              d["cu_seqlens"], **kw)
    torch.cuda.synchronize()
    return o.cpu(), hT.cpu()


@pytest.mark.parametrize("name", list(SMALL))
def test_fwd_small_parity(name):
    B, T, Hqk, Hv, dk, dv, dt, h0, lengths = SMALL[name]
    x = make_inputs(B, T, Hqk, Hv, dk, dv, dt, seed=zlib.crc32(name.encode()) % 1000, h0_std=h0, lengths=lengths)
    o, hT = run_gpu(x)
    ro, rh = fwd_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"],
                       x["cu_seqlens"], chunk=64)
    assert_close(o, ro, dt, f"{name} o")
    assert_close(hT, rh, dt, f"{name} hT")


@pytest.mark.parametrize("name", ["tiny_fp32_full", "f32_d128_ragged", "f32_d64_gqa_varlen", "bf16_d64"])
def test_fwd_cuda_core_weak_decay(name):
    """The CUDA-core sizes with g x 0.01. With the recipe's decay, entries of L and P more than a
    dozen tokens below the diagonal fall under fp32 resolution, so a wrong long-range term would
    go unseen; with mild decay every term of the chunk and the state carried across chunks
    weigh in."""
    B, T, Hqk, Hv, dk, dv, dt, h0, lengths = SMALL[name]
    x = make_inputs(B, T, Hqk, Hv, dk, dv, dt, seed=zlib.crc32(name.encode()) % 1000 + 1, h0_std=h0,
                    lengths=lengths)
    x["g"] = x["g"] * 0.01
    o, hT = run_gpu(x)
    ro, rh = fwd_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"],
                       x["cu_seqlens"], chunk=64)
    assert_close(o, ro, dt, f"{name} weak decay o")
    assert_close(hT, rh, dt, f"{name} weak decay hT")


@pytest.mark.parametrize("exact", [False, True])
@pytest.mark.parametrize("cp", [-1, 1, 2, 3])
def test_fwd_context_parallel_matches_oracle(cp, exact):
    """Forced segment lengths (1..3 chunks), both ways of obtaining a segment's start state
    (gate-driven window, exact affine stitch), against the oracle; packed sequences put the
    segment boundaries at odd token positions."""
    x = make_inputs(1, 0, 2, 4, 128, 128, "bf16", seed=77, h0_std=0.1,
                    lengths=[700, 64, 1, 333, 129])
    o, hT = run_gpu(x, cp_segment_chunks=cp, cp_exact=exact)
    ro, rh = fwd_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"],
                       x["cu_seqlens"], chunk=64)
    assert_close(o, ro, "bf16", f"cp={cp} o")
    assert_close(hT, rh, "bf16", f"cp={cp} hT")


def test_fwd_weak_decay_long_sequence():
    """g close to 0: the state remembers across many chunks (and CP segments); the
    gate-driven window cannot close, so those segments start at the sequence start."""
    x = make_inputs(2, 2000, 1, 2, 128, 128, "bf16", seed=5, h0_std=0.1, g_scale=1.0)
    x["g"] = (x["g"] * 0.01).contiguous()
    for cp, exact in ((-1, False), (4, False), (4, True), (7, True)):
        o, hT = run_gpu(x, cp_segment_chunks=cp, cp_exact=exact)
        ro, rh = fwd_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"],
                           None, chunk=64)
        assert_close(o, ro, "bf16", f"weak decay cp={cp} exact={exact} o")
        assert_close(hT, rh, "bf16", f"weak decay cp={cp} exact={exact} hT")


def _decay_pattern(x, pattern, f=0.01):
    """g scaled along the sequence (and per v-head): 'weak' x f everywhere; 'weak_then_strong'
    / 'strong_then_weak' x f in one half of each sequence; 'mixed_heads' x f on even v-heads."""
    g = x["g"].clone()
    T = g.shape[1]
    if pattern == "weak":
        g *= f
    elif pattern == "weak_then_strong":
        g[:, : T // 2] *= f
    elif pattern == "strong_then_weak":
        g[:, T // 2:] *= f
    elif pattern == "mixed_heads":
        g[:, :, 0::2] *= f
    x["g"] = g.contiguous()
    return x


@pytest.mark.parametrize("pattern", ["weak", "weak_then_strong", "strong_then_weak", "mixed_heads"])
@pytest.mark.parametrize("cp_exact", [2, 0])
def test_fwd_gate_with_exact_fallback(pattern, cp_exact):
    """Segments whose gate window does not close: mode 2 gives them the exact stitch (only where
    needed: a segment after a closing window gets its start straight from phase 1), the default mode
    (0) restarts them at the sequence start; both match the oracle. 3-chunk segments, so a sequence
    has many of them, some closing and some not."""
    x = _decay_pattern(make_inputs(2, 2500, 1, 2, 128, 128, "bf16", seed=17, h0_std=0.1), pattern)
    o, hT = run_gpu(x, cp_segment_chunks=3, cp_exact=cp_exact)
    ro, rh = fwd_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"], None, chunk=64)
    assert_close(o, ro, "bf16", f"{pattern} mode {cp_exact} o")
    assert_close(hT, rh, "bf16", f"{pattern} mode {cp_exact} hT")


def test_fwd_gate_fallback_packed_mixed_heads():
    """Packed sequences of mixed lengths (segment boundaries at odd token positions) with weakly and
    strongly decaying v-heads side by side, the exact fallback (mode 2), against the oracle."""
    x = make_inputs(1, 0, 2, 4, 128, 128, "bf16", seed=19, h0_std=0.1, lengths=[1500, 64, 1, 777, 300])
    x = _decay_pattern(x, "mixed_heads")
    o, hT = run_gpu(x, cp_segment_chunks=2, cp_exact=2)
    ro, rh = fwd_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"], x["cu_seqlens"], chunk=64)
    assert_close(o, ro, "bf16", "o")
    assert_close(hT, rh, "bf16", "hT")


@pytest.mark.parametrize("exact", [False, True])
def test_fwd_context_parallel_dense_unit_norm_violation(exact):
    """Keys far from unit norm (beta |k|^2 > 2): the per-token bound grows instead of
    decaying, the gate-driven window falls back to the sequence start; still exact."""
    x = make_inputs(1, 900, 1, 1, 128, 128, "bf16", seed=8, h0_std=0.1)
    x["k"] = (x["k"].float() * 1.8).to(torch.bfloat16)
    x["g"] = (x["g"] * 0.2).contiguous()
    o, hT = run_gpu(x, cp_segment_chunks=3, cp_exact=exact)
    ro, rh = fwd_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"], None, chunk=64)
    assert_close(o, ro, "bf16", "o")
    assert_close(hT, rh, "bf16", "hT")


def test_fwd_cp_bit_identical_when_segments_decay():
    """Strong decay: the gate-driven start state equals the exact one to fp32 resolution."""
    x = make_inputs(1, 1500, 2, 2, 128, 128, "bf16", seed=12, h0_std=0.1)
    o0, h0 = run_gpu(x, cp_segment_chunks=-1)
    o1, h1 = run_gpu(x, cp_segment_chunks=5)
    o2, h2 = run_gpu(x, cp_segment_chunks=5, cp_exact=True)
    from _helpers import rel_l2
    assert rel_l2(o1, o0) < 2e-3 and rel_l2(o2, o0) < 2e-3
    assert rel_l2(h1, h0) < 2e-3 and rel_l2(h2, h0) < 2e-3


def test_fwd_no_cross_sequence_leakage():
    lengths = [100, 64, 37, 200]
    x = make_inputs(1, 0, 2, 2, 128, 128, "bf16", seed=9, h0_std=0.1, lengths=lengths)
    o1, h1 = run_gpu(x)
    cu = x["cu_seqlens"].tolist()
    m = 1                                       # perturb sequence 1 only
    y = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    s, e = cu[m], cu[m + 1]
    for name in ("q", "k", "v"):
        y[name][:, s:e] = -y[name][:, s:e]
    y["g"][:, s:e] = y["g"][:, s:e] * 0.5
    y["beta"][:, s:e] = 1 - y["beta"][:, s:e]
    y["h0"][m] = 3.0
    o2, h2 = run_gpu(y)
    for n in range(len(lengths)):
        if n == m:
            continue
        a, b = cu[n], cu[n + 1]
        assert torch.equal(o1[:, a:b], o2[:, a:b]), n
        assert torch.equal(h1[n], h2[n]), n
    assert not torch.equal(o1[:, s:e], o2[:, s:e])


@pytest.mark.parametrize("cp_exact", [0, 1, 2])
def test_fwd_no_cross_sequence_leakage_with_context_parallelism(cp_exact):
    """Packed sequences split into 2-chunk segments (every mode of obtaining a segment's start):
    perturbing one sequence, which spans several segments, leaves every other sequence's o and hT
    bit for bit unchanged."""
    lengths = [300, 451, 129, 520, 64]
    x = make_inputs(1, 0, 2, 2, 128, 128, "bf16", seed=29, h0_std=0.1, lengths=lengths)
    o1, h1 = run_gpu(x, cp_segment_chunks=2, cp_exact=cp_exact)
    cu = x["cu_seqlens"].tolist()
    m = 1
    y = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    s, e = cu[m], cu[m + 1]
    for name in ("q", "k", "v"):
        y[name][:, s:e] = -y[name][:, s:e]
    y["g"][:, s:e] = y["g"][:, s:e] * 0.01          # weak decay: its windows do not close
    y["beta"][:, s:e] = 1 - y["beta"][:, s:e]
    y["h0"][m] = 3.0
    o2, h2 = run_gpu(y, cp_segment_chunks=2, cp_exact=cp_exact)
    for n in range(len(lengths)):
        if n == m:
            continue
        a, b = cu[n], cu[n + 1]
        assert torch.equal(o1[:, a:b], o2[:, a:b]), n
        assert torch.equal(h1[n], h2[n]), n
    assert not torch.equal(o1[:, s:e], o2[:, s:e])


def test_fwd_empty_and_zero_length_sequences():
    x = make_inputs(1, 0, 1, 1, 128, 128, "bf16", seed=3, h0_std=0.1, lengths=[0, 70, 0])
    o, hT = run_gpu(x)
    ro, rh = fwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"],
                       x["cu_seqlens"])
    assert_close(o, ro, "bf16", "o")
    assert torch.equal(hT[0], x["h0"][0]) and torch.equal(hT[2], x["h0"][2])


def test_fwd_bad_cu_seqlens_reports_device_status():
    x = make_inputs(1, 0, 1, 1, 128, 128, "bf16", seed=4, h0_std=None, lengths=[64, 64])
    d = to_dev(x)
    d["cu_seqlens"] = torch.tensor([0, 100, 64], dtype=torch.int32, device="cuda")  # not monotone
    ws = torch.zeros(gdn.fwd_workspace_size(1, 128, 1, 1, 128, 128, 2), dtype=torch.uint8,
                     device="cuda")
    gdn.check_device_error()                        # start from a clear per-device word
    gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None, None, d["cu_seqlens"],
                      workspace=ws, check_status=False)
    assert gdn.read_device_status(ws) == 6
    assert gdn.read_device_status(ws) == 0          # reading clears it
    assert gdn.check_device_error() == 6            # the per-device word saw it too
    assert gdn.check_device_error() == 0
    with pytest.raises(gdn.GdnError, match="inconsistent device input"):
        gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None, None, d["cu_seqlens"],
                          workspace=ws, check_status=True)
    gdn.check_device_error()


def test_fwd_bounded_wait_times_out_and_context_stays_usable():
    """The testing hook makes one thread of every CTA wait on a barrier that nothing completes:
    the wait gives up after ~1 ms, the call reports GDN_ERR_DEVICE_TIMEOUT through the workspace
    and the per-device status word, and the next call on the same context works."""
    x = make_inputs(1, 300, 2, 2, 128, 128, "bf16", seed=21, h0_std=0.1)
    d = to_dev(x)
    ws = torch.zeros(gdn.fwd_workspace_size(1, 300, 2, 2, 128, 128, 1), dtype=torch.uint8, device="cuda")
    gdn.check_device_error()
    gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], workspace=ws,
                      test_stall=True, check_status=False)
    assert gdn.read_device_status(ws) == 5
    assert gdn.check_device_error() == 5
    assert gdn.check_device_error() == 0
    o, hT = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], workspace=ws,
                              check_status=True)
    torch.cuda.synchronize()
    ro, rh = fwd_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"], None, chunk=64)
    assert_close(o.cpu(), ro, "bf16", "o after a timed-out call")
    assert_close(hT.cpu(), rh, "bf16", "hT after a timed-out call")
    assert gdn.check_device_error() == 0


def test_fwd_cp_mode_segments_and_deterministic_flag():
    """cp_mode = n (at most n segments per sequence) and deterministic = 1 give the oracle's
    result; with the same segmentation the output is bit-identical to cp_segment_chunks."""
    x = make_inputs(1, 1500, 2, 2, 128, 128, "bf16", seed=13, h0_std=0.1)
    o1, h1 = run_gpu(x, cp_mode=4, deterministic=True)
    o2, h2 = run_gpu(x, cp_segment_chunks=6)         # 24 chunks / 4 segments
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
    ro, rh = fwd_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"], None, chunk=64)
    assert_close(o1, ro, "bf16", "o")
    assert_close(h1, rh, "bf16", "hT")


# ---------------------------------------------------------------- full-size configurations
FULL = {
    # (sequence, v-head) units: first and last head, first and last sequence, others spread out
    "dense_bf16": [(0, 0), (3, 15), (1, 7), (2, 3), (0, 12), (3, 0), (1, 15), (2, 9)],
    "long_gqa_bf16": [(0, 0), (0, 31), (0, 18), (0, 1), (0, 7), (0, 14), (0, 23), (0, 30)],
    "varlen_bf16": None,   # sampled below: the longest, the shortest, ragged ones, the last
}


@pytest.mark.parametrize("name", list(FULL))
def test_fwd_full_size_sampled_units(name):
    x = config_inputs(name)
    o, hT = run_gpu(x)
    assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
    units = FULL[name]
    if units is None:
        L = np.diff(x["cu_seqlens"].numpy())
        ragged = [n for n in range(len(L)) if L[n] % 64][:3]
        units = [(int(np.argmax(L)), 3), (int(np.argmax(L)), 15), (int(np.argmin(L)), 11), (5, 0),
                 (len(L) - 1, 15), (0, 8)] + [(n, (5 * n) % 16) for n in ragged]
    for n, j in units:
        ro, rh, (b, s, e) = oracle_unit_fwd(x, n, j)
        assert_close(o[b, s:e, j], ro, "bf16", f"{name} unit ({n},{j}) o")
        assert_close(hT[n, j], rh, "bf16", f"{name} unit ({n},{j}) hT")
