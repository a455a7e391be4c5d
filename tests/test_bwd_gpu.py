"""GPU parity of gdn_chunk_bwd against the fp64 oracle's token adjoint, through the C ABI."""
import zlib

import numpy as np
import pytest
import torch

import gated_deltanet_chunked_prefill_b200 as gdn
from gated_deltanet_chunked_prefill_b200.workloads import config_inputs, make_inputs
from oracle import bwd_token

from _helpers import assert_close, oracle_unit_bwd, rel_l2, to_dev

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dg", "dbeta", "dh0")

SMALL = {
    # name: (B, T, Hqk, Hv, h0_std, lengths)
    "ragged": (2, 300, 2, 2, 0.1, None),
    "one_chunk": (1, 64, 1, 1, 0.1, None),
    "partial_chunk": (1, 37, 1, 1, None, None),
    "gqa": (1, 257, 2, 4, 0.1, None),
    "varlen": (1, 0, 2, 2, 0.1, [1, 64, 65, 130, 7, 200]),
    "long": (1, 1100, 1, 1, 0.1, None),
}


def run_gpu_bwd(x, **kw):
    d = to_dev(x)
    gr = gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["scale"], d["h0"],
                           d["dhT"], d["cu_seqlens"], **kw)
    torch.cuda.synchronize()
    return {k: (v.cpu() if v is not None else None) for k, v in gr.items()}


def oracle_bwd(x):
    return bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"], x["dhT"],
                     x["cu_seqlens"])


@pytest.mark.parametrize("name", list(SMALL))
def test_bwd_small_parity(name):
    B, T, Hqk, Hv, h0, lengths = SMALL[name]
    x = make_inputs(B, T, Hqk, Hv, 128, 128, "bf16", seed=zlib.crc32(name.encode()) % 1000, h0_std=h0,
                    lengths=lengths, backward=True)
    gr = run_gpu_bwd(x)
    ref = oracle_bwd(x)
    for n in GRADS:
        assert_close(gr[n], ref[n], "bf16", f"{name} {n}")


@pytest.mark.parametrize("exact", [False, True])
@pytest.mark.parametrize("cp", [1, 2, 5])
def test_bwd_context_parallel(cp, exact):
    """Forced segments for the state pass and the reverse chain: gate-driven windows, or the exact
    affine stitch of both (the reverse one carries the state gradient from the sequence end);
    packed sequences put the segment boundaries at odd token positions."""
    x = make_inputs(1, 0, 2, 2, 128, 128, "bf16", seed=31, h0_std=0.1, backward=True,
                    lengths=[700, 64, 1, 333, 129])
    gr = run_gpu_bwd(x, cp_segment_chunks=cp, cp_exact=exact)
    ref = oracle_bwd(x)
    for n in GRADS:
        assert_close(gr[n], ref[n], "bf16", f"cp={cp} exact={exact} {n}")


@pytest.mark.parametrize("exact", [False, True])
def test_bwd_weak_decay_cp(exact):
    """g close to 0 (x 0.02): the state and its gradient remember across many segments."""
    x = make_inputs(1, 1000, 1, 2, 128, 128, "bf16", seed=32, h0_std=0.1, backward=True)
    x["g"] = (x["g"] * 0.02).contiguous()
    ref = oracle_bwd(x)
    for cp in (-1, 3):
        gr = run_gpu_bwd(x, cp_segment_chunks=cp, cp_exact=exact)
        for n in GRADS:
            assert_close(gr[n], ref[n], "bf16", f"weak decay cp={cp} exact={exact} {n}")


@pytest.mark.parametrize("pattern", ["weak", "weak_then_strong", "strong_then_weak", "mixed_heads"])
@pytest.mark.parametrize("cp_exact", [2, 0])
def test_bwd_gate_with_exact_fallback(pattern, cp_exact):
    """Mode 2: the state pass and the reverse chain give segments whose window does not close the
    exact stitch (each direction its own windows); mode 0 restarts them at the sequence end / start.
    3-chunk segments; all six gradients. g x 0.02
    over 1000 tokens: no window closes within 16 chunks, and the unsplit path still meets the bf16
    bars (much longer weakly decaying memories make |dg| large enough that no path does)."""
    from test_fwd_gpu import _decay_pattern
    x = _decay_pattern(make_inputs(1, 1000, 1, 2, 128, 128, "bf16", seed=35, h0_std=0.1, backward=True),
                       pattern, 0.02)
    gr = run_gpu_bwd(x, cp_segment_chunks=3, cp_exact=cp_exact)
    ref = oracle_bwd(x)
    for n in GRADS:
        assert_close(gr[n], ref[n], "bf16", f"{pattern} mode {cp_exact} {n}")


def test_bwd_gate_fallback_packed_cache():
    """Packed sequences with mixed decay per v-head, the exact fallback (mode 2), through the forward's
    cache and through the backward's own state pass: bit-identical, and matching the oracle."""
    from test_fwd_gpu import _decay_pattern
    x = _decay_pattern(make_inputs(1, 0, 2, 4, 128, 128, "bf16", seed=36, h0_std=0.1, backward=True,
                                   lengths=[900, 64, 1, 650, 300]), "mixed_heads", 0.02)
    d = to_dev(x)
    states = _fwd_states(d, cp_segment_chunks=2, cp_exact=2)
    cached = _bwd(d, cp_segment_chunks=2, cp_exact=2, states=states)
    recomputed = _bwd(d, cp_segment_chunks=2, cp_exact=2)
    ref = oracle_bwd(x)
    for n in GRADS:
        assert torch.equal(cached[n], recomputed[n]), n
        assert_close(cached[n], ref[n], "bf16", f"packed fallback {n}")


def test_bwd_exact_stitch_grouped_values_and_cache():
    """Exact stitch in both passes with grouped values; the forward's cache (exact stitch too) gives
    the same gradients, bit for bit, as the backward's own exact state pass."""
    x = make_inputs(1, 1300, 2, 4, 128, 128, "bf16", seed=34, h0_std=0.1, backward=True)
    d = to_dev(x)
    states = _fwd_states(d, cp_segment_chunks=4, cp_exact=True)
    cached = _bwd(d, cp_segment_chunks=4, cp_exact=True, states=states)
    recomputed = _bwd(d, cp_segment_chunks=4, cp_exact=True)
    ref = oracle_bwd(x)
    for n in GRADS:
        assert torch.equal(cached[n], recomputed[n]), n
        assert_close(cached[n], ref[n], "bf16", f"exact gqa {n}")


def test_bwd_no_cross_sequence_leakage():
    lengths = [100, 64, 37, 200]
    x = make_inputs(1, 0, 1, 2, 128, 128, "bf16", seed=33, h0_std=0.1, lengths=lengths, backward=True)
    g1 = run_gpu_bwd(x)
    cu = x["cu_seqlens"].tolist()
    m = 2
    y = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    s, e = cu[m], cu[m + 1]
    for name in ("q", "k", "v", "dO"):
        y[name][:, s:e] = -y[name][:, s:e]
    y["g"][:, s:e] *= 0.5
    y["dhT"][m] = 1.0
    g2 = run_gpu_bwd(y)
    for n in range(len(lengths)):
        if n == m:
            continue
        a, b = cu[n], cu[n + 1]
        for name in ("dq", "dk", "dv", "dg", "dbeta"):
            assert torch.equal(g1[name][:, a:b], g2[name][:, a:b]), (name, n)
        assert torch.equal(g1["dh0"][n], g2["dh0"][n])


@pytest.mark.parametrize("cp_exact", [0, 1, 2])
def test_bwd_no_cross_sequence_leakage_with_context_parallelism(cp_exact):
    """Packed sequences in 2-chunk segments for both sequential passes: perturbing one sequence
    leaves every other sequence's gradients bit for bit unchanged, in every context-parallel mode."""
    lengths = [300, 451, 129, 520, 64]
    x = make_inputs(1, 0, 1, 2, 128, 128, "bf16", seed=37, h0_std=0.1, lengths=lengths, backward=True)
    g1 = run_gpu_bwd(x, cp_segment_chunks=2, cp_exact=cp_exact)
    cu = x["cu_seqlens"].tolist()
    m = 3
    y = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    s, e = cu[m], cu[m + 1]
    for name in ("q", "k", "v", "dO"):
        y[name][:, s:e] = -y[name][:, s:e]
    y["g"][:, s:e] *= 0.01
    y["dhT"][m] = 1.0
    g2 = run_gpu_bwd(y, cp_segment_chunks=2, cp_exact=cp_exact)
    for n in range(len(lengths)):
        if n == m:
            continue
        a, b = cu[n], cu[n + 1]
        for name in ("dq", "dk", "dv", "dg", "dbeta"):
            assert torch.equal(g1[name][:, a:b], g2[name][:, a:b]), (name, n)
        assert torch.equal(g1["dh0"][n], g2["dh0"][n])
    assert not torch.equal(g1["dv"][:, s:e], g2["dv"][:, s:e])


def test_bwd_full_size_sampled_units():
    """The backward workload at full size: all six gradients of 8 (sequence, v-head) units (first
    and last head of both sequences among them) against the oracle's token adjoint."""
    x = config_inputs("bwd_bf16")
    gr = run_gpu_bwd(x)
    for name in GRADS:
        assert torch.isfinite(gr[name].float()).all(), name
    for n, j in [(0, 0), (1, 9), (0, 15), (1, 0), (1, 15), (0, 5), (1, 3), (0, 11)]:
        ref, (b, s, e) = oracle_unit_bwd(x, n, j)
        assert_close(gr["dq"][b, s:e, j], ref["dq"][0, :, 0], "bf16", f"unit ({n},{j}) dq")
        assert_close(gr["dk"][b, s:e, j], ref["dk"][0, :, 0], "bf16", f"unit ({n},{j}) dk")
        assert_close(gr["dv"][b, s:e, j], ref["dv"][0, :, 0], "bf16", f"unit ({n},{j}) dv")
        assert_close(gr["dg"][b, s:e, j], ref["dg"][0, :, 0], "bf16", f"unit ({n},{j}) dg")
        assert_close(gr["dbeta"][b, s:e, j], ref["dbeta"][0, :, 0], "bf16", f"unit ({n},{j}) dbeta")
        assert_close(gr["dh0"][n, j], ref["dh0"][0, 0], "bf16", f"unit ({n},{j}) dh0")


def _fwd_states(d, **kw):
    states = gdn.chunk_states(d["q"], d["v"], d["cu_seqlens"])
    gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], d["cu_seqlens"],
                      states=states, **kw)
    return states


def _bwd(d, **kw):
    gr = gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["scale"], d["h0"],
                           d["dhT"], d["cu_seqlens"], **kw)
    torch.cuda.synchronize()
    return {k: (v.cpu() if v is not None else None) for k, v in gr.items()}


@pytest.mark.parametrize("name,cp", [("ragged", 0), ("gqa", 0), ("varlen", 0), ("varlen", 2), ("long", 3)])
def test_bwd_cached_states_match_recompute(name, cp):
    """States written by the forward give the same gradients, bit for bit, as the backward's
    own forward pass (same segmentation on both sides), and match the oracle."""
    B, T, Hqk, Hv, h0, lengths = SMALL[name]
    x = make_inputs(B, T, Hqk, Hv, 128, 128, "bf16", seed=zlib.crc32(name.encode()) % 1000 + 7, h0_std=h0,
                    lengths=lengths, backward=True)
    d = to_dev(x)
    states = _fwd_states(d, cp_segment_chunks=cp)
    cached = _bwd(d, cp_segment_chunks=cp, states=states)
    recomputed = _bwd(d, cp_segment_chunks=cp)
    ref = oracle_bwd(x)
    for n in GRADS:
        assert torch.equal(cached[n], recomputed[n]), n
        assert_close(cached[n], ref[n], "bf16", f"{name} cached {n}")


def test_bwd_many_short_sequences():
    """260 packed sequences of 0..89 tokens (some empty), two v-heads: a gradient CTA's next item
    lies tens of sequences past its current one, so the scan over the chunk offsets that finds it
    takes several 32-sequence rounds and crosses empty sequences. All six gradients match the
    oracle; the forward's cache gives the recompute path's gradients bit for bit."""
    rng = np.random.default_rng(77)
    lengths = [int(v) for v in rng.integers(0, 90, size=260)]
    lengths[3] = lengths[140] = lengths[141] = 0
    x = make_inputs(1, 0, 1, 2, 128, 128, "bf16", seed=78, h0_std=0.1, lengths=lengths, backward=True)
    d = to_dev(x)
    recomputed = _bwd(d)
    cached = _bwd(d, states=_fwd_states(d))
    ref = oracle_bwd(x)
    for n in GRADS:
        assert torch.equal(cached[n], recomputed[n]), n
        assert_close(recomputed[n], ref[n], "bf16", f"many short sequences {n}")


def test_bwd_cached_states_from_exact_stitch():
    """Forward with the exact affine stitch writes its states from the final pass."""
    x = make_inputs(1, 0, 2, 2, 128, 128, "bf16", seed=41, h0_std=0.1, backward=True, lengths=[700, 64, 333])
    d = to_dev(x)
    states = _fwd_states(d, cp_segment_chunks=2, cp_exact=True)
    cached = _bwd(d, states=states)
    ref = oracle_bwd(x)
    for n in GRADS:
        assert_close(cached[n], ref[n], "bf16", f"exact-stitch cached {n}")


def test_bwd_cached_states_full_size():
    x = config_inputs("bwd_bf16")
    d = to_dev(x)
    states = _fwd_states(d)
    cached = _bwd(d, states=states)
    recomputed = _bwd(d)
    for n in GRADS:
        assert torch.equal(cached[n], recomputed[n]), n
