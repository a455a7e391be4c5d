"""Pins of the CPU fp64 oracle against facts that do not come from the oracle.

Each test below would fail for a plausible slip in the oracle (a dropped decay,
a wrong sign in the delta rule, a transposed state, a reversed cumsum, a
mis-indexed grouped head, a leaking sequence boundary, a wrong adjoint term).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import L2NORM_EPS, bwd_token, fwd_chunk, fwd_token, l2norm, unit_lower_inverse
from gated_deltanet_chunked_prefill_b200.workloads import make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b.ravel())
    return np.linalg.norm((a - b).ravel()) / (nb if nb > 0 else 1.0)


def small(B=1, T=37, Hqk=2, Hv=2, dk=8, dv=6, seed=0, h0=0.1, lengths=None, backward=False,
          dtype="f32", g_scale=1.0):
    return make_inputs(B, T, Hqk, Hv, dk, dv, dtype, seed, h0_std=h0, lengths=lengths,
                       backward=backward, g_scale=g_scale)


def call_fwd(f, x, **kw):
    return f(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"], x["cu_seqlens"], **kw)


# ---------------------------------------------------------------- forward pins
@pytest.mark.parametrize("chunk", [1, 5, 16, 32, 64])
@pytest.mark.parametrize("case", ["mha", "gqa", "varlen", "noh0", "weak_decay", "weak_decay_varlen"])
def test_token_and_chunked_forms_agree(chunk, case):
    # weak decay (g x 0.01): with the recipe's gates, chunk-form terms more than ~30 tokens apart
    # weigh less than the tolerance, so only mild decay pins the far end of each chunk
    if case == "mha":
        x = small(B=2, T=150, seed=1)
    elif case == "gqa":
        x = small(B=1, T=97, Hqk=2, Hv=4, seed=2)
    elif case == "varlen":
        x = small(B=1, Hqk=1, Hv=2, lengths=[5, 70, 1, 64, 33], seed=3)
    elif case == "weak_decay":
        x = small(B=2, T=150, Hqk=1, Hv=2, seed=5)
        x["g"] = x["g"] * 0.01
    elif case == "weak_decay_varlen":
        x = small(B=1, Hqk=1, Hv=2, lengths=[130, 1, 64, 97], seed=6)
        x["g"] = x["g"] * 0.01
    else:
        x = small(B=1, T=130, seed=4, h0=None)
    o1, h1 = call_fwd(fwd_token, x)
    o2, h2 = call_fwd(fwd_chunk, x, chunk=chunk)
    assert rel(o2, o1) <= 1e-10
    assert rel(h2, h1) <= 1e-10


def test_zero_inputs_give_zero():
    x = small(T=40, h0=None)
    z = torch.zeros_like
    o, h = fwd_token(x["q"], x["k"], x["v"], z(x["g"]), z(x["beta"]), x["scale"], None)
    assert np.all(o == 0) and np.all(h == 0)
    o, h = fwd_chunk(x["q"], x["k"], x["v"], z(x["g"]), z(x["beta"]), x["scale"], None, chunk=16)
    assert np.all(o == 0) and np.all(h == 0)


@pytest.mark.parametrize("form", ["token", "chunk"])
def test_single_unit_write_is_retrieved(form):
    dk, dv = 5, 3
    rng = np.random.default_rng(7)
    k = np.zeros((1, 1, 1, dk)); k[0, 0, 0, 2] = 1.0            # exact unit vector
    v = rng.standard_normal((1, 1, 1, dv))
    g = np.zeros((1, 1, 1)); b = np.ones((1, 1, 1))
    f = fwd_token if form == "token" else (lambda *a: fwd_chunk(*a, chunk=4))
    o, hT = f(k, k, v, g, b, 0.25, None)
    # S k = v exactly (h^T k with h = S^T), and with q = k: o = scale * v
    np.testing.assert_array_equal(hT[0, 0].T @ k[0, 0, 0], v[0, 0, 0])
    np.testing.assert_array_equal(o[0, 0, 0], 0.25 * v[0, 0, 0])


@pytest.mark.parametrize("form", ["token", "chunk"])
def test_decay_only_closed_form(form):
    x = small(B=1, T=45, Hqk=1, Hv=3, seed=11, h0=0.5)
    g = x["g"].double().numpy()
    f = fwd_token if form == "token" else (lambda *a: fwd_chunk(*a, chunk=16))
    o, hT = f(x["q"], x["k"], x["v"], x["g"], torch.zeros_like(x["beta"]), x["scale"], x["h0"])
    h0 = x["h0"].double().numpy()
    q = x["q"].double().numpy()
    G = np.cumsum(g[0], axis=0)                               # [T, Hv]
    for j in range(3):
        np.testing.assert_allclose(hT[0, j], math.exp(G[-1, j]) * h0[0, j], rtol=1e-13, atol=0)
        ref_o = x["scale"] * np.exp(G[:, j])[:, None] * (q[0, :, 0] @ h0[0, j])
        np.testing.assert_allclose(o[0, :, j], ref_o, rtol=1e-12, atol=1e-300)


def _exact_s_form(qs, ks, vs, ratios, betas, scale, S0):
    """Exact rational brute force of S_t = a_t S (I - b k k^T) + b v k^T, o = scale S q."""
    dv, dk = len(S0), len(S0[0])
    S = [row[:] for row in S0]
    outs = []
    for q, k, v, a, b in zip(qs, ks, vs, ratios, betas):
        M = [[(Fraction(int(i == j)) - b * k[i] * k[j]) for j in range(dk)] for i in range(dk)]
        S = [[a * sum(S[r][m] * M[m][c] for m in range(dk)) + b * v[r] * k[c]
              for c in range(dk)] for r in range(dv)]
        outs.append([scale * sum(S[r][c] * q[c] for c in range(dk)) for r in range(dv)])
    return outs, S


@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_tiny_exact_rational_brute_force(T):
    rng = np.random.default_rng(100 + T)
    dk, dv = 3, 2

    def fr(lo, hi, den):
        return Fraction(int(rng.integers(lo, hi)), den)
    qs = [[fr(-8, 9, 8) for _ in range(dk)] for _ in range(T)]
    ks = [[fr(-8, 9, 8) for _ in range(dk)] for _ in range(T)]
    vs = [[fr(-8, 9, 4) for _ in range(dv)] for _ in range(T)]
    ratios = [Fraction(int(rng.integers(1, 9)), 8) for _ in range(T)]   # exp(g) in (0, 1]
    betas = [Fraction(int(rng.integers(0, 9)), 8) for _ in range(T)]
    S0 = [[fr(-4, 5, 4) for _ in range(dk)] for _ in range(dv)]
    scale = Fraction(1, 2)
    outs, ST = _exact_s_form(qs, ks, vs, ratios, betas, scale, S0)

    f = lambda a: np.array(a, dtype=np.float64)
    q = f(qs)[None, :, None, :]; k = f(ks)[None, :, None, :]; v = f(vs)[None, :, None, :]
    g = np.log(f(ratios))[None, :, None]; b = f(betas)[None, :, None]
    h0 = f(S0).T[None, None]                                   # h = S^T
    for form in ("token", "chunk"):
        fn = fwd_token if form == "token" else (lambda *a: fwd_chunk(*a, chunk=3))
        o, hT = fn(q, k, v, g, b, 0.5, h0)
        np.testing.assert_allclose(o[0, :, 0], f([[float(c) for c in r] for r in outs]),
                                   rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(hT[0, 0], f([[float(c) for c in r] for r in ST]).T,
                                   rtol=1e-12, atol=1e-13)


def test_hand_worked_example():
    with open(os.path.join(GOLDEN, "worked_example_2x2_T3.json")) as fh:
        ex = json.load(fh)
    i = ex["inputs"]
    arr = lambda a: np.array(a, dtype=np.float64)
    q = arr(i["q"])[None, :, None]; k = arr(i["k"])[None, :, None]; v = arr(i["v"])[None, :, None]
    g = np.log(arr(i["exp_g"]))[None, :, None]; b = arr(i["beta"])[None, :, None]
    for fn in (fwd_token, lambda *a: fwd_chunk(*a, chunk=2)):
        o, hT = fn(q, k, v, g, b, i["scale"], None)
        np.testing.assert_allclose(o[0, :, 0], arr(ex["expected"]["o"]), rtol=0, atol=1e-14)
        np.testing.assert_allclose(hT[0, 0], arr(ex["expected"]["hT"]), rtol=0, atol=1e-14)


def test_affine_in_h0_and_linear_in_v_h0():
    d = 6
    x = small(B=1, T=75, Hqk=1, Hv=2, dk=d, dv=d, seed=21, h0=0.3)
    z = torch.zeros_like
    # Phi from the run with v = 0 and h0 = I (the segment transition used by context parallelism)
    eye = torch.eye(d, dtype=torch.float32).expand(1, 2, d, d).contiguous()
    _, Phi = fwd_token(x["q"], x["k"], z(x["v"]), x["g"], x["beta"], x["scale"], eye)
    _, c0 = fwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], None)
    _, hT = fwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"])
    h0 = x["h0"].double().numpy()
    for j in range(2):
        assert rel(hT[0, j], Phi[0, j] @ h0[0, j] + c0[0, j]) < 1e-12
    o1, h1 = fwd_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"], chunk=16)
    o2, h2 = fwd_chunk(x["q"], x["k"], 2 * x["v"].double(), x["g"], x["beta"], x["scale"],
                       2 * x["h0"].double(), chunk=16)
    assert rel(o2, 2 * o1) < 1e-13 and rel(h2, 2 * h1) < 1e-13


@pytest.mark.parametrize("t1", [1, 33, 64, 90])
def test_resume_from_final_state(t1):
    x = small(B=1, T=128, seed=31, h0=0.2)
    o, hT = call_fwd(fwd_token, x)
    sl = lambda a, s, e: a[:, s:e]
    oa, ha = fwd_chunk(sl(x["q"], 0, t1), sl(x["k"], 0, t1), sl(x["v"], 0, t1),
                       sl(x["g"], 0, t1), sl(x["beta"], 0, t1), x["scale"], x["h0"], chunk=16)
    ob, hb = fwd_chunk(sl(x["q"], t1, 128), sl(x["k"], t1, 128), sl(x["v"], t1, 128),
                       sl(x["g"], t1, 128), sl(x["beta"], t1, 128), x["scale"], ha, chunk=16)
    assert rel(np.concatenate([oa, ob], axis=1), o) < 1e-12
    assert rel(hb, hT) < 1e-12


def test_packed_equals_alone_and_no_leakage():
    lengths = [17, 64, 3, 100]
    x = small(B=1, Hqk=1, Hv=2, lengths=lengths, seed=41)
    o, hT = call_fwd(fwd_chunk, x, chunk=16)
    cu = x["cu_seqlens"].numpy()
    for n in range(len(lengths)):
        s, e = cu[n], cu[n + 1]
        sl = lambda a: a[:, s:e]
        oa, ha = fwd_token(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]), sl(x["beta"]),
                           x["scale"], x["h0"][n:n + 1])
        assert rel(o[:, s:e], oa) < 1e-12 and rel(hT[n], ha[0]) < 1e-12


def test_grouped_heads_equal_repeated_heads():
    x = small(B=1, T=50, Hqk=2, Hv=6, seed=51, backward=True)
    o, hT = call_fwd(fwd_token, x)
    rep = lambda a: a.repeat_interleave(3, dim=2)
    o2, h2 = fwd_token(rep(x["q"]), rep(x["k"]), x["v"], x["g"], x["beta"], x["scale"], x["h0"])
    assert rel(o, o2) < 1e-14 and rel(hT, h2) < 1e-14
    gr = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"], x["dhT"])
    gm = bwd_token(rep(x["q"]), rep(x["k"]), x["v"], x["g"], x["beta"], x["scale"], x["dO"],
                   x["h0"], x["dhT"])
    for name in ("dq", "dk"):
        summed = gm[name].reshape(1, 50, 2, 3, -1).sum(axis=3)
        assert rel(gr[name], summed) < 1e-13
    for name in ("dv", "dg", "dbeta", "dh0"):
        assert rel(gr[name], gm[name]) < 1e-13


def test_state_norm_bound():
    x = small(B=1, T=300, Hqk=1, Hv=2, dk=16, dv=16, seed=61, h0=1.0)
    o, hT = call_fwd(fwd_token, x)
    g = x["g"].double().numpy()[0]; b = x["beta"].double().numpy()[0]
    v = x["v"].double().numpy()[0]; k = x["k"].double().numpy()[0]
    h0 = x["h0"].double().numpy()[0]
    for j in range(2):
        # each step's map h -> e^g (I - b k k^T) h has spectral norm <= e^g for unit k, b in [0, 1]
        bound = np.exp(g[:, j].sum()) * np.linalg.norm(h0[j], 2)
        for t in range(300):
            bound += b[t, j] * np.linalg.norm(k[t, 0]) * np.linalg.norm(v[t, j]) * \
                np.exp(g[t + 1:, j].sum())
        assert np.linalg.norm(hT[0, j], 2) <= bound * (1 + 1e-12)


def test_unit_lower_inverse():
    rng = np.random.default_rng(71)
    L = np.tril(rng.standard_normal((9, 9)), -1) * 0.3
    A = unit_lower_inverse(L)
    np.testing.assert_allclose(A @ (np.eye(9) + L), np.eye(9), atol=1e-13)
    np.testing.assert_allclose(A, np.linalg.inv(np.eye(9) + L), atol=1e-12)


# ---------------------------------------------------------------- backward pins
def _loss(x, dO, dhT, **over):
    a = dict(q=x["q"], k=x["k"], v=x["v"], g=x["g"], beta=x["beta"], h0=x["h0"])
    a.update(over)
    o, hT = fwd_token(a["q"], a["k"], a["v"], a["g"], a["beta"], x["scale"], a["h0"], x["cu_seqlens"])
    return float(np.sum(o * dO) + np.sum(hT * dhT))


@pytest.mark.parametrize("case", ["gqa", "varlen"])
def test_backward_central_differences(case):
    if case == "gqa":
        x = small(B=1, T=6, Hqk=1, Hv=2, dk=3, dv=2, seed=81, backward=True, h0=0.5)
    else:
        x = small(B=1, Hqk=1, Hv=1, dk=3, dv=2, seed=82, backward=True, h0=0.5, lengths=[3, 1, 4])
    base = {n: x[n].double().numpy().copy() for n in ("q", "k", "v", "g", "beta", "h0")}
    dO = x["dO"].double().numpy(); dhT = x["dhT"].double().numpy()
    gr = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"],
                   x["dhT"], x["cu_seqlens"], ckpt=2)
    eps = 1e-6
    names = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", h0="dh0")
    for n, gname in names.items():
        fd = np.zeros_like(base[n])
        it = np.nditer(base[n], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            p = base[n].copy(); p[idx] += eps
            m = base[n].copy(); m[idx] -= eps
            fd[idx] = (_loss(x, dO, dhT, **{n: p}) - _loss(x, dO, dhT, **{n: m})) / (2 * eps)
        np.testing.assert_allclose(gr[gname], fd, rtol=1e-6, atol=1e-8, err_msg=n)


@pytest.mark.parametrize("g_factor", [1.0, 0.01])
def test_backward_directional_derivative(g_factor):
    x = small(B=2, T=40, Hqk=1, Hv=2, dk=5, dv=4, seed=91, backward=True)
    x["g"] = x["g"] * g_factor                  # 0.01: the adjoint carried back over all 40 tokens weighs in
    dO = x["dO"].double().numpy(); dhT = x["dhT"].double().numpy()
    gr = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"],
                   x["dhT"], ckpt=7)
    rng = np.random.default_rng(5)
    names = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", h0="dh0")
    base = {n: x[n].double().numpy() for n in names}
    dirs = {n: rng.standard_normal(base[n].shape) for n in names}
    eps = 1e-5
    lp = _loss(x, dO, dhT, **{n: base[n] + eps * dirs[n] for n in names})
    lm = _loss(x, dO, dhT, **{n: base[n] - eps * dirs[n] for n in names})
    fd = (lp - lm) / (2 * eps)
    an = sum(float(np.sum(gr[names[n]] * dirs[n])) for n in names)
    assert abs(fd - an) <= 1e-7 * max(1.0, abs(an))


def test_backward_single_token_closed_form():
    # T = 1, h0 = 0: o = scale * beta (k.q) v, hT = beta k v^T
    rng = np.random.default_rng(3)
    dk, dv = 4, 3
    q = rng.standard_normal(dk); k = rng.standard_normal(dk); v = rng.standard_normal(dv)
    b = 0.7; s = 0.5; g = -0.3
    do = rng.standard_normal(dv); dht = rng.standard_normal((dk, dv))
    gr = bwd_token(q[None, None, None], k[None, None, None], v[None, None, None],
                   np.full((1, 1, 1), g), np.full((1, 1, 1), b), s, do[None, None, None],
                   None, dht[None, None])
    kv = k @ q
    np.testing.assert_allclose(gr["dv"][0, 0, 0], s * b * kv * do + b * dht.T @ k, rtol=1e-13)
    np.testing.assert_allclose(gr["dq"][0, 0, 0], s * b * (v @ do) * k, rtol=1e-13)
    np.testing.assert_allclose(gr["dk"][0, 0, 0], s * b * (v @ do) * q + b * dht @ v, rtol=1e-13)
    np.testing.assert_allclose(gr["dbeta"][0, 0, 0], s * kv * (v @ do) + k @ dht @ v, rtol=1e-13)
    assert abs(gr["dg"][0, 0, 0]) == 0.0                       # h0 = 0: the decay acts on nothing
    # dh0 = e^g (I - b k k^T) (s q do^T + dht)
    dh = s * np.outer(q, do) + dht
    np.testing.assert_allclose(gr["dh0"][0, 0], np.exp(g) * (dh - b * np.outer(k, k @ dh)),
                               rtol=1e-12)


def test_backward_checkpoint_independent():
    x = small(B=1, T=53, Hqk=1, Hv=2, dk=4, dv=4, seed=95, backward=True)
    args = (x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"], x["dhT"])
    a = bwd_token(*args, ckpt=1)
    b = bwd_token(*args, ckpt=64)
    for n in a:
        assert rel(a[n], b[n]) < 1e-14


# ---------------------------------------------------------------- planted mistakes
# Each mutation plants a plausible slip in a copy of the oracle's source (on the
# CPU); the pins above must reject every one of them.
import inspect  # noqa: E402
import oracle.gdn_oracle as _orc  # noqa: E402

MUTATIONS = [
    ("fwd_chunk", "D = U - W @ h", "D = U + W @ h"),                          # sign of the state term
    ("fwd_chunk", "P = np.tril((Q @ K.T) * E)", "P = np.tril((Q @ K.T) * E, -1)"),  # drops the diagonal
    ("fwd_chunk", "h = np.exp(gam[n - 1]) * h + Kd.T @ D", "h = h + Kd.T @ D"),     # drops the decay
    ("fwd_chunk", "gam = np.cumsum(g[b, c0:c1, j])", "gam = np.cumsum(g[b, c0:c1, j][::-1])[::-1]"),
    ("fwd_chunk", "L = np.tril(bt[:, None] * (K @ K.T) * E, -1)",                 # drops terms > 40 tokens
     "L = np.tril(np.triu(bt[:, None] * (K @ K.T) * E, -40), -1)"),              # below the diagonal
    ("fwd_token", "o[b, t] = scale * np.einsum(\"hkv,hk->hv\", h, qt)",
     "o[b, t] = scale * np.einsum(\"hvk,hk->hv\", h, qt)"),                  # reads S^T instead of S
    ("fwd_token", "h *= np.exp(g[b, t])[:, None, None]", "h *= np.exp(-g[b, t])[:, None, None]"),
    ("bwd_token", "dkt -= ht @ dr", "dkt += ht @ dr"),
    ("bwd_token", "dh = np.exp(gh[t]) * dht", "dh = dht"),
]


def _mutant(fn_name, old, new):
    src = inspect.getsource(_orc)
    assert old in src, old
    ns = {}
    exec(compile(src.replace(old, new), "mutant", "exec"), ns)
    return ns


@pytest.mark.parametrize("fn_name,old,new", MUTATIONS)
def test_pins_reject_planted_mistakes(fn_name, old, new):
    m = _mutant(fn_name, old, new)
    x = small(B=1, T=70, Hqk=1, Hv=2, dk=4, dv=4, seed=99, backward=True)
    if fn_name == "bwd_token":
        gr = m["bwd_token"](x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"],
                            x["h0"], x["dhT"], ckpt=8)
        ok = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"],
                       x["h0"], x["dhT"], ckpt=8)
        # the directional finite difference pins the correct adjoint, not the mutant
        assert max(rel(gr[n], ok[n]) for n in ok) > 1e-6
        return
    if fn_name == "fwd_token":
        with open(os.path.join(GOLDEN, "worked_example_2x2_T3.json")) as fh:
            ex = json.load(fh)
        i = ex["inputs"]
        arr = lambda a: np.array(a, dtype=np.float64)
        o, hT = m["fwd_token"](arr(i["q"])[None, :, None], arr(i["k"])[None, :, None],
                               arr(i["v"])[None, :, None], np.log(arr(i["exp_g"]))[None, :, None],
                               arr(i["beta"])[None, :, None], i["scale"], None)
        assert rel(o[0, :, 0], arr(ex["expected"]["o"])) > 1e-6
        return
    o1, h1 = call_fwd(fwd_token, x)
    o2, h2 = call_fwd(m["fwd_chunk"], x, chunk=16)
    caught = rel(o2, o1) > 1e-6 or rel(h2, h1) > 1e-6
    # a slip in the far end of a chunk shows only with mild decay and full chunks (the weak-decay pin)
    xw = dict(x)
    xw["g"] = x["g"] * 0.01
    o1, h1 = call_fwd(fwd_token, xw)
    o2, h2 = call_fwd(m["fwd_chunk"], xw, chunk=64)
    assert caught or rel(o2, o1) > 1e-6 or rel(h2, h1) > 1e-6


# ---------------------------------------------------------------- q/k normalisation
def test_l2norm_closed_form():
    """|x / sqrt(s + eps)|^2 = s / (s + eps), the direction is kept, a zero row stays zero."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, 3, 16)) * rng.uniform(0.01, 10.0, (5, 3, 1))
    y = l2norm(x)
    s = np.sum(x * x, -1)
    np.testing.assert_allclose(np.sum(y * y, -1), s / (s + L2NORM_EPS), rtol=1e-14)
    np.testing.assert_allclose(y * np.sqrt(s + L2NORM_EPS)[..., None], x, rtol=1e-13)
    assert np.all(l2norm(np.zeros((2, 4))) == 0.0)


def _rescaled_rows(x, lo, hi, seed):
    """q and k with every (token, head) row multiplied by its own factor in [lo, hi] (fp64)."""
    rng = np.random.default_rng(seed)
    out = dict(x)
    for n in ("q", "k"):
        a = x[n].double().numpy() if hasattr(x[n], "double") else np.asarray(x[n], dtype=np.float64)
        out[n] = a * rng.uniform(lo, hi, a.shape[:-1] + (1,))
    return out


@pytest.mark.parametrize("form", [fwd_token, fwd_chunk])
def test_l2norm_forward_row_scale_invariance(form):
    """With the normalisation the outputs depend on each q/k row's direction only: rescaling every
    row by its own positive factor (norms 10..90, where eps moves the result by < 1e-8) leaves o
    and hT unchanged, and with unit rows the result is the plain one up to eps / 2."""
    x = small(B=1, Hqk=1, Hv=2, dk=6, dv=5, seed=61, lengths=[20, 9, 33])
    a = _rescaled_rows(x, 10.0, 30.0, 1)
    b = _rescaled_rows(x, 40.0, 90.0, 2)
    oa, ha = call_fwd(form, a, qk_l2norm=True)
    ob, hb = call_fwd(form, b, qk_l2norm=True)
    assert rel(oa, ob) < 1e-7 and rel(ha, hb) < 1e-7
    o0, h0 = call_fwd(form, x)                  # rows already of unit norm
    assert rel(oa, o0) < 2e-6 and rel(ha, h0) < 2e-6
    assert rel(call_fwd(form, a)[0], o0) > 1.0  # without it the rescaling shows


def test_l2norm_forms_agree():
    x = small(B=2, T=45, Hqk=1, Hv=2, dk=6, dv=4, seed=62)
    a = _rescaled_rows(x, 0.3, 5.0, 3)
    o1, h1 = call_fwd(fwd_token, a, qk_l2norm=True)
    o2, h2 = call_fwd(fwd_chunk, a, qk_l2norm=True, chunk=16)
    assert rel(o2, o1) < 1e-10 and rel(h2, h1) < 1e-10


def _loss_raw(x, dO, dhT, **over):
    a = {n: x[n] for n in ("q", "k", "v", "g", "beta", "h0")}
    a.update(over)
    o, hT = fwd_token(a["q"], a["k"], a["v"], a["g"], a["beta"], x["scale"], a["h0"], x["cu_seqlens"],
                      qk_l2norm=True)
    return float(np.sum(o * dO) + np.sum(hT * dhT))


def test_l2norm_backward_central_differences():
    """Gradients with respect to the raw q and k, through the normalisation, against central
    differences of <o, dO> + <hT, dhT> (grouped values: dq, dk sum over the v-heads)."""
    x = small(B=1, T=7, Hqk=1, Hv=2, dk=3, dv=2, seed=83, backward=True, h0=0.5)
    x = _rescaled_rows(x, 0.5, 3.0, 4)
    dO = x["dO"].double().numpy(); dhT = x["dhT"].double().numpy()
    gr = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"], x["dhT"],
                   ckpt=3, qk_l2norm=True)
    eps = 1e-6
    for n, gname in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("beta", "dbeta"), ("h0", "dh0")):
        base = x[n].double().numpy() if hasattr(x[n], "double") else np.asarray(x[n], dtype=np.float64)
        fd = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            p = base.copy(); p[idx] += eps
            m = base.copy(); m[idx] -= eps
            fd[idx] = (_loss_raw(x, dO, dhT, **{n: p}) - _loss_raw(x, dO, dhT, **{n: m})) / (2 * eps)
        np.testing.assert_allclose(gr[gname], fd, rtol=1e-6, atol=1e-8, err_msg=n)


def test_l2norm_gradients_orthogonal_to_rows():
    """A function of x / |x| does not change along x: each raw row's gradient is orthogonal to the
    row (up to the eps term, relative eps / |x|^2)."""
    x = small(B=1, T=40, Hqk=1, Hv=2, dk=8, dv=4, seed=84, backward=True)
    x = _rescaled_rows(x, 2.0, 5.0, 5)
    gr = bwd_token(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"], x["dhT"],
                   qk_l2norm=True)
    for n, gname in (("q", "dq"), ("k", "dk")):
        a = np.asarray(x[n])
        dot = np.abs(np.sum(a * gr[gname], -1))
        scale_ = np.linalg.norm(a, axis=-1) * np.linalg.norm(gr[gname], axis=-1)
        assert np.all(dot <= 1e-6 * scale_ + 1e-15), n
        assert np.max(scale_) > 0


L2_MUTATIONS = [
    ("_l2norm_adjoint", "return r * (dxn - xn * np.sum(xn * dxn, axis=-1, keepdims=True))",
     "return r * dxn"),                                                       # drops the projection
    ("_l2norm_adjoint", "return r * (dxn - xn * np.sum(xn * dxn, axis=-1, keepdims=True))",
     "return dxn - xn * np.sum(xn * dxn, axis=-1, keepdims=True)"),           # drops the 1 / |x|
    ("fwd_chunk", "    if qk_l2norm:\n        q, k = l2norm(q), l2norm(k)\n    B, T, Hqk, dk = q.shape\n"
                  "    Hv, dv = v.shape[2], v.shape[3]\n    hm = qk_head_of(Hqk, Hv)\n"
                  "    spans = sequences(B, T, cu_seqlens)\n    o = np.zeros((B, T, Hv, dv))\n"
                  "    hT = np.zeros((len(spans), Hv, dk, dv))\n    for n_seq",
     "    if qk_l2norm:\n        q = l2norm(q)\n    B, T, Hqk, dk = q.shape\n"
     "    Hv, dv = v.shape[2], v.shape[3]\n    hm = qk_head_of(Hqk, Hv)\n"
     "    spans = sequences(B, T, cu_seqlens)\n    o = np.zeros((B, T, Hv, dv))\n"
     "    hT = np.zeros((len(spans), Hv, dk, dv))\n    for n_seq"),           # k left unnormalised
    ("l2norm", "return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)",
     "return x / np.sqrt(np.sum(x * x, axis=-2, keepdims=True) + eps)"),      # wrong axis
]


@pytest.mark.parametrize("fn_name,old,new", L2_MUTATIONS)
def test_l2norm_pins_reject_planted_mistakes(fn_name, old, new):
    m = _mutant(fn_name, old, new)
    if fn_name == "_l2norm_adjoint":
        x = _rescaled_rows(small(B=1, T=30, Hqk=1, Hv=2, dk=4, dv=4, seed=98, backward=True), 0.5, 3.0, 6)
        args = (x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dO"], x["h0"], x["dhT"])
        gr = m["bwd_token"](*args, qk_l2norm=True)
        ok = bwd_token(*args, qk_l2norm=True)         # pinned by the finite differences above
        assert max(rel(gr[n], ok[n]) for n in ("dq", "dk")) > 1e-6
        return
    x = small(B=1, Hqk=1, Hv=2, dk=6, dv=5, seed=61, lengths=[20, 9, 33])
    a = _rescaled_rows(x, 10.0, 30.0, 1)
    b = _rescaled_rows(x, 40.0, 90.0, 2)
    oa, ha = call_fwd(m["fwd_chunk"], a, qk_l2norm=True)
    ob, hb = call_fwd(m["fwd_chunk"], b, qk_l2norm=True)
    assert rel(oa, ob) > 1e-6 or rel(ha, hb) > 1e-6   # the row-scale invariance pin rejects it
