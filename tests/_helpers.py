"""Shared helpers of the GPU parity tests (comparison metrics, unit sampling)."""
import numpy as np
import torch

from oracle import as_f64, fwd_token, bwd_token

# Parity bars of the operator: bf16 I/O with fp32 accumulation, and fp32 I/O.
BF16_REL, BF16_ABS = 5e-3, 2e-2
F32_REL = 1e-4


def rel_l2(x, ref):
    x = as_f64(x).ravel()
    ref = as_f64(ref).ravel()
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (n if n > 0 else 1.0))


def max_abs(x, ref):
    x = as_f64(x).ravel()
    ref = as_f64(ref).ravel()
    return float(np.max(np.abs(x - ref))) if x.size else 0.0


def assert_close(x, ref, dtype, what):
    r = rel_l2(x, ref)
    if dtype == "bf16":
        a = max_abs(x, ref)
        assert r <= BF16_REL and a <= BF16_ABS, f"{what}: rel_l2={r:.3e} max_abs={a:.3e}"
    else:
        assert r <= F32_REL, f"{what}: rel_l2={r:.3e}"
    return r


def to_dev(x):
    out = {}
    for k, v in x.items():
        out[k] = v.cuda() if isinstance(v, torch.Tensor) else v
    return out


def unit_inputs(x, n, j):
    """Inputs of one (sequence n, v-head j) unit as a stand-alone B=1, Hqk=Hv=1 problem."""
    sh = x["shape"]
    hq = j // (sh["Hv"] // sh["Hqk"])
    if x["cu_seqlens"] is not None:
        cu = x["cu_seqlens"].tolist()
        b, s, e = 0, cu[n], cu[n + 1]
    else:
        b, s, e = n, 0, sh["T"]
    sl = lambda t, h: t[b:b + 1, s:e, h:h + 1]
    u = dict(q=sl(x["q"], hq), k=sl(x["k"], hq), v=sl(x["v"], j), g=x["g"][b:b + 1, s:e, j:j + 1],
             beta=x["beta"][b:b + 1, s:e, j:j + 1],
             h0=None if x["h0"] is None else x["h0"][n:n + 1, j:j + 1], scale=x["scale"])
    if "dO" in x:
        u["dO"] = sl(x["dO"], j)
        u["dhT"] = x["dhT"][n:n + 1, j:j + 1]
    return u, (b, s, e)


def oracle_unit_fwd(x, n, j):
    u, span = unit_inputs(x, n, j)
    o, hT = fwd_token(u["q"], u["k"], u["v"], u["g"], u["beta"], u["scale"], u["h0"])
    return o[0, :, 0], hT[0, 0], span


def oracle_unit_bwd(x, n, j):
    u, span = unit_inputs(x, n, j)
    gr = bwd_token(u["q"], u["k"], u["v"], u["g"], u["beta"], u["scale"], u["dO"], u["h0"],
                   u["dhT"])
    return gr, span
