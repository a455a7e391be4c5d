"""CPU fp64 oracle for the Gated DeltaNet (GDN) chunked-prefill operator.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links
this module: only the tests, the smoke check and the CPU-baseline leg of the
benchmark use it. It shares no code with the CUDA library.

What it computes (the GDN recurrence; the pages "Qwen's FlashQLA targets the
expensive bit of long-context AI" (What happened) and "FlashQLA resource"
(section 2, the "What it serves" row) name the operator, GDN chunked prefill,
forward and backward; the recurrence itself is the operator's definition):

    S_t = exp(g_t) * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
    o_t = scale * S_t q_t

S is dv x dk. The oracle keeps its transpose h = S^T (dk x dv), which is also the
layout of the h0 / hT tensors [N, Hv, dk, dv]. With h = S^T one token step is

    h~  = exp(g_t) h                    (decay first)
    r   = v_t - h~^T k_t                (delta-rule residual)
    h   = h~ + beta_t k_t r^T           (rank-1 write)
    o_t = scale * h^T q_t               (read after the write)

Readings taken where the operator definition leaves a step open (each is the
plainest one the formula supports):
  * g is the raw per-token log-decay; the operator forms the cumulative sums.
  * q and k are used as given (normalisation belongs to the input recipe), unless
    qk_l2norm asks for the in-operator normalisation below.
  * grouped values: v-head j reads q/k head j // (Hv // Hqk).
  * packed sequences: cu_seqlens = [0, cumsum(lengths)], B == 1; h0 / hT are
    per sequence. Sequences never interact.
  * all arithmetic in fp64 on the exact (upcast) input values.

Three independent forms:
  fwd_token   -- the recurrence above, token by token (the reference semantics)
  fwd_chunk   -- the chunk-parallel (WY/UT) algebra, written out from the
                 recurrence, with the unit-lower-triangular inverse by forward
                 substitution; chunk size is a parameter
  bwd_token   -- the exact adjoint of fwd_token, token by token in reverse

Optional q/k normalisation (qk_l2norm=True on every form): rows of q and k become
x / sqrt(|x|^2 + 1e-6) before the recurrence, and the backward maps the gradients back
through that normalisation to the raw q and k.

Pins (tests/test_oracle.py): the token and chunked forms agree to 1e-10 for
every chunk size; beta=0, g=0, h0=0 gives zero; a single unit-norm write is
retrieved exactly; decay-only inputs follow the closed form; tiny cases match
exact rational brute force of the S-form with explicit matrices; the affine
map in h0, linearity, resume, packed-vs-alone, a hand-derived worked example,
and the backward against central finite differences and closed forms. The
normalisation: the squared row norm s / (s + eps) in closed form, invariance of
the outputs to a positive rescaling of each row, the gradients orthogonal to
their rows, and central finite differences through it.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "as_f64", "sequences", "qk_head_of", "fwd_token", "fwd_chunk", "bwd_token",
    "unit_lower_inverse", "l2norm", "L2NORM_EPS",
]

# Optional normalisation of q and k inside the operator (the flash-linear-attention entry point's
# use_qk_l2norm_in_kernel, which the pages say the library's entry signature follows): every
# row x (one token of one q/k head) becomes x / sqrt(|x|^2 + eps). The pages fix no eps; 1e-6
# keeps an all-zero row at zero instead of dividing by zero.
L2NORM_EPS = 1e-6


def l2norm(x, eps=L2NORM_EPS):
    """Rows of x (last axis) divided by sqrt(sum of squares + eps), in fp64."""
    x = as_f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def as_f64(x):
    """Exact upcast of a tensor/array (any float dtype) to a float64 numpy array."""
    if x is None:
        return None
    if hasattr(x, "detach"):               # torch tensor (bf16 has no numpy view)
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def sequences(B, T, cu_seqlens):
    """List of (batch row, start, end) spans: one per batch row, or per packed sequence."""
    if cu_seqlens is None:
        return [(b, 0, T) for b in range(B)]
    cu = [int(c) for c in np.asarray(cu_seqlens).reshape(-1)]
    if B != 1:
        raise ValueError("packed sequences require B == 1")
    return [(0, cu[i], cu[i + 1]) for i in range(len(cu) - 1)]


def qk_head_of(Hqk, Hv):
    """q/k head read by each v-head (consecutive v-heads share one q/k head)."""
    if Hv % Hqk != 0:
        raise ValueError("Hv must be a multiple of Hqk")
    return np.arange(Hv) // (Hv // Hqk)


def _unpack(q, k, v, g, beta, h0):
    q, k, v, g, beta, h0 = (as_f64(a) for a in (q, k, v, g, beta, h0))
    return q, k, v, g, beta, h0


# --------------------------------------------------------------------------
# token recurrence
# --------------------------------------------------------------------------
def fwd_token(q, k, v, g, beta, scale, h0=None, cu_seqlens=None, qk_l2norm=False):
    """Token-by-token recurrence.

    q, k: [B,T,Hqk,dk]; v: [B,T,Hv,dv]; g, beta: [B,T,Hv]; h0: [N,Hv,dk,dv] or None.
    Returns (o [B,T,Hv,dv], hT [N,Hv,dk,dv]) in fp64. Vectorised over heads only;
    every token is one step of the recurrence in the module docstring. qk_l2norm: q and k
    rows are normalised first (l2norm).
    """
    q, k, v, g, beta, h0 = _unpack(q, k, v, g, beta, h0)
    if qk_l2norm:
        q, k = l2norm(q), l2norm(k)
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    hm = qk_head_of(Hqk, Hv)
    spans = sequences(B, T, cu_seqlens)
    o = np.zeros((B, T, Hv, dv))
    hT = np.zeros((len(spans), Hv, dk, dv))
    for n, (b, s, e) in enumerate(spans):
        h = np.zeros((Hv, dk, dv)) if h0 is None else h0[n].copy()
        for t in range(s, e):
            kt = k[b, t, hm]                               # [Hv, dk]
            qt = q[b, t, hm]
            h *= np.exp(g[b, t])[:, None, None]            # h~ = e^g h
            r = v[b, t] - np.einsum("hkv,hk->hv", h, kt)   # r = v - h~^T k
            h += beta[b, t][:, None, None] * kt[:, :, None] * r[:, None, :]
            o[b, t] = scale * np.einsum("hkv,hk->hv", h, qt)
        hT[n] = h
    return o, hT


# --------------------------------------------------------------------------
# chunked (WY / UT) form
# --------------------------------------------------------------------------
def unit_lower_inverse(L):
    """(I + L)^-1 for strictly-lower-triangular L, by forward substitution.

    Row i of A = (I + L)^-1 satisfies A_i = e_i - sum_{j<i} L_ij A_j.
    """
    n = L.shape[0]
    A = np.zeros((n, n))
    for i in range(n):
        A[i, i] = 1.0
        for j in range(i):
            A[i] -= L[i, j] * A[j]
    return A


def fwd_chunk(q, k, v, g, beta, scale, h0=None, cu_seqlens=None, chunk=64, qk_l2norm=False):
    """Chunk-parallel form of the same recurrence.

    For each sequence, v-head and chunk of n <= `chunk` tokens, with h the state
    at the chunk start (dk x dv) and local positions i = 1..n:
        gam_i = sum_{j<=i} g_j                       (chunk-local inclusive cumsum)
        E_ij  = exp(gam_i - gam_j)
        L     = strict_lower( diag(beta) K K^T * E )
        A     = (I + L)^-1
        W     = A diag(beta exp(gam)) K,   U = A diag(beta) V
        D     = U - W h                            (per-token residuals times beta)
        O     = scale [ diag(exp(gam)) Q h + (Q K^T * E * lower_incl) D ]
        h'    = exp(gam_n) h + (diag(exp(gam_n - gam)) K)^T D
    Chunks never cross a sequence boundary; the last chunk may be partial. qk_l2norm: q and k
    rows are normalised first (l2norm).
    """
    q, k, v, g, beta, h0 = _unpack(q, k, v, g, beta, h0)
    if qk_l2norm:
        q, k = l2norm(q), l2norm(k)
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    hm = qk_head_of(Hqk, Hv)
    spans = sequences(B, T, cu_seqlens)
    o = np.zeros((B, T, Hv, dv))
    hT = np.zeros((len(spans), Hv, dk, dv))
    for n_seq, (b, s, e) in enumerate(spans):
        for j in range(Hv):
            a = hm[j]
            h = np.zeros((dk, dv)) if h0 is None else h0[n_seq, j].copy()
            for c0 in range(s, e, chunk):
                c1 = min(c0 + chunk, e)
                n = c1 - c0
                Q = q[b, c0:c1, a]
                K = k[b, c0:c1, a]
                V = v[b, c0:c1, j]
                bt = beta[b, c0:c1, j]
                gam = np.cumsum(g[b, c0:c1, j])
                E = np.exp(gam[:, None] - gam[None, :])
                L = np.tril(bt[:, None] * (K @ K.T) * E, -1)
                A = unit_lower_inverse(L)
                W = A @ ((bt * np.exp(gam))[:, None] * K)
                U = A @ (bt[:, None] * V)
                D = U - W @ h
                P = np.tril((Q @ K.T) * E)
                o[b, c0:c1, j] = scale * (np.exp(gam)[:, None] * (Q @ h) + P @ D)
                Kd = np.exp(gam[n - 1] - gam)[:, None] * K
                h = np.exp(gam[n - 1]) * h + Kd.T @ D
            hT[n_seq, j] = h
    return o, hT


# --------------------------------------------------------------------------
# token adjoint (backward)
# --------------------------------------------------------------------------
def _head_forward_states(qh, kh, vh, gh, bh, h_init, ckpt):
    """States at every `ckpt`-th token boundary of one (sequence, v-head) run."""
    Tn = kh.shape[0]
    saved = {0: h_init.copy()}
    h = h_init.copy()
    for t in range(Tn):
        h *= np.exp(gh[t])
        r = vh[t] - h.T @ kh[t]
        h += bh[t] * np.outer(kh[t], r)
        if (t + 1) % ckpt == 0:
            saved[t + 1] = h.copy()
    return saved, h


def _l2norm_adjoint(x, dxn, eps=L2NORM_EPS):
    """Gradient with respect to the raw rows x of a function of xn = l2norm(x), given its
    gradient dxn with respect to xn: with r = (|x|^2 + eps)^(-1/2), xn = r x and
    d xn / d x = r (I - xn xn^T), so dx = r (dxn - xn <xn, dxn>), row by row."""
    r = 1.0 / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)
    xn = r * x
    return r * (dxn - xn * np.sum(xn * dxn, axis=-1, keepdims=True))


def bwd_token(q, k, v, g, beta, scale, dO, h0=None, dhT=None, cu_seqlens=None, ckpt=64, qk_l2norm=False):
    """Exact adjoint of fwd_token, in reverse token order.

    Per token, with dh the adjoint of h_t carried from later tokens:
        dh  += scale q_t do_t^T;     dq_t = scale h_t do_t
        dbeta_t = k_t^T dh r_t;      dk_t = beta_t dh r_t;   dr = beta_t dh^T k_t
        dv_t = dr;                   dh~ = dh - k_t dr^T;    dk_t -= h~_t dr
        dg_t = <dh~, h~_t>;          dh <- exp(g_t) dh~      (adjoint of h_{t-1})
    dh starts at dhT (or 0) and ends as dh0. Grouped values: dq and dk of a q/k
    head are the sums over the v-heads that read it. Forward states are kept at
    every `ckpt` tokens and recomputed in between (memory, not arithmetic).
    Returns dict dq, dk [B,T,Hqk,dk]; dv [B,T,Hv,dv]; dg, dbeta [B,T,Hv];
    dh0 [N,Hv,dk,dv] (fp64). qk_l2norm: the recurrence runs on l2norm(q), l2norm(k), and the
    returned dq, dk are taken with respect to the raw q, k through that normalisation.
    """
    q, k, v, g, beta, h0 = _unpack(q, k, v, g, beta, h0)
    if qk_l2norm:
        q_raw, k_raw = q, k
        q, k = l2norm(q), l2norm(k)
    dO = as_f64(dO)
    dhT = as_f64(dhT)
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    hm = qk_head_of(Hqk, Hv)
    spans = sequences(B, T, cu_seqlens)
    dq = np.zeros_like(q)
    dkk = np.zeros_like(k)
    dvv = np.zeros_like(v)
    dg = np.zeros_like(g)
    db = np.zeros_like(beta)
    dh0 = np.zeros((len(spans), Hv, dk, dv))
    for n_seq, (b, s, e) in enumerate(spans):
        for j in range(Hv):
            a = hm[j]
            qh, kh, vh = q[b, s:e, a], k[b, s:e, a], v[b, s:e, j]
            gh, bh, doh = g[b, s:e, j], beta[b, s:e, j], dO[b, s:e, j]
            h_init = np.zeros((dk, dv)) if h0 is None else h0[n_seq, j]
            saved, _ = _head_forward_states(qh, kh, vh, gh, bh, h_init, ckpt)
            dh = np.zeros((dk, dv)) if dhT is None else dhT[n_seq, j].copy()
            Tn = e - s
            for blk in range((Tn - 1) // ckpt * ckpt if Tn else 0, -1, -ckpt):
                if blk >= Tn:
                    continue
                # recompute h~_t, r_t, h_t for the tokens of this block
                h = saved[blk].copy()
                hts, htil, rs = [], [], []
                for t in range(blk, min(blk + ckpt, Tn)):
                    ht = np.exp(gh[t]) * h
                    r = vh[t] - ht.T @ kh[t]
                    h = ht + bh[t] * np.outer(kh[t], r)
                    htil.append(ht)
                    rs.append(r)
                    hts.append(h)
                for i in range(len(hts) - 1, -1, -1):
                    t = blk + i
                    ht, r, h_t = htil[i], rs[i], hts[i]
                    dh += scale * np.outer(qh[t], doh[t])
                    dq[b, s + t, a] += scale * (h_t @ doh[t])
                    db[b, s + t, j] = kh[t] @ dh @ r
                    dkt = bh[t] * (dh @ r)
                    dr = bh[t] * (dh.T @ kh[t])
                    dvv[b, s + t, j] = dr
                    dht = dh - np.outer(kh[t], dr)
                    dkt -= ht @ dr
                    dkk[b, s + t, a] += dkt
                    dg[b, s + t, j] = np.sum(dht * ht)
                    dh = np.exp(gh[t]) * dht
            dh0[n_seq, j] = dh
    if qk_l2norm:
        dq, dkk = _l2norm_adjoint(q_raw, dq), _l2norm_adjoint(k_raw, dkk)
    return dict(dq=dq, dk=dkk, dv=dvv, dg=dg, dbeta=db, dh0=dh0)
