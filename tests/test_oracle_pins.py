"""Pins for the fp64 oracle: each check ties the oracle to something other than itself.

Where a pin comes from:
  * golden index tables typed by hand from the readings of the HSTU blog,
    section 3.2 (relative attention bias) and the MTGR pages' mask rules;
  * special cases that reduce to library routines (numpy matmul, scipy expit,
    torch layer_norm in float64);
  * invariants of the method (causality, no row normalisation, jagged equals
    per-sequence, M-FALCON equals a candidate appended to its history, candidate
    permutation equivariance);
  * closed forms (one key; LayerNorm moments);
  * central finite differences (with Richardson extrapolation) of the forward
    for every backward output.
"""
import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
from hstu_jagged_pointwise_b200 import workloads as W

from conftest import read_golden


def silu_np(x):
    return x * expit(x)


def bf16_round(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


# ----------------------------------------------------------------------------
# index rules against hand-derived golden tables
# ----------------------------------------------------------------------------

def test_time_bucket_golden():
    for line in read_golden("time_buckets.txt"):
        ti, tj, want = (int(x) for x in line.split())
        m, pi, tb, po = oracle.indices([0, 2], [ti, tj], oracle.MASK_CAUSAL)
        # pair (1, 0) and (0, 1) both carry |ti - tj|
        assert tb[1 * 2 + 0] == want, (ti, tj, tb[2], want)
        assert tb[0 * 2 + 1] == want
        assert tb[0] == 0 and tb[3] == 0


def test_pos_index_golden():
    for line in read_golden("pos_index.txt"):
        kind, S, R, L, i, j, want = (int(x) for x in line.split())
        ts = np.arange(L, dtype=np.int64)
        ns = np.array([S], np.int32) if kind == 1 else None
        nr = np.array([R], np.int32) if kind == 1 else None
        m, pi, tb, po = oracle.indices([0, L], ts, kind, ns, nr)
        assert pi[i * L + j] == want, (line, pi[i * L + j])


def test_mtgr_mask_golden():
    rows = read_golden("mtgr_mask_8.txt")
    S = int(rows[0].split()[1])
    R = int(rows[1].split()[1])
    ts = np.array([int(x) for x in rows[2].split()[1:]], np.int64)
    want = np.array([[int(c) for c in r] for r in rows[3:]], np.uint8)
    L = len(ts)
    m, pi, tb, po = oracle.indices([0, L], ts, oracle.MASK_MTGR, [S], [R])
    np.testing.assert_array_equal(m.reshape(L, L), want)


def test_causal_mask_is_lower_triangle():
    L = 7
    m, _, _, _ = oracle.indices([0, L], np.arange(L), oracle.MASK_CAUSAL)
    np.testing.assert_array_equal(m.reshape(L, L), np.tril(np.ones((L, L), np.uint8)))


# ----------------------------------------------------------------------------
# forward: special cases that reduce to library routines
# ----------------------------------------------------------------------------

def _zero_rab(w):
    w.rab_pos = torch.zeros_like(w.rab_pos)
    w.rab_time = torch.zeros_like(w.rab_time)
    return w


def _dense_blocks(w, seq):
    s0, s1 = int(w.offsets[seq]), int(w.offsets[seq + 1])
    q = oracle.f32(w.q)[s0:s1].astype(np.float64)
    k = oracle.f32(w.k)[s0:s1].astype(np.float64)
    v = oracle.f32(w.v)[s0:s1].astype(np.float64)
    return s0, s1, q, k, v


def test_bidirectional_no_rab_equals_matmul_route():
    """All pairs visible (one static MTGR segment) and zero rab: Y = SiLU(Q K^T) V / alpha."""
    L = [9, 33]
    w = W.make_mtgr(n_profile=[2, 3], n_long=[7, 30], n_rt=[0, 0], n_cand=[0, 0], H=2, d=8,
                    dtype=torch.float32, seed=3, alpha=7.0)
    _zero_rab(w)
    y = oracle.attn_fwd(w)
    for b in range(2):
        s0, s1, q, k, v = _dense_blocks(w, b)
        for h in range(2):
            sl = slice(h * 8, (h + 1) * 8)
            want = silu_np(q[:, sl] @ k[:, sl].T) @ v[:, sl] / 7.0
            np.testing.assert_allclose(y[s0:s1, sl], want, rtol=1e-12, atol=1e-12)
    assert sum(L) == w.T


def test_bf16_operand_model_equals_matmul_route_with_torch_rounding():
    """The oracle's bf16 error model (used only for tolerances): all pairs visible, zero
    rab, so A = SiLU(Q K^T) and dz = (dY V^T / alpha) * SiLU'(Q K^T); with the model on,
    Y = bf16(A) V / alpha, dV = bf16(A)^T dY / alpha, dQ = bf16(dz) K, dK = bf16(dz)^T Q,
    and the rab gradients keep the unrounded dz.  bf16() here is torch's rounding."""
    w = W.make_mtgr(n_profile=[2], n_long=[30], n_rt=[0], n_cand=[0], H=1, d=8, dtype=torch.float32,
                    seed=13, alpha=5.0)
    _zero_rab(w)
    dy = np.random.default_rng(14).standard_normal((w.T, 8))
    with oracle.bf16_operands():
        y = oracle.attn_fwd(w)
        dq, dk, dv, drp, drt = oracle.attn_bwd(w, dy)
    q, k, v = (oracle.f32(t).astype(np.float64) for t in (w.q, w.k, w.v))
    s = q @ k.T
    a = bf16_round(silu_np(s)).astype(np.float64)
    sig = expit(s)
    dz = (dy @ v.T / 5.0) * (sig + s * sig * (1 - sig))
    dzb = bf16_round(dz).astype(np.float64)
    np.testing.assert_allclose(y, a @ v / 5.0, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dv, a.T @ dy / 5.0, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dq, dzb @ k, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dk, dzb.T @ q, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(drp.sum(), dz.sum(), rtol=1e-11)
    assert not np.allclose(a, silu_np(s), rtol=1e-6)          # the rounding really happened
    # and the model is off again outside the context
    np.testing.assert_allclose(oracle.attn_fwd(w), silu_np(s) @ v / 5.0, rtol=1e-12, atol=1e-12)


def test_causal_no_rab_equals_tril_matmul_route():
    w = _zero_rab(W.make_causal([1, 12, 40], H=3, d=16, dtype=torch.float32, seed=5, alpha=40.0))
    y = oracle.attn_fwd(w)
    for b in range(3):
        s0, s1, q, k, v = _dense_blocks(w, b)
        for h in range(3):
            sl = slice(h * 16, (h + 1) * 16)
            a = silu_np(q[:, sl] @ k[:, sl].T) * np.tril(np.ones((s1 - s0, s1 - s0)))
            np.testing.assert_allclose(y[s0:s1, sl], a @ v[:, sl] / 40.0, rtol=1e-12, atol=1e-12)


def test_single_key_closed_form():
    w = W.make_causal([1], H=1, d=32, dtype=torch.float32, seed=11, alpha=3.0)
    q, k, v = (oracle.f32(t)[0].astype(np.float64) for t in (w.q, w.k, w.v))
    z = q @ k + float(w.rab_pos[255]) + float(w.rab_time[0])
    np.testing.assert_allclose(oracle.attn_fwd(w)[0], z / (1 + np.exp(-z)) * v / 3.0, rtol=1e-13)


def test_rab_readout_matches_indices():
    """With Q = 0 the score is the bias alone; with one-hot V rows, Y reads out A.

    SiLU(0) = 0, so a one-hot table entry c lights exactly the pairs whose index
    equals that entry; those pairs must be the ones the index rules give."""
    L = 20
    lens = [L]
    for kind in ("causal", "mtgr"):
        if kind == "causal":
            w = W.make_causal(lens, H=1, d=L, dtype=torch.float32, seed=2, alpha=1.0)
        else:
            w = W.make_mtgr([2], [6], [4], [8], H=1, d=L, dtype=torch.float32, seed=2, alpha=1.0)
        w.q = torch.zeros_like(w.q)
        w.v = torch.eye(L, dtype=torch.float32)
        kind_id = 1 if kind == "mtgr" else 0
        m, pi, tb, _ = oracle.indices(w.offsets, w.ts, kind_id, w.n_static, w.n_realtime)
        m, pi, tb = m.reshape(L, L), pi.reshape(L, L), tb.reshape(L, L)
        c = 1.5
        for p in sorted(set(pi[m == 1].tolist()))[:6]:
            w.rab_pos = torch.zeros(511)
            w.rab_pos[p] = c
            w.rab_time = torch.zeros(64)
            a = oracle.attn_fwd(w)
            np.testing.assert_allclose(a, silu_np(c) * ((pi == p) & (m == 1)), atol=1e-15)
        for t in sorted(set(tb[m == 1].tolist()))[:6]:
            w.rab_pos = torch.zeros(511)
            w.rab_time = torch.zeros(64)
            w.rab_time[t] = c
            a = oracle.attn_fwd(w)
            np.testing.assert_allclose(a, silu_np(c) * ((tb == t) & (m == 1)), atol=1e-15)


# ----------------------------------------------------------------------------
# forward: invariants
# ----------------------------------------------------------------------------

def test_causal_prefix_invariance():
    w = W.make_causal([30], H=2, d=8, dtype=torch.float32, seed=7)
    y0 = oracle.attn_fwd(w)
    cut = 13
    for name in ("q", "k", "v"):
        t = getattr(w, name).clone()
        t[cut + 1:] = torch.randn(t[cut + 1:].shape)
        w2 = W.make_causal([30], H=2, d=8, dtype=torch.float32, seed=7)
        setattr(w2, name, t)
        w2.ts = w.ts.copy()
        w2.ts[cut + 1:] += 12345
        y1 = oracle.attn_fwd(w2)
        assert np.array_equal(y0[:cut + 1], y1[:cut + 1])
        assert not np.allclose(y0[cut + 1:], y1[cut + 1:])


def test_linear_in_v_and_alpha_scaling():
    w = W.make_mtgr([2], [5], [3], [4], H=2, d=8, dtype=torch.float32, seed=9, alpha=5.0)
    y = oracle.attn_fwd(w)
    w.v = w.v * 2
    np.testing.assert_array_equal(oracle.attn_fwd(w), 2 * y)
    w.v = w.v / 2
    w.alpha = 1.0
    np.testing.assert_allclose(oracle.attn_fwd(w) / 5.0, y, rtol=1e-15)


def test_not_row_normalised():
    """Pointwise aggregation: duplicating a key adds its contribution again, and
    the weights of a row do not sum to one (HSTU blog, section 3.1)."""
    Ls = 12
    w = W.make_mtgr([Ls], [0], [0], [0], H=1, d=8, dtype=torch.float32, seed=4, alpha=1.0)
    w.rab_pos = torch.full((511,), 0.3)   # position-free, so a duplicate is a true copy
    y_old = oracle.attn_fwd(w)
    j = 5
    # contribution of token j alone: zero all other values
    w_only = W.make_mtgr([Ls], [0], [0], [0], H=1, d=8, dtype=torch.float32, seed=4, alpha=1.0)
    w_only.rab_pos = w.rab_pos
    vj = torch.zeros_like(w.v)
    vj[j] = w.v[j]
    w_only.v = vj
    contrib = oracle.attn_fwd(w_only)
    # append a copy of token j
    w2 = W.make_mtgr([Ls + 1], [0], [0], [0], H=1, d=8, dtype=torch.float32, seed=4, alpha=1.0)
    for name in ("q", "k", "v", "u"):
        t = getattr(w, name)
        setattr(w2, name, torch.cat([t, t[j:j + 1]]))
    w2.ts = np.concatenate([w.ts, w.ts[j:j + 1]])
    w2.rab_pos, w2.rab_time = w.rab_pos, w.rab_time
    y_new = oracle.attn_fwd(w2)
    np.testing.assert_allclose(y_new[:Ls], y_old + contrib, rtol=1e-12, atol=1e-12)
    # weights do not sum to one
    w.v = torch.ones_like(w.v)
    s = oracle.attn_fwd(w)[:, 0]
    assert np.max(np.abs(s - 1.0)) > 0.5 and np.ptp(s) > 0.1


def test_jagged_equals_per_sequence_and_padded():
    lens = [5, 1, 17, 0, 9]
    w = W.make_causal(lens, H=2, d=8, dtype=torch.float32, seed=12, alpha=17.0)
    y = oracle.attn_fwd(w)
    Lmax = max(lens)
    # per sequence alone
    for b, L in enumerate(lens):
        if L == 0:
            continue
        s0 = int(w.offsets[b])
        wb = W.make_causal([L], H=2, d=8, dtype=torch.float32, seed=1, alpha=17.0)
        for name in ("q", "k", "v"):
            setattr(wb, name, getattr(w, name)[s0:s0 + L])
        wb.ts = w.ts[s0:s0 + L]
        wb.rab_pos, wb.rab_time = w.rab_pos, w.rab_time
        np.testing.assert_array_equal(oracle.attn_fwd(wb), y[s0:s0 + L])
    # padded to Lmax with garbage tails: valid rows unchanged
    wp = W.make_causal([Lmax] * len(lens), H=2, d=8, dtype=torch.float32, seed=99, alpha=17.0)
    ts_p = wp.ts.copy()
    for b, L in enumerate(lens):
        s0 = int(w.offsets[b])
        for name in ("q", "k", "v"):
            getattr(wp, name)[b * Lmax:b * Lmax + L] = getattr(w, name)[s0:s0 + L]
        ts_p[b * Lmax:b * Lmax + L] = w.ts[s0:s0 + L]
        if L < Lmax:
            ts_p[b * Lmax + L:(b + 1) * Lmax] = w.ts[s0 + L - 1] + np.arange(1, Lmax - L + 1) if L else 0
    wp.ts = ts_p
    wp.rab_pos, wp.rab_time = w.rab_pos, w.rab_time
    yp = oracle.attn_fwd(wp)
    for b, L in enumerate(lens):
        s0 = int(w.offsets[b])
        np.testing.assert_array_equal(yp[b * Lmax:b * Lmax + L], y[s0:s0 + L])


# ----------------------------------------------------------------------------
# M-FALCON
# ----------------------------------------------------------------------------

def test_mfalcon_equals_candidate_appended_to_history():
    wm = W.make_mfalcon([11, 300], [4, 3], H=2, d=8, dtype=torch.float32, seed=21)
    y = oracle.mfalcon(wm)
    for b in range(2):
        h0, h1 = int(wm.hist_offsets[b]), int(wm.hist_offsets[b + 1])
        n = h1 - h0
        for c in range(int(wm.cand_offsets[b]), int(wm.cand_offsets[b + 1])):
            wc = W.make_causal([n + 1], H=2, d=8, dtype=torch.float32, seed=1, alpha=wm.alpha)
            wc.q = torch.cat([torch.zeros(n, 16), wm.cand_q[c:c + 1]])
            wc.k = torch.cat([wm.hist_k[h0:h1], wm.cand_k[c:c + 1]])
            wc.v = torch.cat([wm.hist_v[h0:h1], wm.cand_v[c:c + 1]])
            wc.ts = np.concatenate([wm.hist_ts[h0:h1], wm.cand_ts[c:c + 1]])
            wc.rab_pos, wc.rab_time = wm.rab_pos, wm.rab_time
            yc = oracle.attn_fwd(wc, rows=[n])
            np.testing.assert_allclose(y[c], yc[0], rtol=1e-13, atol=1e-14)


def test_mfalcon_permutation_equivariance():
    wm = W.make_mfalcon([40], [9], H=2, d=8, dtype=torch.float32, seed=22)
    y = oracle.mfalcon(wm)
    perm = np.random.default_rng(0).permutation(9)
    for name in ("cand_q", "cand_k", "cand_v", "cand_u"):
        setattr(wm, name, getattr(wm, name)[torch.as_tensor(perm)])
    wm.cand_ts = wm.cand_ts[perm]
    np.testing.assert_array_equal(oracle.mfalcon(wm), y[perm])


def test_mtgr_candidates_reduce_to_mfalcon():
    """With no real-time tokens and every candidate after all history, an MTGR
    candidate row equals the M-FALCON score of that candidate."""
    n_prof, n_long, K = 3, 25, 6
    w = W.make_mtgr([n_prof], [n_long], [0], [K], H=2, d=8, dtype=torch.float32, seed=23, alpha=9.0)
    n = n_prof + n_long
    last = int(w.ts[n - 1])
    w.ts[n:] = last + 1 + np.arange(K) * 7
    y = oracle.attn_fwd(w)
    wm = W.make_mfalcon([n], [K], H=2, d=8, dtype=torch.float32, seed=1, alpha=9.0)
    wm.hist_k, wm.hist_v, wm.hist_ts = w.k[:n], w.v[:n], w.ts[:n]
    wm.cand_q, wm.cand_k, wm.cand_v, wm.cand_ts = w.q[n:], w.k[n:], w.v[n:], w.ts[n:]
    wm.rab_pos, wm.rab_time = w.rab_pos, w.rab_time
    np.testing.assert_allclose(oracle.mfalcon(wm), y[n:], rtol=1e-13, atol=1e-14)


def test_full_sequence_mfalcon_matches_cache_and_causal_history():
    """[history ; candidates] in one pass: candidate rows equal the cached M-FALCON
    scores (no timestamp filter: some candidates share the last history timestamp),
    history rows equal a causal layer over the history alone."""
    wm = W.make_mfalcon([0, 17, 130], [3, 5, 2], H=2, d=8, dtype=torch.float32, seed=24, alpha=131.0)
    ho = np.asarray(wm.hist_offsets)
    for b in range(len(ho) - 1):          # a candidate at the same second as the last history token
        if ho[b + 1] > ho[b]:
            wm.cand_ts[wm.cand_offsets[b]] = wm.hist_ts[ho[b + 1] - 1]
    ws = W.mfalcon_seq_from(wm, seed=3)
    y = oracle.attn_fwd(ws)
    off = np.asarray(ws.offsets)
    cand_rows = np.concatenate([np.arange(off[b] + ws.n_realtime[b], off[b + 1]) for b in range(len(off) - 1)])
    np.testing.assert_allclose(y[cand_rows], oracle.mfalcon(wm), rtol=1e-12, atol=1e-14)
    for b in range(len(off) - 1):
        n = int(ws.n_realtime[b])
        if n == 0:
            continue
        rows = slice(off[b], off[b] + n)
        wc = W.make_causal([n], H=2, d=8, dtype=torch.float32, seed=1, alpha=ws.alpha,
                           ts_list=[ws.ts[rows]])
        wc.q, wc.k, wc.v = ws.q[rows], ws.k[rows], ws.v[rows]
        wc.rab_pos, wc.rab_time = ws.rab_pos, ws.rab_time
        np.testing.assert_allclose(y[rows], oracle.attn_fwd(wc), rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------
# LayerNorm (.) U
# ----------------------------------------------------------------------------

def test_ln_mul_matches_torch_layer_norm():
    rng = np.random.default_rng(1)
    y = rng.normal(size=(37, 96)) * 3 + 1
    u = rng.normal(size=(37, 96)).astype(np.float32)
    g = (1 + 0.1 * rng.normal(size=96)).astype(np.float32)
    b = (0.1 * rng.normal(size=96)).astype(np.float32)
    o, mu, rs = oracle.ln_mul_fwd(y, u, g, b, 1e-5)
    ref = torch.nn.functional.layer_norm(torch.tensor(y), (96,), torch.tensor(g, dtype=torch.float64),
                                         torch.tensor(b, dtype=torch.float64), 1e-5)
    np.testing.assert_allclose(o, ref.numpy() * u, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(mu, y.mean(1), rtol=1e-12)
    np.testing.assert_allclose(rs, 1 / np.sqrt(y.var(1) + 1e-5), rtol=1e-12)


def test_ln_moments_closed_form():
    rng = np.random.default_rng(2)
    y = rng.normal(size=(5, 64)) * np.array([[0.01], [1], [10], [100], [0.001]])
    D = 64
    o, _, _ = oracle.ln_mul_fwd(y, np.ones((5, D), np.float32), np.ones(D, np.float32),
                                np.zeros(D, np.float32), 1e-5)
    var = y.var(1)
    np.testing.assert_allclose(o.mean(1), 0, atol=1e-12)
    np.testing.assert_allclose(o.var(1), var / (var + 1e-5), rtol=1e-10)


def _gln_case(seed=3, n=41, D=64, G=4):
    rng = np.random.default_rng(seed)
    y = rng.normal(size=(n, D)) * 2 + 0.5
    u = rng.normal(size=(n, D)).astype(np.float32)
    g = (1 + 0.1 * rng.normal(size=(G, D))).astype(np.float32)
    b = (0.1 * rng.normal(size=(G, D))).astype(np.float32)
    grp = rng.integers(0, G - 1, size=n).astype(np.uint8)   # group G-1 has no tokens
    grad = rng.normal(size=(n, D)).astype(np.float32)
    return y, u, g, b, grp, grad


def test_group_layer_norm_matches_torch_autograd():
    """Group LayerNorm against float64 torch autograd: F.layer_norm without affine, then the
    per-token rows gamma[group], beta[group]; the affine gradients come back to their groups."""
    y, u, g, b, grp, grad = _gln_case()
    o, mu, rs = oracle.gln_mul_fwd(y, u, g, b, grp, 1e-5)
    dy, du, dg, db = oracle.gln_mul_bwd(y, u, g, b, grp, grad, 1e-5)
    ty = torch.tensor(y, requires_grad=True)
    tu = torch.tensor(u, dtype=torch.float64, requires_grad=True)
    tg = torch.tensor(g, dtype=torch.float64, requires_grad=True)
    tb = torch.tensor(b, dtype=torch.float64, requires_grad=True)
    idx = torch.tensor(grp.astype(np.int64))
    ref = (torch.nn.functional.layer_norm(ty, (y.shape[1],), eps=1e-5) * tg[idx] + tb[idx]) * tu
    ref.backward(torch.tensor(grad, dtype=torch.float64))
    np.testing.assert_allclose(o, ref.detach().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dy, ty.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(du, tu.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dg, tg.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(db, tb.grad.numpy(), rtol=1e-10, atol=1e-11)
    assert not dg[-1].any() and not db[-1].any()            # the empty group gets exactly zero
    np.testing.assert_allclose(mu, y.mean(1), rtol=1e-12)


def test_group_layer_norm_with_equal_groups_is_layer_norm():
    y, u, g, b, grp, grad = _gln_case(seed=4)
    gs, bs = np.repeat(g[:1], len(g), 0), np.repeat(b[:1], len(b), 0)
    o, _, _ = oracle.gln_mul_fwd(y, u, gs, bs, grp, 1e-5)
    o1, _, _ = oracle.ln_mul_fwd(y, u, g[0], b[0], 1e-5)
    np.testing.assert_allclose(o, o1, rtol=1e-13, atol=1e-13)
    dy, du, dg, db = oracle.gln_mul_bwd(y, u, gs, bs, grp, grad, 1e-5)
    dy1, du1, dg1, db1 = oracle.ln_mul_bwd(y, u, g[0], b[0], grad, 1e-5)
    np.testing.assert_allclose(dy, dy1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(du, du1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dg.sum(0), dg1, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(db.sum(0), db1, rtol=1e-11, atol=1e-12)


def test_layer_norm_step_uses_each_tokens_group_row():
    """The layer's Norm step with token groups, against float64 torch autograd of layer_norm with
    each token's own affine row, applied to the oracle's attention output."""
    w = W.with_group_norm(W.make_causal([7, 20, 13], H=2, d=16, dtype=torch.float32, seed=21, with_grad=True),
                          seed=22, groups=3)
    y, o, _, _ = oracle.layer_fwd(w)
    ref = oracle.layer_bwd(w)
    ty = torch.tensor(np.asarray(y, dtype=np.float64))
    tu = torch.tensor(oracle.f32(w.u), dtype=torch.float64, requires_grad=True)
    tg = torch.tensor(oracle.f32(w.gamma), dtype=torch.float64, requires_grad=True)
    tb = torch.tensor(oracle.f32(w.beta), dtype=torch.float64, requires_grad=True)
    ty.requires_grad_(True)
    idx = torch.tensor(np.asarray(w.token_group).astype(np.int64))
    out = (torch.nn.functional.layer_norm(ty, (w.D,), eps=w.eps) * tg[idx] + tb[idx]) * tu
    out.backward(torch.tensor(oracle.f32(w.grad), dtype=torch.float64))
    np.testing.assert_allclose(o, out.detach().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ref["dy"], ty.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(ref["du"], tu.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(ref["dgamma"], tg.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(ref["dbeta"], tb.grad.numpy(), rtol=1e-10, atol=1e-11)


def test_mtgr_token_groups_follow_segments():
    w = W.with_group_norm(W.make_mtgr([3, 2], [5, 0], [2, 4], [3, 1], H=1, d=32, dtype=torch.float32, seed=5))
    np.testing.assert_array_equal(w.token_group, [0, 0, 0, 1, 1, 1, 1, 1, 2, 2, 3, 3, 3, 0, 0, 2, 2, 2, 2, 3])
    assert w.gamma.shape == (4, 32) and w.n_groups == 4


# ----------------------------------------------------------------------------
# projections: f1 (phi1 = SiLU, split U V Q K) and f2
# ----------------------------------------------------------------------------

def test_f1_split_order_and_silu_closed_form():
    """W1 made of four scaled identity blocks: block r of the output is SiLU(c_r x) in the
    order U, V, Q, K, with SiLU(z) = z * expit(z) from scipy."""
    T, D = 9, 16
    x = np.random.default_rng(6).normal(size=(T, D)).astype(np.float32)
    scales = [1.0, -2.0, 0.5, 3.0]
    w1 = np.concatenate([c * np.eye(D, dtype=np.float32) for c in scales])
    z, *blocks = oracle.f1_fwd(x, w1, None, D)
    for c, blk in zip(scales, blocks):
        ref = c * x.astype(np.float64)
        np.testing.assert_allclose(blk, ref * expit(ref), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(z[:, D:2 * D], -2.0 * x, rtol=0, atol=0)
    b1 = np.arange(4 * D, dtype=np.float32)
    z0, *_ = oracle.f1_fwd(np.zeros((2, D), np.float32), w1, b1, D)
    np.testing.assert_array_equal(z0, np.tile(b1, (2, 1)))


def test_f2_zero_weight_is_bias_plus_residual():
    rng = np.random.default_rng(7)
    o = rng.normal(size=(5, 32)).astype(np.float32)
    b2 = rng.normal(size=48).astype(np.float32)
    res = rng.normal(size=(5, 48)).astype(np.float32)
    out = oracle.f2_fwd(o, np.zeros((48, 32), np.float32), b2, res)
    np.testing.assert_allclose(out, b2.astype(np.float64) + res, rtol=0, atol=0)


def test_projection_gradients_match_torch_autograd():
    """f1 and f2 backward against float64 torch autograd of the forward definition."""
    w = W.make_projection(23, 48, 16, 40, seed=8, dtype=torch.float32)
    x = torch.tensor(w.x.numpy(), dtype=torch.float64, requires_grad=True)
    w1 = torch.tensor(w.w1.numpy(), dtype=torch.float64, requires_grad=True)
    b1 = torch.tensor(w.b1.numpy(), dtype=torch.float64, requires_grad=True)
    z = x @ w1.T + b1
    a = torch.nn.functional.silu(z)
    a.backward(torch.tensor(w.dact.numpy(), dtype=torch.float64))
    D = w.D
    zo, *_ = oracle.f1_fwd(w.x, w.w1, w.b1, D)
    dact = w.dact.numpy()
    dz, dx, dw1, db1 = oracle.f1_bwd(w.x, w.w1, zo, dact[:, :D], dact[:, D:2 * D], dact[:, 2 * D:3 * D],
                                     dact[:, 3 * D:])
    np.testing.assert_allclose(dx, x.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dw1, w1.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(db1, b1.grad.numpy(), rtol=1e-11, atol=1e-12)
    o = torch.tensor(w.o_pre.numpy(), dtype=torch.float64, requires_grad=True)
    w2 = torch.tensor(w.w2.numpy(), dtype=torch.float64, requires_grad=True)
    b2 = torch.tensor(w.b2.numpy(), dtype=torch.float64, requires_grad=True)
    (o @ w2.T + b2).backward(torch.tensor(w.g_out.numpy(), dtype=torch.float64))
    do, dw2, db2 = oracle.f2_bwd(w.o_pre, w.w2, w.g_out)
    np.testing.assert_allclose(do, o.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dw2, w2.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(db2, b2.grad.numpy(), rtol=1e-11, atol=1e-12)


# ----------------------------------------------------------------------------
# Stochastic Length sampler and token-balanced batches
# ----------------------------------------------------------------------------

def test_splitmix64_known_answers():
    rows = [r.split() for r in read_golden("splitmix64_seed1234567.txt")]
    n = np.array([int(a) for a, _ in rows], dtype=np.uint64)
    want = np.array([int(b) for _, b in rows], dtype=np.uint64)
    np.testing.assert_array_equal(oracle.splitmix64(1234567, n), want)


def test_sl_keeps_cap_events_in_order_and_short_rows_whole():
    lens = [776, 777, 4096, 5, 0, 1000]
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    new, idx = oracle.sl_sample(off, 776, seed=42)
    np.testing.assert_array_equal(np.diff(new), [776, 776, 776, 5, 0, 776])
    for b in range(len(lens)):
        g = idx[new[b]:new[b + 1]]
        assert np.all(np.diff(g) > 0)                                  # original order, no repeats
        assert np.all((g >= off[b]) & (g < off[b + 1]))
    np.testing.assert_array_equal(idx[new[0]:new[1]], np.arange(776))  # at the cap: untouched
    np.testing.assert_array_equal(idx[new[3]:new[4]], off[3] + np.arange(5))
    # the 777-event row drops exactly the event with the largest key
    keys = oracle.sl_keys(42, 1, 777)
    assert int(np.argmax(keys)) not in set((idx[new[1]:new[2]] - off[1]).tolist())


def test_sl_subset_is_uniform():
    """Each of L = 20 events is kept with probability cap / L = 1/4 (over 4000 seeds),
    and every 2-subset of positions appears with probability (5*4)/(20*19)."""
    L, cap, n = 20, 5, 4000
    off = np.array([0, L], np.int32)
    hits = np.zeros(L)
    pair = 0
    for s in range(n):
        _, idx = oracle.sl_sample(off, cap, seed=s)
        hits[idx] += 1
        pair += (0 in idx) and (19 in idx)
    p = cap / L
    sd = np.sqrt(n * p * (1 - p))
    assert np.all(np.abs(hits - n * p) < 5 * sd), hits
    p2 = cap * (cap - 1) / (L * (L - 1))
    assert abs(pair - n * p2) < 5 * np.sqrt(n * p2 * (1 - p2))


def test_pack_balanced_contiguous_and_balanced():
    rng = np.random.default_rng(10)
    lens = rng.integers(16, 4096, size=300)
    off = np.concatenate([[0], np.cumsum(lens)])
    start, tokens, weights = oracle.pack_balanced(off, 8)
    assert start[0] == 0 and start[-1] == 300 and np.all(np.diff(start) >= 0)
    assert tokens.sum() == off[-1]
    assert np.all(np.abs(tokens - off[-1] / 8) <= lens.max())          # within one sequence of even
    np.testing.assert_allclose(weights.sum(), 1.0)
    # equal lengths split into equal bins
    off_eq = np.arange(0, 65 * 100, 100)
    s2, t2, w2 = oracle.pack_balanced(off_eq, 4)
    np.testing.assert_array_equal(s2, [0, 16, 32, 48, 64])
    np.testing.assert_allclose(w2, 0.25)


def test_pack_balanced_worked_example():
    """Sequences of 10, 20, 5 and 65 tokens (T = 100) into 2 bins, worked by hand from the
    midpoint rule: midpoints 5, 20, 32.5 and 67.5 give bins floor(2 m / 100) = 0, 0, 0, 1."""
    start, tokens, weights = oracle.pack_balanced([0, 10, 30, 35, 100], 2)
    np.testing.assert_array_equal(start, [0, 3, 4])
    np.testing.assert_array_equal(tokens, [35, 65])
    np.testing.assert_allclose(weights, [0.75, 0.25])


def test_pack_balanced_weights_give_the_mean_over_sequences():
    """The weighted sum of per-bin mean gradients is the mean of the per-sequence gradients."""
    rng = np.random.default_rng(11)
    lens = rng.integers(1, 3000, size=97)
    off = np.concatenate([[0], np.cumsum(lens)])
    start, _, weights = oracle.pack_balanced(off, 8)
    g = rng.normal(size=(97, 5))
    total = sum(weights[r] * g[start[r]:start[r + 1]].mean(0) for r in range(8) if start[r + 1] > start[r])
    np.testing.assert_allclose(total, g.mean(0), rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------
# backward: central finite differences with Richardson extrapolation
# ----------------------------------------------------------------------------

def _loss(w):
    _, o, _, _ = oracle.layer_fwd(w)
    return float(np.sum(o * oracle.f32(w.grad).astype(np.float64)))


def _fd(w, arr, idx, h):
    x0 = arr[idx]
    arr[idx] = x0 + h
    fp = _loss(w)
    arr[idx] = x0 - h
    fm = _loss(w)
    arr[idx] = x0
    return (fp - fm) / (2 * h)


def _fd_rich(w, arr, idx):
    h = 2.0 ** -8
    d1 = _fd(w, arr, idx, h)
    d2 = _fd(w, arr, idx, h / 2)
    return (4 * d2 - d1) / 3


def _as_np_bf16(w):
    for name in ("q", "k", "v", "u", "grad"):
        setattr(w, name, bf16_round(oracle.f32(getattr(w, name))))
    w.rab_pos = bf16_round(oracle.f32(w.rab_pos) * 20)   # larger bias so its gradient matters
    w.rab_time = bf16_round(oracle.f32(w.rab_time) * 20)
    w.gamma = bf16_round(oracle.f32(w.gamma))
    w.beta = bf16_round(oracle.f32(w.beta))
    return w


@pytest.mark.parametrize("kind", ["causal", "mtgr"])
def test_backward_finite_differences(kind):
    if kind == "causal":
        w = W.make_causal([3, 6], H=2, d=4, dtype=torch.float32, seed=31, alpha=4.0,
                          random_affine=True, with_grad=True)
    else:
        w = W.make_mtgr([1, 2], [2, 2], [2, 1], [3, 2], H=2, d=4, dtype=torch.float32, seed=32,
                        alpha=4.0, random_affine=True, with_grad=True)
    w = _as_np_bf16(w)
    g = oracle.layer_bwd(w)
    rng = np.random.default_rng(0)
    checks = {"q": "dq", "k": "dk", "v": "dv", "u": "du"}
    for name, gname in checks.items():
        arr = getattr(w, name)
        for _ in range(12):
            idx = (rng.integers(arr.shape[0]), rng.integers(arr.shape[1]))
            num = _fd_rich(w, arr, idx)
            ana = g[gname][idx]
            assert abs(num - ana) <= 1e-7 + 1e-6 * np.abs(g[gname]).max(), (name, idx, num, ana)
    m, pi, tb, _ = oracle.indices(w.offsets, w.ts, 1 if kind == "mtgr" else 0, w.n_static, w.n_realtime)
    used_p = sorted(set(pi[m == 1].tolist()))
    used_t = sorted(set(tb[m == 1].tolist()))
    for p in used_p:
        num = _fd_rich(w, w.rab_pos, p)
        assert abs(num - g["d_rab_pos"][p]) <= 1e-7 + 1e-6 * np.abs(g["d_rab_pos"]).max(), (p, num)
    for t in used_t:
        num = _fd_rich(w, w.rab_time, t)
        assert abs(num - g["d_rab_time"][t]) <= 1e-7 + 1e-6 * np.abs(g["d_rab_time"]).max(), (t, num)
    # entries no pair uses have zero gradient
    unused = np.setdiff1d(np.arange(511), used_p)
    assert np.all(g["d_rab_pos"][unused] == 0)
    for c in range(w.D):
        num = _fd_rich(w, w.gamma, c)
        assert abs(num - g["dgamma"][c]) <= 1e-7 + 1e-6 * np.abs(g["dgamma"]).max()
        num = _fd_rich(w, w.beta, c)
        assert abs(num - g["dbeta"][c]) <= 1e-7 + 1e-6 * np.abs(g["dbeta"]).max()


def test_workload_shapes():
    w0 = W.tiny_fp32()
    assert list(w0.lengths) == [17, 64, 100, 255] and w0.alpha == 255.0 and w0.D == 64
    assert W.stochastic_length_cap(4096, 1.6) == 776
    # timestamps strictly increase within each sequence
    for b in range(w0.B):
        t = w0.ts[w0.offsets[b]:w0.offsets[b + 1]]
        assert np.all(np.diff(t) > 0)
