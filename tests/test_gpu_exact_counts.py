"""Exact tests of the integer decisions inside the production bf16 tcgen05 kernels.

The mask, the relative-position index pidx and the time bucket tb (Meta HSTU blog,
section 3.2; MTGR deep-dive section 2 and MTGR report section 3.1 for the dynamic
mixed mask; HSTU blog section 4.2 for the full-sequence M-FALCON mask) are decided in
several fast paths of the fused kernels: constant-bias blocks, rows of 64 biases
indexed by j - i or by j, per-element time buckets, one-of-two buckets, fully masked
blocks and the element-by-element rules at ragged edges.  These tests make those
kernels compute integers, so that every decision is compared with the oracle's
(oracle.indices) bit for bit:

  * Q.K = 0 and bias tables of +-100, so z is exactly +100 or -100 on every pair.
    The kernels' SiLU gives exactly 100 and 0 there (and 2 SiLU'(z) exactly 2 and 0).
  * V row j is the one-hot vector e_(j mod d), so Y_i[r] * alpha / 100 counts the
    visible keys j == r (mod d) whose bias is +100: an integer, recovered by rounding
    (bf16 keeps it within 1/8 of the integer for the sizes here).
  * Backward (hstu_attn_bwd_dy, from dL/dY): dY row i = e_(i mod d), and Q or K one-hot,
    so dQ, dK, dV and the bias-table gradients are counts too (alpha a power of two).

The bias tables are +100 on a seeded random half of the entries and -100 on the
rest, in several draws: a pair whose pidx or tb the kernel got wrong moves a count
whenever the two entries differ, which is half of the draws.
"""
import numpy as np
import pytest
import torch

import oracle
from hstu_jagged_pointwise_b200 import ops
from hstu_jagged_pointwise_b200 import workloads as W
from parity import dev

pytestmark = pytest.mark.gpu

ALPHA = 1024.0      # a power of two: every scaling below is exact
ZV = 100.0          # |z| on every pair
N_DRAWS = 4         # random sign patterns per table


# ----------------------------------------------------------------------------
# inputs
# ----------------------------------------------------------------------------

def _local_index(offsets):
    off = np.asarray(offsets, np.int64)
    return np.concatenate([np.arange(off[b + 1] - off[b]) for b in range(len(off) - 1)]) \
        if off[-1] else np.zeros(0, np.int64)


def _onehot(offsets, H, d):
    """[T, H*d] bf16: token with local index j is e_(j mod d) in every head."""
    j = _local_index(offsets)
    x = torch.zeros(len(j), H, d, dtype=torch.float32)
    if len(j):
        x[torch.arange(len(j)), :, torch.as_tensor(j % d)] = 1.0
    return x.reshape(len(j), H * d).to(torch.bfloat16)


def _tables(w, pos_sign=None, time_sign=None):
    """rab_pos, rab_time with rp + rt = +-ZV on every pair: both ZV/2 (mask only), or one
    table +-ZV by a sign pattern and the other 0."""
    P, nb = w.n_pos, w.n_tbuckets
    if pos_sign is None and time_sign is None:
        return torch.full((2 * P - 1,), ZV / 2), torch.full((nb,), ZV / 2)
    if pos_sign is not None:
        return torch.as_tensor(np.where(pos_sign, ZV, -ZV), dtype=torch.float32), torch.zeros(nb)
    return torch.zeros(2 * P - 1), torch.as_tensor(np.where(time_sign, ZV, -ZV), dtype=torch.float32)


def _layer(w, d):
    return ops.Layer(d["offsets"], d["ts"], w.H, w.d, torch.bfloat16, ALPHA, max(w.max_len, 1),
                     mask_kind=w.kind, n_static=d.get("n_static"), n_realtime=d.get("n_realtime"),
                     n_pos=w.n_pos, n_tbuckets=w.n_tbuckets)


def _seg(w):
    kind = {"causal": oracle.MASK_CAUSAL, "mtgr": oracle.MASK_MTGR, "mfalcon_seq": oracle.MASK_MFSEQ}[w.kind]
    ns = w.n_static if w.kind == "mtgr" else None
    nr = w.n_realtime if w.kind in ("mtgr", "mfalcon_seq") else None
    return kind, ns, nr


# ----------------------------------------------------------------------------
# expected counts from the oracle's per-pair decisions
# ----------------------------------------------------------------------------

def _pairs(w):
    kind, ns, nr = _seg(w)
    m, pi, tb, po = oracle.indices(w.offsets, w.ts, kind, ns, nr, w.n_pos, w.n_tbuckets)
    return m.astype(bool), pi.astype(np.int64), tb.astype(np.int64), po


def _live(pi, tb, pos_sign, time_sign):
    """Pairs whose bias is +ZV."""
    if pos_sign is not None:
        return np.asarray(pos_sign)[pi]
    if time_sign is not None:
        return np.asarray(time_sign)[tb]
    return np.ones(pi.shape, bool)


def _per_seq(w, po, flat):
    off = np.asarray(w.offsets, np.int64)
    for b in range(len(off) - 1):
        L = int(off[b + 1] - off[b])
        yield b, int(off[b]), L, flat[po[b]:po[b + 1]].reshape(L, L)


def _y_counts(w, m, live, po):
    """[T, d]: Y_i[r] * alpha / ZV = #{j : pair (i, j) visible and live, j = r mod d}."""
    out = np.zeros((int(w.offsets[-1]), w.d), np.int64)
    for _, s0, L, A in _per_seq(w, po, m & live):
        jr = np.arange(L) % w.d
        for r in range(w.d):
            out[s0:s0 + L, r] = A[:, jr == r].sum(1)
    return out


def _decode(x, unit, name):
    """Integer counts from a tensor whose entries are unit * count; the entries must sit
    within 1/4 of an integer."""
    v = x.detach().float().cpu().numpy().astype(np.float64) / unit
    r = np.rint(v)
    bad = np.abs(v - r) > 0.25
    assert not bad.any(), f"{name}: {int(bad.sum())} entries are not whole counts, e.g. {v[bad][:4]}"
    return r.astype(np.int64)


def _heads(x, H, d):
    return x.reshape(x.shape[0], H, d)


# ----------------------------------------------------------------------------
# cases
# ----------------------------------------------------------------------------

def _causal_case(d):
    """Lengths around every tile and block edge, a sequence past the position clamp, gaps
    of ~1 h (time buckets change inside blocks), 2^40-second gaps (64-bit time spans),
    equal timestamps (bucket 0 everywhere) and int64 extremes."""
    rng = np.random.default_rng(61)
    lens = [1, 5, 31, 32, 33, 127, 128, 129, 255, 256, 257, 300, 513, 700]
    ts = [W.increasing_ts(rng, L) for L in lens]
    lens += [400, 300, 150]
    ts.append(np.cumsum(rng.integers(1, 2**40, size=400)).astype(np.int64))
    ts.append(np.full(300, 1_700_000_000, np.int64))
    i = np.arange(150)
    ts.append(np.where(i % 3 == 0, np.iinfo(np.int64).max - i, np.iinfo(np.int64).min + i).astype(np.int64))
    return W.make_causal(lens, H=2, d=d, seed=62, alpha=ALPHA, ts_list=ts)


def _mtgr_case(d):
    """Rows with real-time tokens, none (R = 0), only static tokens, candidates whose
    timestamps tie history timestamps, and long behaviour segments."""
    rng = np.random.default_rng(63)
    prof, long_, rt, cand = [3, 24, 5, 2, 24], [40, 280, 20, 150, 600], [8, 0, 0, 40, 64], [6, 30, 0, 70, 100]
    ts = [W.mtgr_user(rng, a, b, c, e) for a, b, c, e in zip(prof, long_, rt, cand)]
    # ties: copy history timestamps onto some candidates of row 0 and row 3
    for r in (0, 3):
        S, R = prof[r] + long_[r], rt[r]
        c0 = S + R
        ts[r][c0:c0 + 3] = ts[r][S + R - 3:S + R] if R >= 3 else ts[r][S - 3:S]
    return W.make_mtgr(prof, long_, rt, cand, H=2, d=d, seed=64, alpha=ALPHA, ts_list=ts)


def _mfseq_case(d):
    w = W.make_mfalcon([0, 0, 1, 200, 300, 129, 64, 700], [0, 3, 5, 130, 300, 1, 0, 90], H=2, d=d, seed=65,
                       alpha=ALPHA)
    ws = W.mfalcon_seq_from(w, seed=66)
    ws.alpha = ALPHA
    return ws


CASES = {"causal": _causal_case, "mtgr": _mtgr_case, "mfalcon_seq": _mfseq_case}


def _draws(w, seed):
    rng = np.random.default_rng(seed)
    yield None, None
    for _ in range(N_DRAWS):
        yield rng.random(2 * w.n_pos - 1) < 0.5, None
    for _ in range(N_DRAWS):
        yield None, rng.random(w.n_tbuckets) < 0.5


# ----------------------------------------------------------------------------
# forward
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("kind,d", [("causal", 128), ("causal", 64), ("mtgr", 128), ("mtgr", 64),
                                    ("mfalcon_seq", 128)])
def test_forward_counts_exact(kind, d):
    w = CASES[kind](d)
    T = int(w.offsets[-1])
    w.q = torch.zeros(T, w.H * d, dtype=torch.bfloat16)
    w.k = torch.zeros(T, w.H * d, dtype=torch.bfloat16)
    w.v = _onehot(w.offsets, w.H, d)
    w.u = torch.ones(T, w.H * d, dtype=torch.bfloat16)
    dv = dev(w)
    layer = _layer(w, dv)
    m, pi, tb, po = _pairs(w)
    for n, (ps, ts_) in enumerate(_draws(w, seed=70 + d)):
        rp, rt = _tables(w, ps, ts_)
        out = layer.forward(dv["q"], dv["k"], dv["v"], dv["u"], rp.cuda(), rt.cuda(), dv["gamma"], dv["beta"])
        torch.cuda.synchronize()
        assert layer.check_device_error() == 0
        want = _y_counts(w, m, _live(pi, tb, ps, ts_), po)
        got = _decode(out["y"], ZV / ALPHA, f"y (draw {n})")
        for h in range(w.H):
            bad = np.argwhere(_heads(got, w.H, d)[:, h] != want)
            assert len(bad) == 0, (f"{kind} d={d} draw {n} head {h}: {len(bad)} counts differ, first "
                                   f"(token, r) {bad[:3].tolist()}")


def test_mfalcon_cached_scorer_counts_exact():
    """The cached-history scorer: candidates see every history token (bias by pidx(n, j) and
    tb(ts_c, ts_j)) and themselves; the self term is switched off here (candidate v = 0) and
    the history part compared with the one-row layout's candidate rows in the oracle."""
    d = 128
    w = W.make_mfalcon([0, 1, 200, 300, 129, 700], [3, 5, 130, 300, 1, 90], H=2, d=d, seed=67, alpha=ALPHA)
    ws = W.mfalcon_seq_from(w, seed=68)
    m, pi, tb, po = _pairs(ws)
    ho, co = np.asarray(w.hist_offsets, np.int64), np.asarray(w.cand_offsets, np.int64)
    w.cand_q = torch.zeros_like(w.cand_q)
    w.hist_k = torch.zeros_like(w.hist_k)
    w.cand_v = torch.zeros_like(w.cand_v)
    w.hist_v = _onehot(w.hist_offsets, w.H, d)
    dv = dev(w)
    lm, lc = int(np.diff(ho).max()), int(np.diff(co).max())
    sc = ops.MFalcon(dv["hist_offsets"], dv["hist_ts"], dv["cand_offsets"], dv["cand_ts"], w.H, d, ALPHA, 128, lm,
                     lc, n_pos=w.n_pos, n_tbuckets=w.n_tbuckets)
    for n, (ps, ts_) in enumerate(_draws(ws, seed=77)):
        rp, rt = _tables(ws, ps, ts_)
        out = sc.score(dv["hist_k"], dv["hist_v"], dv["cand_q"], dv["cand_k"], dv["cand_v"], dv["cand_u"],
                       rp.cuda(), rt.cuda(), dv["gamma"], dv["beta"])
        torch.cuda.synchronize()
        assert sc.check_device_error() == 0
        live = m & _live(pi, tb, ps, ts_)
        want = np.zeros((int(co[-1]), d), np.int64)
        for b, s0, L, A in _per_seq(ws, po, live):
            nh = int(ho[b + 1] - ho[b])
            jr = np.arange(nh) % d
            for r in range(d):
                want[co[b]:co[b + 1], r] = A[nh:, :nh][:, jr == r].sum(1)
        got = _decode(out["y"], ZV / ALPHA, f"y (draw {n})")
        for h in range(w.H):
            assert np.array_equal(_heads(got, w.H, d)[:, h], want), f"draw {n} head {h}"


# ----------------------------------------------------------------------------
# backward (attention only, from dL/dY)
# ----------------------------------------------------------------------------

def _bwd_counts(w, live_pairs, po):
    """Counts of the backward with dY_i = e_(i mod d), V_j = e_(j mod d) and z = +-ZV:
       dV_j[r]   = #{i : (i, j) live, i = r}          (unit ZV / alpha)
       dQ_i[r]   = #{j : (i, j) live, j = i = r}      (K one-hot; unit 1 / alpha)
       dK_j[r]   = #{i : (i, j) live, i = j = r}      (Q one-hot; unit 1 / alpha)
       d_rab_pos[p], d_rab_time[t] = #{live (i, j) : i = j mod d, pidx = p / tb = t}."""
    T, d = int(w.offsets[-1]), w.d
    dv = np.zeros((T, d), np.int64)
    dq = np.zeros((T, d), np.int64)
    dk = np.zeros((T, d), np.int64)
    same = np.zeros(live_pairs.shape, bool)
    for b, s0, L, A in _per_seq(w, po, live_pairs):
        ir = np.arange(L) % d
        eq = ir[:, None] == ir[None, :]
        same[po[b]:po[b + 1]] = (A & eq).reshape(-1)
        for r in range(d):
            dv[s0:s0 + L, r] = A[ir == r, :].sum(0)
        c = (A & eq)
        dq[s0 + np.arange(L), ir] = c.sum(1)
        dk[s0 + np.arange(L), ir] = c.sum(0)
    return dv, dq, dk, same


@pytest.mark.parametrize("kind,d", [("causal", 128), ("causal", 64), ("mtgr", 128)])
def test_backward_counts_exact(kind, d):
    w = CASES[kind](d)
    T = int(w.offsets[-1])
    zeros = torch.zeros(T, w.H * d, dtype=torch.bfloat16)
    oh = _onehot(w.offsets, w.H, d)
    w.q, w.k, w.v, w.u = zeros, oh, oh, torch.ones_like(zeros)
    dvv = dev(w)
    dy = oh.cuda()
    layer = _layer(w, dvv)
    m, pi, tb, po = _pairs(w)
    for n, (ps, ts_) in enumerate(_draws(w, seed=80 + d)):
        if n > 2 and n != N_DRAWS + 1:
            continue                   # mask only, two position draws, one time draw
        rp, rt = _tables(w, ps, ts_)
        rp, rt = rp.cuda(), rt.cuda()
        live = m & _live(pi, tb, ps, ts_)
        want_dv, want_dq, want_dk, same = _bwd_counts(w, live, po)
        # run A: Q = 0, K one-hot -> dQ counts (dK = 0), dV, bias-table gradients
        g = layer.backward_from_dy(dvv["q"] * 0, dvv["k"], dvv["v"], rp, rt, dy)
        torch.cuda.synchronize()
        assert layer.check_device_error() == 0
        got_dv = _decode(g["dv"], ZV / ALPHA, f"dv (draw {n})")
        got_dq = _decode(g["dq"], 1.0 / ALPHA, f"dq (draw {n})")
        assert not g["dk"].float().abs().max().item(), "dk must be 0 with Q = 0"
        for h in range(w.H):
            assert np.array_equal(_heads(got_dv, w.H, d)[:, h], want_dv), f"dv draw {n} head {h}"
            assert np.array_equal(_heads(got_dq, w.H, d)[:, h], want_dq), f"dq draw {n} head {h}"
        # every head adds the same counts to the shared tables
        want_p = np.bincount(pi[same], minlength=2 * w.n_pos - 1) * w.H
        want_t = np.bincount(tb[same], minlength=w.n_tbuckets) * w.H
        assert np.array_equal(_decode(g["d_rab_pos"], 1.0 / ALPHA, "d_rab_pos"), want_p), f"d_rab_pos draw {n}"
        assert np.array_equal(_decode(g["d_rab_time"], 1.0 / ALPHA, "d_rab_time"), want_t), f"d_rab_time draw {n}"
        # run B: Q one-hot, K = 0 -> dK counts (dQ = 0)
        g = layer.backward_from_dy(dvv["k"], dvv["q"] * 0, dvv["v"], rp, rt, dy)
        torch.cuda.synchronize()
        assert layer.check_device_error() == 0
        got_dk = _decode(g["dk"], 1.0 / ALPHA, f"dk (draw {n})")
        assert not g["dq"].float().abs().max().item(), "dq must be 0 with K = 0"
        for h in range(w.H):
            assert np.array_equal(_heads(got_dk, w.H, d)[:, h], want_dk), f"dk draw {n} head {h}"
