"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle on the
same seeded inputs.  Small cases are compared element by element; full-size
workloads on sampled rows (sequences are independent, so the oracle computes
only the sampled rows or sequences)."""
import numpy as np
import pytest
import torch

import oracle
from hstu_jagged_pointwise_b200 import workloads as W
from parity import (assert_bf16, assert_f32, bf16, errors, run_layer, run_mfalcon, storage_bwd, storage_fwd,
                    storage_mfalcon)

pytestmark = pytest.mark.gpu


# ----------------------------------------------------------------------------
# integer decisions: bit-exact
# ----------------------------------------------------------------------------

def _boundary_ts():
    return np.array([0, 1, 2, 3, 4, 7, 8, 15, 16, 3599, 3600, 4096, 2**31 - 1, 2**31, 2**40,
                     2**62 - 1, 2**62, 2**62 + 5, 2**63 - 1], dtype=np.int64)


def test_debug_indices_bit_exact():
    from hstu_jagged_pointwise_b200 import ops
    cases = []
    # causal: lengths around the position clamp (254..256 apart) and boundary time deltas
    ts_a = _boundary_ts()
    ts_b = W.increasing_ts(np.random.default_rng(0), 300)
    ts_c = np.array([-2**62, 0, 2**62], dtype=np.int64)
    cases.append(("causal", [ts_a, ts_b, ts_c, np.array([5], np.int64)], None, None))
    # MTGR: hand row, tie timestamps, all-static row, no real-time row
    hand = np.array([0, 10, 20, 30, 40, 35, 15, 40], np.int64)
    rng = np.random.default_rng(1)
    u1 = W.mtgr_user(rng, 3, 40, 8, 6)
    u2 = W.mtgr_user(rng, 2, 280, 0, 30)
    u3 = W.mtgr_user(rng, 5, 20, 0, 0)
    cases.append(("mtgr", [hand, u1, u2, u3], [3, 43, 282, 25], [2, 8, 0, 0]))
    # full-sequence M-FALCON: candidates before, at and after the history's last timestamp,
    # a history longer than the position clamp, no history, no candidates
    h1 = W.increasing_ts(rng, 300)
    c1 = np.concatenate([h1[-1] + np.array([0, 5, 1]), h1[:2]])
    cases.append(("mfalcon_seq", [np.concatenate([h1, c1]), ts_a[:6], ts_b[:40]], None, [300, 0, 40]))
    for kind, ts_list, ns, nr in cases:
        lens = [len(t) for t in ts_list]
        off = np.zeros(len(lens) + 1, np.int32)
        off[1:] = np.cumsum(lens)
        ts = np.concatenate(ts_list)
        k = {"causal": oracle.MASK_CAUSAL, "mtgr": oracle.MASK_MTGR, "mfalcon_seq": oracle.MASK_MFSEQ}[kind]
        m0, p0, t0, _ = oracle.indices(off, ts, k, ns, nr)
        dn = lambda a, dt: torch.as_tensor(np.asarray(a, dt)).cuda()
        m1, p1, t1, _ = ops.debug_indices(dn(off, np.int32), dn(ts, np.int64), kind,
                                          None if ns is None else dn(ns, np.int32),
                                          None if nr is None else dn(nr, np.int32))
        np.testing.assert_array_equal(m1.cpu().numpy(), m0)
        np.testing.assert_array_equal(p1.cpu().numpy(), p0)
        np.testing.assert_array_equal(t1.cpu().numpy(), t0)


# ----------------------------------------------------------------------------
# fp32 path (the tiny configuration): relative error <= 1e-5
# ----------------------------------------------------------------------------

def test_tiny_fp32_forward():
    w = W.tiny_fp32(seed=0)
    out, _, _ = run_layer(w)
    y, o, mu, rs = oracle.layer_fwd(w)
    assert_f32(out["y"], y, "y")
    assert_f32(out["o_pre"], o, "o_pre")
    assert_f32(out["mean"], mu, "mean")
    assert_f32(out["rstd"], rs, "rstd")


@pytest.mark.parametrize("kind", ["causal", "mtgr"])
def test_fp32_backward(kind):
    if kind == "causal":
        w = W.make_causal([17, 64, 100, 255], H=2, d=32, dtype=torch.float32, seed=3, alpha=255.0,
                          random_affine=True, with_grad=True)
    else:
        w = W.make_mtgr([4, 24], [30, 150], [5, 20], [7, 40], H=2, d=32, dtype=torch.float32, seed=4,
                        random_affine=True, with_grad=True)
    out, _, _ = run_layer(w, backward=True)
    ref = oracle.layer_bwd(w)
    assert_f32(out["y"], ref["y"], "y")
    for k in ("dq", "dk", "dv", "du", "d_rab_pos", "d_rab_time"):
        assert_f32(out[k], ref[k], k)
    assert_f32(out["d_gamma"], ref["dgamma"], "d_gamma")
    assert_f32(out["d_beta"], ref["dbeta"], "d_beta")


# ----------------------------------------------------------------------------
# bf16 tcgen05 forward: several tiles, ragged tails, empty and 1-token sequences
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("d", [128, 64])
def test_bf16_causal_forward_ragged(d):
    w = W.make_causal([1, 127, 128, 129, 0, 300, 513, 2], H=2, d=d, seed=5)
    out, _, _ = run_layer(w)
    y, o, mu, rs = oracle.layer_fwd(w)
    st = storage_fwd(w)
    assert_bf16(out["y"], y, "y", st["y"])
    assert_bf16(out["o_pre"], o, "o_pre", st["o_pre"])


def test_bf16_causal_forward_long_positions_and_times():
    """Rows far from the diagonal (clamped position index) and huge time gaps."""
    rng = np.random.default_rng(7)
    ts = np.cumsum(rng.integers(1, 2**40, size=700)).astype(np.int64)
    w = W.make_causal([700, 900], H=2, d=128, seed=6,
                      ts_list=[ts, W.increasing_ts(rng, 900)])
    out, _, _ = run_layer(w)
    y, o, _, _ = oracle.layer_fwd(w)
    st = storage_fwd(w)
    assert_bf16(out["y"], y, "y", st["y"])
    assert_bf16(out["o_pre"], o, "o_pre", st["o_pre"])


def test_bf16_mtgr_forward_small():
    w = W.make_mtgr([24, 3, 24, 5], [40, 300, 150, 0], [8, 0, 64, 3], [6, 150, 20, 7], H=2, d=128,
                    seed=8, alpha=500.0)
    out, _, _ = run_layer(w)
    y, o, _, _ = oracle.layer_fwd(w)
    st = storage_fwd(w)
    assert_bf16(out["y"], y, "y", st["y"])
    assert_bf16(out["o_pre"], o, "o_pre", st["o_pre"])


@pytest.mark.parametrize("kind,d", [("causal", 128), ("mtgr", 128), ("causal", 64), ("mtgr", 64)])
def test_bf16_backward_small(kind, d):
    if kind == "causal":
        w = W.make_causal([1, 127, 129, 300], H=2, d=d, seed=9, random_affine=True, with_grad=True)
    else:
        w = W.make_mtgr([24, 2], [100, 190], [10, 0], [20, 70], H=2, d=d, seed=10, random_affine=True,
                        with_grad=True)
    out, _, _ = run_layer(w, backward=True)
    ref = oracle.layer_bwd(w)
    st = storage_bwd(w)
    assert_bf16(out["y"], ref["y"], "y", st["y"])
    for k in ("dq", "dk", "dv", "du", "d_rab_pos", "d_rab_time"):
        assert_bf16(out[k], ref[k], k, st[k])
    assert_bf16(out["d_gamma"], ref["dgamma"], "d_gamma", st["dgamma"])
    assert_bf16(out["d_beta"], ref["dbeta"], "d_beta", st["dbeta"])


def test_reproducible_outputs_across_runs():
    """Two runs of the same forward + backward on a batch that spreads over many CTAs (dynamic
    work fetch) give bitwise-equal Y, O_pre, dK, dV, dU, dgamma and dbeta: each of those is
    summed in a fixed order (key tiles in order inside one CTA, fixed-order LayerNorm
    partials).  dQ and the rab gradients are accumulated with reductions whose order follows
    the warps' timing, so they are only checked to agree closely."""
    w = W.make_causal([1000, 700, 2048, 3000, 129, 1], H=4, d=128, seed=31, random_affine=True, with_grad=True)
    a, _, _ = run_layer(w, backward=True)
    b, _, _ = run_layer(w, backward=True)
    for k in ("y", "o_pre", "dk", "dv", "du", "d_gamma", "d_beta"):
        assert torch.equal(a[k], b[k]), f"{k} differs between two runs"
    for k in ("dq", "d_rab_pos", "d_rab_time"):
        rel, mx, rms = errors(a[k], b[k])
        assert rel <= 1e-3, f"{k}: runs differ by rel {rel:.2e}"


# ----------------------------------------------------------------------------
# Group LayerNorm (one gamma / beta row per token source)
# ----------------------------------------------------------------------------

def _check_layer_fwd_bwd(w, f32=False):
    out, _, _ = run_layer(w, backward=True)
    y, o, _, _ = oracle.layer_fwd(w)
    ref = oracle.layer_bwd(w)
    if f32:
        assert_f32(out["y"], y, "y")
        assert_f32(out["o_pre"], o, "o_pre")
        for k in ("dq", "dk", "dv", "du", "d_rab_pos", "d_rab_time"):
            assert_f32(out[k], ref[k], k)
        assert_f32(out["d_gamma"], ref["dgamma"], "d_gamma")
        assert_f32(out["d_beta"], ref["dbeta"], "d_beta")
        return
    sf, sb = storage_fwd(w), storage_bwd(w)
    assert_bf16(out["y"], y, "y", sf["y"])
    assert_bf16(out["o_pre"], o, "o_pre", sf["o_pre"])
    for k in ("dq", "dk", "dv", "du", "d_rab_pos", "d_rab_time"):
        assert_bf16(out[k], ref[k], k, sb[k])
    assert_bf16(out["d_gamma"], ref["dgamma"], "d_gamma", sb["dgamma"])
    assert_bf16(out["d_beta"], ref["dbeta"], "d_beta", sb["dbeta"])


def test_bf16_extreme_timestamps_forward_backward():
    """Timestamps near both ends of int64 inside every warp's keys and queries, so 64-bit time
    differences wrap around: the kernels' 32-bit time offsets must fall back to 64 bits.  The
    time-bias table is large and q, k small, so one wrong bucket shows far above tolerance."""
    lo, hi = np.iinfo(np.int64).min, np.iinfo(np.int64).max
    i = np.arange(300)
    ts_a = np.where(i % 2 == 0, hi - (i % 7), lo + (i % 5)).astype(np.int64)
    ts_b = W.increasing_ts(np.random.default_rng(3), 200)
    ts_b[::37] = lo + 3
    ts_c = np.where(i[:150] % 3 == 0, hi, -(i[:150] % 11)).astype(np.int64)
    w = W.make_causal([300, 200, 150], H=2, d=128, seed=31, ts_list=[ts_a, ts_b, ts_c], random_affine=True,
                      with_grad=True)
    w.q = (w.q.float() * 0.25).to(w.dtype)
    w.k = (w.k.float() * 0.25).to(w.dtype)
    w.rab_time = torch.randn(w.rab_time.shape, generator=torch.Generator().manual_seed(32)) * 4.0
    _check_layer_fwd_bwd(w)


@pytest.mark.parametrize("d", [128, 64])
def test_gln_mtgr_forward_backward(d):
    """MTGR rows with groups profile / behaviour / real-time / candidate from the segments."""
    w = W.make_mtgr([24, 2, 5], [100, 190, 0], [10, 0, 30], [20, 70, 9], H=2, d=d, seed=21, random_affine=True,
                    with_grad=True)
    _check_layer_fwd_bwd(W.with_group_norm(w, seed=22))


def test_gln_fp32_random_groups():
    w = W.make_causal([17, 64, 100, 255], H=2, d=32, dtype=torch.float32, seed=23, alpha=255.0, with_grad=True)
    _check_layer_fwd_bwd(W.with_group_norm(w, seed=24, groups=3), f32=True)


def test_gln_bad_group_flagged():
    from hstu_jagged_pointwise_b200 import capi
    w = W.with_group_norm(W.make_causal([40, 9], H=2, d=64, seed=25), seed=26, groups=4)
    out, layer, d = run_layer(w)
    layer.token_group[5] = 9                                    # no such group
    layer.forward(d["q"], d["k"], d["v"], d["u"], d["rab_pos"], d["rab_time"], d["gamma"], d["beta"])
    assert layer.check_device_error() == capi.HSTU_ERR_DEVICE_BOUNDS
    assert layer.check_device_error() == capi.HSTU_OK


# ----------------------------------------------------------------------------
# M-FALCON
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("head_dim", [128, 64])
def test_mfalcon_small_and_microbatch_invariance(head_dim):
    w = W.make_mfalcon([0, 1, 200, 300, 129], [3, 5, 130, 300, 1], H=2, d=head_dim, seed=11, b_m=256,
                       alpha=301.0)
    y_ref, o_ref = oracle.mfalcon_layer(w)
    st = storage_mfalcon(w)
    out, d = run_mfalcon(w)
    assert_bf16(out["y"], y_ref, "y", st["y"])
    assert_bf16(out["o_pre"], o_ref, "o_pre", st["o_pre"])
    for bm in (1, 100, 128, 1000):
        o2, _ = run_mfalcon(w, b_m=bm, d=d)
        assert torch.equal(o2["y"], out["y"]), f"b_m={bm} changed the results"


def test_mfalcon_permutation_equivariance():
    w = W.make_mfalcon([400], [200], H=2, d=128, seed=12, alpha=401.0)
    out, _ = run_mfalcon(w)
    perm = np.random.default_rng(0).permutation(200)
    pt = torch.as_tensor(perm)
    for name in ("cand_q", "cand_k", "cand_v", "cand_u"):
        setattr(w, name, getattr(w, name)[pt].contiguous())
    w.cand_ts = w.cand_ts[perm]
    out2, _ = run_mfalcon(w)
    assert torch.equal(out2["y"], out["y"][pt.cuda()])


# ----------------------------------------------------------------------------
# full-sequence M-FALCON: [history ; candidates] in one jagged row
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("d", [128, 64])
def test_mfalcon_seq_forward_small(d):
    # empty row, no history, one history token, splits off the 128-row tile grid, no candidates
    w = W.make_mfalcon([0, 0, 1, 200, 300, 129, 64], [0, 3, 5, 130, 300, 1, 0], H=2, d=d, seed=13,
                       alpha=301.0)
    ws = W.mfalcon_seq_from(w, seed=14)
    out, _, _ = run_layer(ws)
    y, o, _, _ = oracle.layer_fwd(ws)
    st = storage_fwd(ws)
    assert_bf16(out["y"], y, "y", st["y"])
    assert_bf16(out["o_pre"], o, "o_pre", st["o_pre"])
    if d == 128:
        # the candidate rows score like the cached-history kernel on the same users
        cand = np.concatenate([np.arange(ws.offsets[b] + ws.n_realtime[b], ws.offsets[b + 1])
                               for b in range(ws.B)]).astype(np.int64)
        oc, _ = run_mfalcon(w)
        rel, _, _ = errors(out["y"][torch.as_tensor(cand).cuda()], oc["y"])
        assert rel < 5e-3, f"cached-history and one-row candidate scores differ: rel {rel:.2e}"


def test_mfalcon_seq_forward_fp32():
    w = W.make_mfalcon([0, 5, 70, 40], [2, 0, 9, 33], H=2, d=32, dtype=torch.float32, seed=19, alpha=71.0)
    ws = W.mfalcon_seq_from(w, seed=20)
    out, _, _ = run_layer(ws)
    y, o, _, _ = oracle.layer_fwd(ws)
    assert_f32(out["y"], y, "y")
    assert_f32(out["o_pre"], o, "o_pre")


def _cache_from_one_row(ws, dtype=None):
    from hstu_jagged_pointwise_b200 import ops
    cast = (lambda t: t.cuda()) if dtype is None else (lambda t: t.to(dtype).cuda())
    off = torch.as_tensor(ws.offsets).cuda()
    ts = torch.as_tensor(ws.ts).cuda()
    nh = torch.as_tensor(np.asarray(ws.n_realtime, np.int32)).cuda()
    out = ops.mfalcon_cache_history(off, ts, nh, cast(ws.k), cast(ws.v))
    torch.cuda.synchronize()
    return out


def test_mfalcon_cache_producer_exact_and_scores_identically():
    """The history rows of the one-row layout, packed, are the cache the scorer reads: bit-exact."""
    w = W.make_mfalcon([0, 0, 1, 200, 300, 129, 64, 3], [0, 3, 5, 130, 300, 1, 0, 2], H=2, d=128, seed=15,
                       alpha=301.0)
    ws = W.mfalcon_seq_from(w, seed=16)
    c = _cache_from_one_row(ws)
    assert int(c["status"].item()) == 0
    np.testing.assert_array_equal(c["hist_offsets"].cpu().numpy(), np.asarray(w.hist_offsets, np.int32))
    np.testing.assert_array_equal(c["hist_ts"].cpu().numpy(), np.asarray(w.hist_ts, np.int64))
    assert torch.equal(c["hist_k"].cpu(), w.hist_k) and torch.equal(c["hist_v"].cpu(), w.hist_v)
    # fp32 rows take the same path
    c32 = _cache_from_one_row(ws, torch.float32)
    assert torch.equal(c32["hist_k"].cpu(), w.hist_k.float()) and torch.equal(c32["hist_v"].cpu(), w.hist_v.float())
    # scoring from the produced cache is the scoring from the original one
    ref, d = run_mfalcon(w)
    d2 = dict(d, hist_k=c["hist_k"], hist_v=c["hist_v"], hist_offsets=c["hist_offsets"], hist_ts=c["hist_ts"])
    got, _ = run_mfalcon(w, d=d2)
    assert torch.equal(got["y"], ref["y"]) and torch.equal(got["o_pre"], ref["o_pre"])


def test_mfalcon_cache_producer_rejects_bad_batches():
    from hstu_jagged_pointwise_b200 import ops
    w = W.make_mfalcon([10, 20], [4, 5], H=2, d=64, seed=17, alpha=21.0)
    ws = W.mfalcon_seq_from(w, seed=18)
    off = torch.as_tensor(ws.offsets).cuda()
    ts = torch.as_tensor(ws.ts).cuda()
    k, v = ws.k.cuda(), ws.v.cuda()
    for nh, rows in (([10, 26], 36), ([-1, 20], 30), ([10, 20], 29)):   # R > L, R < 0, no room
        out = dict(hist_offsets=torch.full((3,), -7, dtype=torch.int32, device="cuda"),
                   hist_ts=torch.full((rows,), -7, dtype=torch.int64, device="cuda"),
                   hist_k=torch.full((rows, k.shape[1]), -7.0, dtype=k.dtype, device="cuda"),
                   hist_v=torch.full((rows, k.shape[1]), -7.0, dtype=k.dtype, device="cuda"),
                   status=torch.zeros(1, dtype=torch.int32, device="cuda"))
        ops.mfalcon_cache_history(off, ts, torch.tensor(nh, dtype=torch.int32, device="cuda"), k, v, out=out)
        torch.cuda.synchronize()
        assert int(out["status"].item()) == 1, nh
        assert bool((out["hist_offsets"] == -7).all()) and bool((out["hist_ts"] == -7).all())
        assert bool((out["hist_k"] == -7).all()) and bool((out["hist_v"] == -7).all())


def _seq_slice(w, b):
    """Row b of a full-sequence M-FALCON workload alone (rows are independent)."""
    import dataclasses
    s0, s1 = int(w.offsets[b]), int(w.offsets[b + 1])
    sub = dataclasses.replace(w, offsets=np.array([0, s1 - s0], np.int32), ts=w.ts[s0:s1],
                              n_realtime=np.asarray(w.n_realtime[b:b + 1], np.int32),
                              q=w.q[s0:s1], k=w.k[s0:s1], v=w.v[s0:s1], u=w.u[s0:s1])
    return sub, s0


def test_mfalcon_ranking_full_sequence_sampled_rows():
    """256 users x [2048 history ; 1024 candidates] in one launch; sampled rows of four users."""
    w = W.mfalcon_ranking(seed=0)
    ws = W.mfalcon_seq_from(w, seed=1)
    out, _, _ = run_layer(ws)
    # the KV cache produced from this batch is the ranking workload's cache, exactly
    c = _cache_from_one_row(ws)
    assert int(c["status"].item()) == 0
    assert torch.equal(c["hist_k"].cpu(), w.hist_k) and torch.equal(c["hist_v"].cpu(), w.hist_v)
    np.testing.assert_array_equal(c["hist_ts"].cpu().numpy(), np.asarray(w.hist_ts, np.int64))
    del c
    rng = np.random.default_rng(5)
    for b in (0, 97, 200, 255):
        sub, s0 = _seq_slice(ws, b)
        nh = int(sub.n_realtime[0])
        rows = np.unique(np.concatenate([rng.integers(0, nh, 6), [0, nh - 1, nh, sub.T - 1],
                                         rng.integers(nh, sub.T, 6)])).astype(np.int64)
        y, o, _, _ = oracle.layer_fwd(sub, rows)
        st = storage_fwd(sub, rows)
        rt = torch.as_tensor(rows + s0).cuda()
        assert_bf16(out["y"][rt], y, f"y[user {b}]", st["y"])
        assert_bf16(out["o_pre"][rt], o, f"o_pre[user {b}]", st["o_pre"])


# ----------------------------------------------------------------------------
# projections: f1 (X -> U, V, Q, K with SiLU) and f2, forward and backward
# ----------------------------------------------------------------------------

def _bf(a):
    return torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16)


def _status_ok(out):
    assert int(out["status"].item()) == 0


def test_projections_small_forward_backward():
    """Tails everywhere: T = 300 rows (2.3 row tiles), d_in = 224 (K tail of 32, and a partial
    column tile for dX), d_out = 224 (a partial column tile and half a stored chunk)."""
    from hstu_jagged_pointwise_b200 import ops
    w = W.make_projection(300, 224, 64, 224, seed=31)
    c = {n: getattr(w, n).cuda() for n in ("x", "w1", "b1", "o_pre", "w2", "b2", "g_out")}
    D = w.D
    f = ops.f1_fwd(c["x"], c["w1"], c["b1"], D)
    torch.cuda.synchronize()
    _status_ok(f)
    z, u, v, q, k = oracle.f1_fwd(w.x, w.w1, w.b1, D)
    for name, ref in (("z", z), ("u", u), ("v", v), ("q", q), ("k", k)):
        assert_bf16(f[name], ref, name, bf16(ref))
    o = ops.f2_fwd(c["o_pre"], c["w2"], c["b2"], residual=c["x"])
    torch.cuda.synchronize()
    _status_ok(o)
    ref = oracle.f2_fwd(w.o_pre, w.w2, w.b2, w.x)
    assert_bf16(o["out"], ref, "out", bf16(ref))
    # backward of f1 from the oracle's Z (rounded to the bf16 the layer stores)
    zb = _bf(z)
    dact = w.dact
    blocks = [dact[:, i * D:(i + 1) * D].contiguous() for i in range(4)]
    b = ops.f1_bwd(c["x"], c["w1"], zb.cuda(), *[t.cuda() for t in blocks])
    torch.cuda.synchronize()
    _status_ok(b)
    dz, dx, dw1, db1 = oracle.f1_bwd(w.x, w.w1, zb, *blocks)
    dzb = bf16(dz)                                          # the kernel keeps dZ in bf16
    assert_bf16(b["dx"], dx, "dx", bf16(dzb @ oracle.f32(w.w1).astype(np.float64)))
    assert_bf16(b["dw1"], dw1, "dw1", dzb.T @ oracle.f32(w.x).astype(np.float64))
    assert_bf16(b["db1"], db1, "db1", dzb.sum(0))
    g = ops.f2_bwd(c["o_pre"], c["w2"], c["g_out"])
    torch.cuda.synchronize()
    _status_ok(g)
    do, dw2, db2 = oracle.f2_bwd(w.o_pre, w.w2, w.g_out)
    assert_bf16(g["d_o_pre"], do, "d_o_pre", bf16(do))
    assert_bf16(g["dw2"], dw2, "dw2")
    assert_bf16(g["db2"], db2, "db2")


def test_projections_large_sampled():
    """The large layer's projections (262,144 tokens, d_model 1024) in the bench's launch
    configuration: sampled rows of every row-wise output, sampled entries of the weight
    gradients and bias gradients (each a sum over all tokens)."""
    from hstu_jagged_pointwise_b200 import ops
    w = W.projection_large(seed=0, device="cuda")
    D = w.D
    f = ops.f1_fwd(w.x, w.w1, w.b1, D)
    o = ops.f2_fwd(w.o_pre, w.w2, w.b2, residual=w.x)
    blocks = [w.dact[:, i * D:(i + 1) * D].contiguous() for i in range(4)]
    b = ops.f1_bwd(w.x, w.w1, w.z, *blocks)
    g = ops.f2_bwd(w.o_pre, w.w2, w.g_out)
    torch.cuda.synchronize()
    for out in (f, o, b, g):
        _status_ok(out)
    rng = np.random.default_rng(9)
    rows = np.unique(np.concatenate([rng.integers(0, w.T, 40), [0, w.T - 1]]))
    rt = torch.as_tensor(rows).cuda()
    cpu = lambda t: t[rt].cpu()
    z, u, v, q, k = oracle.f1_fwd(cpu(w.x), w.w1.cpu(), w.b1.cpu(), D)
    for name, ref in (("z", z), ("u", u), ("v", v), ("q", q), ("k", k)):
        assert_bf16(f[name][rt], ref, name, bf16(ref))
    ref = oracle.f2_fwd(cpu(w.o_pre), w.w2.cpu(), w.b2.cpu(), cpu(w.x))
    assert_bf16(o["out"][rt], ref, "out", bf16(ref))
    dz, dx, _, _ = oracle.f1_bwd(cpu(w.x), w.w1.cpu(), cpu(w.z), *[cpu(t) for t in blocks])
    assert_bf16(b["dx"][rt], dx, "dx", bf16(bf16(dz) @ oracle.f32(w.w1.cpu()).astype(np.float64)))
    do, _, _ = oracle.f2_bwd(cpu(w.o_pre), w.w2.cpu(), cpu(w.g_out))
    assert_bf16(g["d_o_pre"][rt], do, "d_o_pre", bf16(do))
    # weight and bias gradients: sampled columns, sums over all 262,144 tokens
    ci = np.array([0, 5, 1023, 1024, 2047, 3000, 4095])          # output columns of f1 (all four blocks)
    cj = np.array([0, 17, 511, 1023])                             # input columns
    zc = w.z[:, torch.as_tensor(ci).cuda()].cpu()
    dc = w.dact[:, torch.as_tensor(ci).cuda()].cpu()
    empty = torch.zeros(w.T, 0, dtype=torch.bfloat16)
    xs = w.x[:, torch.as_tensor(cj).cuda()].cpu()
    dz_c, _, dw1_c, db1_c = oracle.f1_bwd(xs, torch.zeros(len(ci), len(cj), dtype=torch.bfloat16), zc, dc, empty,
                                          empty, empty)
    got_w1 = b["dw1"][torch.as_tensor(ci).cuda()][:, torch.as_tensor(cj).cuda()]
    assert_bf16(got_w1, dw1_c, "dw1 (sampled)", bf16(dz_c).T @ oracle.f32(xs).astype(np.float64))
    assert_bf16(b["db1"][torch.as_tensor(ci).cuda()], db1_c, "db1 (sampled)", bf16(dz_c).sum(0))
    oi = np.array([0, 300, 1023])
    gs = w.g_out[:, torch.as_tensor(oi).cuda()].cpu()
    os_ = w.o_pre[:, torch.as_tensor(cj).cuda()].cpu()
    _, dw2_c, db2_c = oracle.f2_bwd(os_, torch.zeros(len(oi), len(cj), dtype=torch.bfloat16), gs)
    assert_bf16(g["dw2"][torch.as_tensor(oi).cuda()][:, torch.as_tensor(cj).cuda()], dw2_c, "dw2 (sampled)")
    assert_bf16(g["db2"][torch.as_tensor(oi).cuda()], db2_c, "db2 (sampled)")


# ----------------------------------------------------------------------------
# a whole HSTU layer: f1 -> attention -> Norm * U -> f2 (+ X), forward and backward
# ----------------------------------------------------------------------------

def _layer_chain(lw, store):
    """The layer through the oracle.  store=False: exact (float64 between the steps);
    store=True: the values rounded to bf16 wherever the library stores them."""
    import copy
    r = bf16 if store else (lambda a: np.asarray(a, np.float64))
    a = lw.attn
    D = a.D
    z, u, v, q, k = oracle.f1_fwd(lw.x, lw.w1, lw.b1, D)
    aw = copy.copy(a)
    aw.q, aw.k, aw.v, aw.u = (torch.as_tensor(r(t)) for t in (q, k, v, u))
    if store:
        sf = storage_fwd(aw)
        o_pre = sf["o_pre"]
    else:
        _, o_pre, _, _ = oracle.layer_fwd(aw)
    out = r(oracle.f2_fwd(o_pre, lw.w2, lw.b2, lw.x))
    d_o_pre, dw2, db2 = oracle.f2_bwd(o_pre, lw.w2, lw.g_out)
    aw.grad = torch.as_tensor(r(d_o_pre))
    g = storage_bwd(aw) if store else oracle.layer_bwd(aw)
    dz, dx, dw1, db1 = oracle.f1_bwd(lw.x, lw.w1, r(z), g["du"], g["dv"], g["dq"], g["dk"])
    if store:
        dzb = bf16(dz)
        w1 = oracle.f32(lw.w1).astype(np.float64)
        dx = dzb @ w1
        dw1 = dzb.T @ oracle.f32(lw.x).astype(np.float64)
        db1 = dzb.sum(0)
    dx = r(dx + oracle.f32(lw.g_out))
    return dict(out=out, dx=dx, dw1=dw1, db1=db1, dw2=dw2, db2=db2, d_rab_pos=g["d_rab_pos"],
                d_rab_time=g["d_rab_time"], d_ln_gamma=g["dgamma"], d_ln_beta=g["dbeta"])


@pytest.mark.parametrize("kind", ["causal", "mtgr"])
def test_full_layer_forward_backward(kind):
    from hstu_jagged_pointwise_b200 import ops
    if kind == "causal":
        a = W.make_causal([1, 127, 129, 300], H=2, d=64, seed=41, random_affine=True, with_grad=True)
    else:
        a = W.with_group_norm(W.make_mtgr([24, 2], [100, 190], [10, 0], [20, 70], H=2, d=64, seed=42,
                                          random_affine=True, with_grad=True), seed=43)
    lw = W.make_layer(a, d_model=96, seed=44)
    c = {n: getattr(lw, n).cuda() for n in ("x", "w1", "b1", "w2", "b2", "g_out")}
    prm = dict(w1=c["w1"], b1=c["b1"], w2=c["w2"], b2=c["b2"], rab_pos=a.rab_pos.cuda(),
               rab_time=a.rab_time.cuda(), ln_gamma=a.gamma.cuda(), ln_beta=a.beta.cuda())
    tg = torch.as_tensor(np.asarray(a.token_group, np.uint8)).cuda() if a.n_groups > 1 else None
    layer = ops.HSTULayer(torch.as_tensor(a.offsets).cuda(), torch.as_tensor(a.ts).cuda(), 96, a.H, a.d, a.alpha,
                          a.max_len, mask_kind=a.kind,
                          n_static=None if a.n_static is None else torch.as_tensor(a.n_static).cuda(),
                          n_realtime=None if a.n_realtime is None else torch.as_tensor(a.n_realtime).cuda(),
                          n_groups=a.n_groups, token_group=tg)
    fwd = layer.forward(c["x"], prm)
    grads = layer.backward(fwd, c["g_out"], prm)
    torch.cuda.synchronize()
    assert layer.check_device_error() == 0
    ref, st = _layer_chain(lw, False), _layer_chain(lw, True)
    assert_bf16(fwd["out"], ref["out"], "out", st["out"], chain=True)
    for k in ("dx", "dw1", "db1", "dw2", "db2", "d_rab_pos", "d_rab_time", "d_ln_gamma", "d_ln_beta"):
        assert_bf16(grads[k], ref[k], k, st[k], chain=True)


# ----------------------------------------------------------------------------
# the data step: Stochastic Length sampling, gathers, token-balanced bins (bit-exact)
# ----------------------------------------------------------------------------

def _sl_check(lens, cap, seed, width=256):
    from hstu_jagged_pointwise_b200 import ops
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    new_ref, idx_ref = oracle.sl_sample(off, cap, seed)
    o = ops.sl_sample(torch.as_tensor(off).cuda(), cap, seed)
    torch.cuda.synchronize()
    assert int(o["status"].item()) == 0
    np.testing.assert_array_equal(o["offsets"].cpu().numpy(), new_ref)
    n = int(new_ref[-1])
    np.testing.assert_array_equal(o["gather"][:n].cpu().numpy(), idx_ref)
    return off, o, n, idx_ref


def test_sl_sample_small_bit_exact():
    lens = [0, 1, 775, 776, 777, 4096, 8192, 3, 1500, 0]
    for seed in (0, 1, 2**63 + 12345):
        off, o, n, idx_ref = _sl_check(lens, 776, seed)
    # gathers: features (16-byte rows) and timestamps (8-byte rows) of the kept tokens
    from hstu_jagged_pointwise_b200 import ops
    T = int(off[-1])
    gen = torch.Generator().manual_seed(3)
    feats = torch.randn(T, 256, generator=gen).to(torch.bfloat16)
    ts = torch.as_tensor(W.increasing_ts(np.random.default_rng(4), T))
    gf = ops.gather_rows(feats.cuda(), o["gather"], n)
    gt = ops.gather_rows(ts.cuda(), o["gather"], n)
    torch.cuda.synchronize()
    assert torch.equal(gf.cpu(), feats[torch.as_tensor(idx_ref)])
    assert torch.equal(gt.cpu(), ts[torch.as_tensor(idx_ref)])


def test_sl_sample_training_and_large_batches_bit_exact():
    rng = np.random.default_rng(11)
    _sl_check(W.zipf_lengths(rng, 64), W.stochastic_length_cap(4096, 1.6), seed=5)     # raw training batch
    _sl_check(W.lognormal_lengths(rng, 262144), 776, seed=6)                            # 262,144 tokens


def test_sl_sample_flags_bad_batches():
    from hstu_jagged_pointwise_b200 import ops
    bad = torch.tensor([0, 10, 5, 20], dtype=torch.int32, device="cuda")       # a negative length
    o = ops.sl_sample(bad, 8, 1, out_capacity=100)
    torch.cuda.synchronize()
    assert int(o["status"].item()) == 1
    ok = torch.tensor([0, 10, 30], dtype=torch.int32, device="cuda")
    o = ops.sl_sample(ok, 8, 1, out_capacity=15)                              # needs 16 rows
    torch.cuda.synchronize()
    assert int(o["status"].item()) == 1


def test_pack_balanced_matches_oracle():
    from hstu_jagged_pointwise_b200 import ops
    rng = np.random.default_rng(12)
    for lens, R in ((rng.integers(16, 4096, size=300), 8), (np.full(64, 100), 4), (np.array([5]), 3),
                    (np.zeros(0, np.int64), 2), (W.lognormal_lengths(rng, 262144), 16)):
        off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        start, tokens, weights = oracle.pack_balanced(off, R)
        o = ops.pack_balanced(torch.as_tensor(off).cuda(), R)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(o["bin_seq_start"].cpu().numpy(), start)
        np.testing.assert_array_equal(o["bin_tokens"].cpu().numpy(), tokens)
        np.testing.assert_allclose(o["bin_weight"].cpu().numpy(), weights, rtol=1e-6, atol=0)


# ----------------------------------------------------------------------------
# the named workloads at full size
# ----------------------------------------------------------------------------

def test_training_sl_full_forward_backward():
    w = W.training_sl(seed=0)
    out, _, _ = run_layer(w, backward=True)
    ref = oracle.layer_bwd(w)
    _, o, _, _ = oracle.layer_fwd(w)
    st = storage_bwd(w)
    sf = storage_fwd(w)
    assert_bf16(out["y"], ref["y"], "y", st["y"])
    assert_bf16(out["o_pre"], o, "o_pre", sf["o_pre"])
    for k in ("dq", "dk", "dv", "du", "d_rab_pos", "d_rab_time"):
        assert_bf16(out[k], ref[k], k, st[k])
    assert_bf16(out["d_gamma"], ref["dgamma"], "d_gamma", st["dgamma"])
    assert_bf16(out["d_beta"], ref["dbeta"], "d_beta", st["dbeta"])


def _sample_rows(w, rng, per_seq=4, n_seq=12):
    off = w.offsets
    seqs = rng.choice(w.B, size=min(n_seq, w.B), replace=False)
    rows = []
    for b in seqs:
        L = int(off[b + 1] - off[b])
        if L == 0:
            continue
        picks = {0, L - 1} | set(rng.integers(0, L, size=per_seq).tolist())
        rows += [int(off[b]) + i for i in sorted(picks)]
    return np.array(sorted(rows), dtype=np.int64)


def test_mtgr_medium_sampled_rows():
    w = W.mtgr_medium(seed=0)
    out, _, _ = run_layer(w)
    rng = np.random.default_rng(2)
    rows = _sample_rows(w, rng)
    # make sure every segment kind is sampled: first real-time and candidate rows of a few users
    extra = []
    for b in range(6):
        s0 = int(w.offsets[b])
        S, R = int(w.n_static[b]), int(w.n_realtime[b])
        extra += [s0 + S - 1, s0 + S, s0 + S + R, int(w.offsets[b + 1]) - 1]
    rows = np.unique(np.concatenate([rows, np.array(extra, np.int64)]))
    y, o, _, _ = oracle.layer_fwd(w, rows)
    st = storage_fwd(w, rows)
    rt = torch.as_tensor(rows).cuda()
    assert_bf16(out["y"][rt], y, "y", st["y"])
    assert_bf16(out["o_pre"][rt], o, "o_pre", st["o_pre"])


def test_mfalcon_ranking_sampled_candidates():
    w = W.mfalcon_ranking(seed=0)
    out, _ = run_mfalcon(w)
    rng = np.random.default_rng(3)
    rows = np.unique(rng.integers(0, w.T, size=96)).astype(np.int64)
    y, o = oracle.mfalcon_layer(w, rows)
    st = storage_mfalcon(w, rows)
    rt = torch.as_tensor(rows).cuda()
    assert_bf16(out["y"][rt], y, "y", st["y"])
    assert_bf16(out["o_pre"][rt], o, "o_pre", st["o_pre"])


def _sub_workload(w, b):
    """Sequence b of w alone (sequences are independent)."""
    s0, s1 = int(w.offsets[b]), int(w.offsets[b + 1])
    ws = W.make_causal([s1 - s0], H=w.H, d=w.d, dtype=w.dtype, seed=0, alpha=w.alpha,
                       ts_list=[w.ts[s0:s1]], with_grad=True)
    for name in ("q", "k", "v", "u", "grad"):
        setattr(ws, name, getattr(w, name)[s0:s1])
    ws.rab_pos, ws.rab_time, ws.gamma, ws.beta = w.rab_pos, w.rab_time, w.gamma, w.beta
    return ws, s0, s1


def _golden_reduced(path):
    """name -> (exact, storage) arrays from a reduced-gradient golden file."""
    rows = {}
    with open(path) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, i, a, b = line.split()
            rows.setdefault(name, []).append((int(i), float(a), float(b)))
    out = {}
    for name, r in rows.items():
        r.sort()
        out[name] = (np.array([x[1] for x in r]), np.array([x[2] for x in r]))
    return out


def _check_seq_backward(out, w, b, label):
    """Every per-token backward output of sequence b of a batch against the oracle run on
    that sequence alone (sequences are independent)."""
    ws, s0, s1 = _sub_workload(w, b)
    ref = oracle.layer_bwd(ws)
    st = storage_bwd(ws)
    for k in ("dq", "dk", "dv", "du"):
        assert_bf16(out[k][s0:s1], ref[k], f"{k}[{label}]", st[k])
    return ws, ref, st


def test_large_layer_sampled_forward_and_full_size_backward():
    """The large layer (262,144 tokens, 165 sequences up to 7,585 long, 8 heads x 128) in the
    bench's launch configuration.  Forward: sampled rows.  Backward: the reduced gradients
    (d_rab_pos, d_rab_time, d_gamma, d_beta: sums over all 3.1e9 visible pairs or all tokens)
    against the fp64 oracle's values for this seeded batch (tests/golden, written by
    make_large_layer_reduced.py from the oracle alone), and every per-token gradient of the
    longest sequence, of the shortest and of one near 1000 tokens."""
    import os
    w = W.large_layer(seed=0)
    out, _, _ = run_layer(w, backward=True)
    rng = np.random.default_rng(4)
    rows = _sample_rows(w, rng, per_seq=3, n_seq=10)
    y, o, _, _ = oracle.layer_fwd(w, rows)
    st = storage_fwd(w, rows)
    rt = torch.as_tensor(rows).cuda()
    assert_bf16(out["y"][rt], y, "y", st["y"])
    assert_bf16(out["o_pre"][rt], o, "o_pre", st["o_pre"])
    gold = _golden_reduced(os.path.join(os.path.dirname(__file__), "golden",
                                        "large_layer_T262144_seed0_reduced.txt"))
    for k, name in (("d_rab_pos", "d_rab_pos"), ("d_rab_time", "d_rab_time"), ("d_gamma", "dgamma"),
                    ("d_beta", "dbeta")):
        exact, storage = gold[name]
        assert_bf16(out[k], exact, f"{k} (all 165 sequences)", storage)
    L = w.lengths
    for b in (int(np.argmax(L)), int(np.argmin(L)), int(np.argmin(np.abs(L - 1000)))):
        _check_seq_backward(out, w, b, f"seq {b}, L={int(L[b])}")


def test_large_layer_longest_sequence_as_its_own_batch():
    """The longest sequence of the large layer (7,585 tokens: the most query tiles per key
    tile and the most time-bucket runs) as a batch of one: all eight backward outputs."""
    w = W.large_layer(seed=0)
    b = int(np.argmax(w.lengths))
    ws, _, _ = _sub_workload(w, b)
    out, _, _ = run_layer(ws, backward=True)
    ref = oracle.layer_bwd(ws)
    st = storage_bwd(ws)
    _, o, _, _ = oracle.layer_fwd(ws)
    assert_bf16(out["y"], ref["y"], "y", st["y"])
    assert_bf16(out["o_pre"], o, "o_pre", storage_fwd(ws)["o_pre"])
    for k in ("dq", "dk", "dv", "du", "d_rab_pos", "d_rab_time"):
        assert_bf16(out[k], ref[k], k, st[k])
    assert_bf16(out["d_gamma"], ref["dgamma"], "d_gamma", st["dgamma"])
    assert_bf16(out["d_beta"], ref["dbeta"], "d_beta", st["dbeta"])


# ----------------------------------------------------------------------------
# device-side validation and error status
# ----------------------------------------------------------------------------

def test_invalid_offsets_set_device_status_and_recover():
    from hstu_jagged_pointwise_b200 import capi
    w = W.make_causal([100, 50], H=2, d=128, seed=13)
    out, layer, d = run_layer(w)
    bad = torch.tensor([0, 120, 150], dtype=torch.int32, device="cuda")   # length 120 > max 100
    layer.seq_offsets.copy_(bad)
    layer.forward(d["q"], d["k"], d["v"], d["u"], d["rab_pos"], d["rab_time"], d["gamma"], d["beta"])
    assert layer.check_device_error() == capi.HSTU_ERR_DEVICE_BOUNDS
    assert layer.check_device_error() == capi.HSTU_OK          # cleared
    layer.seq_offsets.copy_(torch.tensor([0, 100, 150], dtype=torch.int32, device="cuda"))
    out2 = layer.forward(d["q"], d["k"], d["v"], d["u"], d["rab_pos"], d["rab_time"], d["gamma"], d["beta"])
    torch.cuda.synchronize()
    assert layer.check_device_error() == capi.HSTU_OK
    assert torch.equal(out2["y"], out["y"])


def test_mtgr_bad_segments_flagged():
    from hstu_jagged_pointwise_b200 import capi
    w = W.make_mtgr([2], [10], [3], [4], H=2, d=128, seed=14)
    out, layer, d = run_layer(w)
    layer.n_static.fill_(30)       # static + real-time longer than the row
    layer.forward(d["q"], d["k"], d["v"], d["u"], d["rab_pos"], d["rab_time"], d["gamma"], d["beta"])
    assert layer.check_device_error() == capi.HSTU_ERR_DEVICE_BOUNDS
