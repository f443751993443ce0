"""fp64 CPU oracle for jagged HSTU pointwise attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  The CUDA library never calls it and shares no code
with it.  The arithmetic lives in ``hstu_oracle.c`` (plain C, double
precision, OpenMP over rows); this module only compiles it with gcc, converts
arrays and calls it through ctypes.

Parity pins (what ties each function to the pages rather than to itself) are
in ``tests/test_oracle_pins.py``; every function here is pinned.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hstu_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "libhstu_oracle.so")
_lock = threading.Lock()
_lib = None

MASK_CAUSAL = 0
MASK_MTGR = 1
MASK_MFSEQ = 2   # full-sequence M-FALCON: [history ; candidates], n_realtime = history length


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (double precision, no fast-math, no FMA contraction)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = C.CDLL(build())
            _declare(_lib)
    return _lib


_p = C.c_void_p
_i32 = C.c_int32
_i64 = C.c_int64
_f64 = C.c_double


def _declare(L):
    L.hstu_oracle_indices.argtypes = [_i32, _p, _p, _i32, _p, _p, _i32, _i32, _p, _p, _p, _p]
    L.hstu_oracle_attn_fwd.argtypes = [_i32, _p, _i32, _i32, _i32, _p, _p, _p, _p, _p, _i32, _p,
                                       _i32, _i32, _p, _p, _f64, _i64, _p, _p]
    L.hstu_oracle_ln_mul_fwd.argtypes = [_i64, _i32, _p, _p, _p, _p, _f64, _p, _p, _p]
    L.hstu_oracle_ln_mul_bwd.argtypes = [_i64, _i32, _p, _p, _p, _p, _f64, _p, _p, _p, _p, _p]
    L.hstu_oracle_attn_bwd.argtypes = [_i32, _p, _i32, _i32, _i32, _p, _p, _p, _p, _p, _i32, _p,
                                       _i32, _i32, _p, _p, _f64, _p, _p, _p, _p, _p, _p]
    L.hstu_oracle_mfalcon.argtypes = [_i32, _p, _p, _i32, _i32, _i32, _p, _p, _p, _p, _p, _p, _p,
                                      _p, _i32, _p, _i32, _f64, _i64, _p, _p]
    L.hstu_oracle_set_bf16_operands.argtypes = [C.c_int]
    L.hstu_oracle_num_threads.restype = C.c_int
    L.hstu_oracle_set_num_threads.argtypes = [C.c_int]


class bf16_operands:
    """Inside this context the oracle's attention (forward, backward, M-FALCON) rounds the
    operands a bf16 tensor-core implementation must hold in bf16 -- A = SiLU(z) before it
    multiplies V or dY, and dz before it multiplies K or Q -- to bf16, round to nearest
    even.  An error model used to derive tolerances, never a reference by itself."""

    def __enter__(self):
        lib().hstu_oracle_set_bf16_operands(1)
        return self

    def __exit__(self, *exc):
        lib().hstu_oracle_set_bf16_operands(0)
        return False


def num_threads() -> int:
    return int(lib().hstu_oracle_num_threads())


def set_num_threads(n: int) -> None:
    lib().hstu_oracle_set_num_threads(int(n))


# ----------------------------------------------------------------------------
# array helpers
# ----------------------------------------------------------------------------

def f32(x) -> np.ndarray:
    """Exact float32 copy of a bf16/fp32 torch tensor or numpy array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float32).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _c(x, dtype):
    return np.ascontiguousarray(np.asarray(x, dtype=dtype))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _kind(w) -> int:
    return {"mtgr": MASK_MTGR, "mfalcon_seq": MASK_MFSEQ}.get(w.kind, MASK_CAUSAL)


def _segs(w):
    if w.kind == "mtgr":
        return _c(w.n_static, np.int32), _c(w.n_realtime, np.int32)
    if w.kind == "mfalcon_seq":
        return np.zeros(len(w.n_realtime), np.int32), _c(w.n_realtime, np.int32)
    return None, None


# ----------------------------------------------------------------------------
# public functions (all return float64 numpy arrays)
# ----------------------------------------------------------------------------

def pair_offsets(offsets) -> np.ndarray:
    L = np.diff(np.asarray(offsets, dtype=np.int64))
    po = np.zeros(len(L) + 1, dtype=np.int64)
    po[1:] = np.cumsum(L * L)
    return po


def indices(offsets, ts, kind: int, n_static=None, n_rt=None, P: int = 256, nb: int = 64):
    """Per-pair (mask, pos index, time bucket) for every (b, i, j), flattened by pair_offsets."""
    off = _c(offsets, np.int32)
    tsa = _c(ts, np.int64)
    po = pair_offsets(off)
    n = int(po[-1])
    m = np.zeros(n, np.uint8)
    pi = np.zeros(n, np.int16)
    tb = np.zeros(n, np.int8)
    ns = None if n_static is None else _c(n_static, np.int32)
    nr = None if n_rt is None else _c(n_rt, np.int32)
    lib().hstu_oracle_indices(len(off) - 1, _ptr(off), _ptr(tsa), kind, _ptr(ns), _ptr(nr), P, nb,
                              _ptr(po), _ptr(m), _ptr(pi), _ptr(tb))
    return m, pi, tb, po


def attn_fwd_raw(offsets, H, dqk, dv, q, k, v, ts, rab_pos, rab_time, kind, n_static, n_rt, alpha,
                 rows=None, P=256, nb=64):
    off = _c(offsets, np.int32)
    q, k, v = f32(q), f32(k), f32(v)
    tsa = _c(ts, np.int64)
    rp, rt = f32(rab_pos), f32(rab_time)
    ns = None if n_static is None else _c(n_static, np.int32)
    nr = None if n_rt is None else _c(n_rt, np.int32)
    r = None if rows is None else _c(rows, np.int64)
    n = int(off[-1]) if r is None else len(r)
    y = np.zeros((n, H * dv), np.float64)
    lib().hstu_oracle_attn_fwd(len(off) - 1, _ptr(off), H, dqk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(tsa),
                               _ptr(rp), P, _ptr(rt), nb, kind, _ptr(ns), _ptr(nr), float(alpha),
                               0 if r is None else len(r), _ptr(r), _ptr(y))
    return y


def attn_fwd(w, rows=None, q=None, k=None, v=None):
    """Y = (sum_j mask * SiLU(q.k + rab) v_j) / alpha for the listed token rows (all by default)."""
    ns, nr = _segs(w)
    return attn_fwd_raw(w.offsets, w.H, w.d, w.d, w.q if q is None else q, w.k if k is None else k,
                        w.v if v is None else v, w.ts, w.rab_pos, w.rab_time, _kind(w), ns, nr,
                        w.alpha, rows, w.n_pos, w.n_tbuckets)


def ln_mul_fwd(y, u, gamma, beta, eps=1e-5):
    """o = LayerNorm(y) * gamma + beta, times u; returns (o, mean, rstd)."""
    y = _c(y, np.float64)
    n, D = y.shape
    u, g, b = f32(u), f32(gamma), f32(beta)
    o = np.zeros((n, D), np.float64)
    mu = np.zeros(n, np.float64)
    rs = np.zeros(n, np.float64)
    lib().hstu_oracle_ln_mul_fwd(n, D, _ptr(y), _ptr(u), _ptr(g), _ptr(b), float(eps), _ptr(o),
                                 _ptr(mu), _ptr(rs))
    return o, mu, rs


def ln_mul_bwd(y, u, gamma, beta, grad, eps=1e-5):
    """Returns (dy, du, dgamma, dbeta) for g = dL/d o."""
    y = _c(y, np.float64)
    n, D = y.shape
    u, g, b, gr = f32(u), f32(gamma), f32(beta), f32(grad)
    dy = np.zeros((n, D), np.float64)
    du = np.zeros((n, D), np.float64)
    dg = np.zeros(D, np.float64)
    db = np.zeros(D, np.float64)
    lib().hstu_oracle_ln_mul_bwd(n, D, _ptr(y), _ptr(u), _ptr(g), _ptr(b), float(eps), _ptr(gr),
                                 _ptr(dy), _ptr(du), _ptr(dg), _ptr(db))
    return dy, du, dg, db


def attn_bwd_raw(offsets, H, dqk, dv, q, k, v, ts, rab_pos, rab_time, kind, n_static, n_rt, alpha, dy,
                 P=256, nb=64):
    off = _c(offsets, np.int32)
    q, k, v = f32(q), f32(k), f32(v)
    tsa = _c(ts, np.int64)
    rp, rt = f32(rab_pos), f32(rab_time)
    ns = None if n_static is None else _c(n_static, np.int32)
    nr = None if n_rt is None else _c(n_rt, np.int32)
    dy = _c(dy, np.float64)
    T = int(off[-1])
    dq = np.zeros((T, H * dqk), np.float64)
    dk = np.zeros((T, H * dqk), np.float64)
    dvv = np.zeros((T, H * dv), np.float64)
    drp = np.zeros(2 * P - 1, np.float64)
    drt = np.zeros(nb, np.float64)
    lib().hstu_oracle_attn_bwd(len(off) - 1, _ptr(off), H, dqk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(tsa),
                               _ptr(rp), P, _ptr(rt), nb, kind, _ptr(ns), _ptr(nr), float(alpha), _ptr(dy),
                               _ptr(dq), _ptr(dk), _ptr(dvv), _ptr(drp), _ptr(drt))
    return dq, dk, dvv, drp, drt


def attn_bwd(w, dy):
    ns, nr = _segs(w)
    return attn_bwd_raw(w.offsets, w.H, w.d, w.d, w.q, w.k, w.v, w.ts, w.rab_pos, w.rab_time, _kind(w),
                        ns, nr, w.alpha, dy, w.n_pos, w.n_tbuckets)


def mfalcon(w, rows=None):
    """Per-candidate Y over cached history plus the candidate itself (rows = candidate indices)."""
    ho, co = _c(w.hist_offsets, np.int32), _c(w.cand_offsets, np.int32)
    hk, hv = f32(w.hist_k), f32(w.hist_v)
    cq, ck, cv = f32(w.cand_q), f32(w.cand_k), f32(w.cand_v)
    hts, cts = _c(w.hist_ts, np.int64), _c(w.cand_ts, np.int64)
    rp, rt = f32(w.rab_pos), f32(w.rab_time)
    r = None if rows is None else _c(rows, np.int64)
    n = int(co[-1]) if r is None else len(r)
    y = np.zeros((n, w.H * w.d), np.float64)
    lib().hstu_oracle_mfalcon(len(co) - 1, _ptr(ho), _ptr(co), w.H, w.d, w.d, _ptr(hk), _ptr(hv), _ptr(hts),
                              _ptr(cq), _ptr(ck), _ptr(cv), _ptr(cts), _ptr(rp), w.n_pos, _ptr(rt),
                              w.n_tbuckets, float(w.alpha), 0 if r is None else len(r), _ptr(r), _ptr(y))
    return y


# ----------------------------------------------------------------------------
# whole-layer conveniences
# ----------------------------------------------------------------------------

def gln_mul_fwd(y, u, gamma, beta, group, eps=1e-5):
    """Group LayerNorm times u (MTGR deep-dive section 2; MTGR report, GLN): token t is
    normalised over D as in ln_mul_fwd, with the affine row gamma[group[t]],
    beta[group[t]].  Rows of one group go through ln_mul_fwd together."""
    y = _c(y, np.float64)
    u, g, b = f32(u), f32(gamma), f32(beta)
    grp = np.asarray(group).astype(np.int64)
    n, D = y.shape
    o, mu, rs = np.zeros((n, D)), np.zeros(n), np.zeros(n)
    for k in np.unique(grp):
        r = np.nonzero(grp == k)[0]
        o[r], mu[r], rs[r] = ln_mul_fwd(y[r], u[r], g[k], b[k], eps)
    return o, mu, rs


def gln_mul_bwd(y, u, gamma, beta, group, grad, eps=1e-5):
    """Backward of gln_mul_fwd: (dy, du, dgamma [G, D], dbeta [G, D]); group k's affine
    gradients sum over its own tokens only (zero for a group with no tokens)."""
    y = _c(y, np.float64)
    u, g, b, gr = f32(u), f32(gamma), f32(beta), f32(grad)
    grp = np.asarray(group).astype(np.int64)
    n, D = y.shape
    dy, du = np.zeros((n, D)), np.zeros((n, D))
    dg, db = np.zeros(g.shape), np.zeros(b.shape)
    for k in np.unique(grp):
        r = np.nonzero(grp == k)[0]
        dy[r], du[r], dg[k], db[k] = ln_mul_bwd(y[r], u[r], g[k], b[k], gr[r], eps)
    return dy, du, dg, db


def norm_fwd(w, y, rows=None):
    """The layer's Norm(y) * u for the listed rows: LayerNorm, or Group LayerNorm when
    the workload names token groups."""
    sel = slice(None) if rows is None else np.asarray(rows)
    u = f32(w.u)[sel]
    if getattr(w, "n_groups", 1) > 1:
        return gln_mul_fwd(y, u, w.gamma, w.beta, np.asarray(w.token_group)[sel], w.eps)
    return ln_mul_fwd(y, u, w.gamma, w.beta, w.eps)


def norm_bwd(w, y, grad):
    if getattr(w, "n_groups", 1) > 1:
        return gln_mul_bwd(y, w.u, w.gamma, w.beta, w.token_group, grad, w.eps)
    return ln_mul_bwd(y, w.u, w.gamma, w.beta, grad, w.eps)


# ----------------------------------------------------------------------------
# the projections around the attention (Meta HSTU blog, section 3 formula):
# U, V, Q, K = Split(phi1(f1(X))) with phi1 = SiLU, O = f2(Norm(A V) * U)
# ----------------------------------------------------------------------------

def _as_f64(a):
    """float64 view of an input: bf16/fp32 tensors and arrays exactly, float64 arrays as they are."""
    if isinstance(a, np.ndarray) and a.dtype == np.float64:
        return a
    return np.asarray(f32(a), dtype=np.float64)


def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def f1_fwd(x, w1, b1, D):
    """Z = X W1^T + b1 in float64 (W1 stored [4D, d_in]); returns Z and the four column
    blocks of SiLU(Z) in the order U, V, Q, K."""
    z = _as_f64(x) @ _as_f64(w1).T
    if b1 is not None:
        z = z + _as_f64(b1)
    a = z * sigmoid(z)
    return z, a[:, :D], a[:, D:2 * D], a[:, 2 * D:3 * D], a[:, 3 * D:]


def f2_fwd(o_pre, w2, b2=None, residual=None):
    """out = O_pre W2^T + b2 (+ residual), float64 (W2 stored [d_out, D])."""
    o = _as_f64(o_pre) @ _as_f64(w2).T
    if b2 is not None:
        o = o + _as_f64(b2)
    if residual is not None:
        o = o + _as_f64(residual)
    return o


def f1_bwd(x, w1, z, du, dv, dq, dk):
    """dZ = [dU dV dQ dK] * SiLU'(Z), SiLU'(z) = s (1 + z (1 - s)); dX = dZ W1, dW1 = dZ^T X,
    db1 = column sums of dZ.  Returns (dz, dx, dw1, db1)."""
    z = _as_f64(z)
    s = sigmoid(z)
    dz = np.concatenate([_as_f64(du), _as_f64(dv), _as_f64(dq), _as_f64(dk)], axis=1) * s * (1 + z * (1 - s))
    return dz, dz @ _as_f64(w1), dz.T @ _as_f64(x), dz.sum(0)


def f2_bwd(o_pre, w2, g):
    """d_O_pre = G W2, dW2 = G^T O_pre, db2 = column sums of G for G = dL/d out."""
    g = _as_f64(g)
    return g @ _as_f64(w2), g.T @ _as_f64(o_pre), g.sum(0)


# ----------------------------------------------------------------------------
# Stochastic Length (HSTU blog, section 3.4) and token-balanced batches (MTGR
# deep-dive, section 3, contribution 3)
# ----------------------------------------------------------------------------

_SM_GAMMA = np.uint64(0x9E3779B97F4A7C15)


def splitmix64(state: int, n) -> np.ndarray:
    """Output n (n >= 1) of SplitMix64 from `state` (Steele, Lea and Flood, OOPSLA 2014):
    z = state + n * gamma, then the published xor-shift-multiply finaliser."""
    with np.errstate(over="ignore"):
        z = np.uint64(state) + np.asarray(n, dtype=np.uint64) * _SM_GAMMA
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


def sl_keys(seed: int, b: int, L: int) -> np.ndarray:
    """Random key of event i of sequence b: SplitMix64 output number b * 2^32 + i + 1."""
    return splitmix64(seed, np.uint64(b) * np.uint64(1 << 32) + np.arange(L, dtype=np.uint64) + np.uint64(1))


def sl_sample(offsets, cap: int, seed: int):
    """Stochastic Length: a sequence longer than cap keeps the cap events with the smallest
    keys (ties by index) -- a uniform random subset -- in their original order.  Returns
    (new offsets int32 [B+1], gather indices int64 into the input tokens)."""
    off = np.asarray(offsets, dtype=np.int64)
    new = [0]
    idx = []
    for b in range(len(off) - 1):
        L = int(off[b + 1] - off[b])
        if L <= cap:
            keep = np.arange(L)
        else:
            keys = sl_keys(seed, b, L)
            order = np.lexsort((np.arange(L), keys))      # by key, then by index
            keep = np.sort(order[:cap])
        idx.append(off[b] + keep)
        new.append(new[-1] + len(keep))
    gather = np.concatenate(idx) if idx else np.zeros(0, np.int64)
    return np.asarray(new, dtype=np.int32), gather.astype(np.int64)


def pack_balanced(offsets, n_bins: int):
    """Token-balanced contiguous batches: sequence b (tokens [s_b, s_b + L_b) of T) goes to
    bin floor((s_b + L_b / 2) * n_bins / T), clamped to n_bins - 1.  Returns (bin_seq_start
    [n_bins+1], bin_tokens [n_bins], weights [n_bins] = sequences in the bin / B, the factor
    that makes the weighted sum of per-bin mean gradients the mean over all sequences)."""
    off = np.asarray(offsets, dtype=np.int64)
    B = len(off) - 1
    T = int(off[-1])
    bins = np.zeros(B, np.int64)
    for b in range(B):
        mid2 = 2 * off[b] + (off[b + 1] - off[b])        # twice the midpoint, kept integral
        bins[b] = min(n_bins - 1, (mid2 * n_bins) // (2 * T)) if T > 0 else 0
    start = np.zeros(n_bins + 1, np.int64)
    for r in range(n_bins + 1):
        start[r] = int(np.searchsorted(bins, r, side="left"))
    tokens = np.array([off[start[r + 1]] - off[start[r]] for r in range(n_bins)], np.int64)
    weights = np.array([(start[r + 1] - start[r]) / B if B else 0.0 for r in range(n_bins)])
    return start.astype(np.int32), tokens, weights


def layer_fwd(w, rows=None):
    """(y, o_pre, mean, rstd) for the listed rows: attention, then Norm(y) * u."""
    y = attn_fwd(w, rows)
    o, mu, rs = norm_fwd(w, y, rows)
    return y, o, mu, rs


def layer_bwd(w):
    """Full backward of o_pre = Norm(attn(q,k,v)) * u for the upstream gradient w.grad."""
    y = attn_fwd(w)
    dy, du, dg, db = norm_bwd(w, y, w.grad)
    dq, dk, dv, drp, drt = attn_bwd(w, dy)
    return dict(y=y, dy=dy, du=du, dgamma=dg, dbeta=db, dq=dq, dk=dk, dv=dv, d_rab_pos=drp, d_rab_time=drt)


def mfalcon_layer(w, rows=None):
    y = mfalcon(w, rows)
    u = f32(w.cand_u) if rows is None else f32(w.cand_u)[np.asarray(rows)]
    o, _, _ = ln_mul_fwd(y, u, w.gamma, w.beta, w.eps)
    return y, o
