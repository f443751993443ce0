"""Seeded synthetic inputs for jagged HSTU pointwise attention.

This module draws inputs only: sequence lengths, timestamps, segment sizes and
dense random tensors.  It holds none of the attention arithmetic, so both the
CUDA path and the fp64 oracle can be fed from it without sharing any of the
method's code.

Shapes follow the workloads described for HSTU and MTGR:
  * jagged (padding-free) layout: values are ``[T, H*d]`` row-major with
    ``offsets[B+1]`` (MTGR deep-dive, section 2 "user-granularity compression";
    section 6 "JaggedTensor + variable-length HSTU operator");
  * Stochastic Length: a sequence longer than ``N**(alpha/2)`` keeps a random
    subset of that many events (HSTU blog, section 3.4: alpha = 1.6 maps 4096
    to about 776);
  * MTGR user-aggregated rows: static profile tokens, a long-term behaviour
    sequence, real-time behaviours and K candidates (MTGR deep-dive section 2
    "dynamic mixed mask"; MTGR report section 3.1 "dynamic masking");
  * M-FALCON: cached history K/V plus candidates scored in microbatches of b_m
    (HSTU blog, sections 4.2-4.3).

Dense tensors come from a seeded torch CPU generator (N(0,1) unless stated),
structure from numpy PCG64 with the same seed.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

T0 = 1_700_000_000          # first timestamp, seconds
GAP_MEAN = 3600.0           # mean gap between events, seconds
N_POS = 256                 # rab_pos has 2*N_POS-1 entries
N_TBUCKETS = 64             # rab_time entries
RAB_STD = 0.02

MASK_CAUSAL = 0
MASK_MTGR = 1


@dataclass
class Workload:
    """One batch of synthetic inputs (torch CPU tensors / numpy arrays)."""
    name: str
    kind: str                      # "causal" | "mtgr" | "mfalcon" | "mfalcon_seq"
    dtype: torch.dtype             # element type of q/k/v/u (bf16 or fp32)
    H: int
    d: int
    alpha: float
    rab_pos: torch.Tensor          # fp32 [2P-1]
    rab_time: torch.Tensor         # fp32 [nb]
    gamma: torch.Tensor            # fp32 [D]
    beta: torch.Tensor             # fp32 [D]
    eps: float = 1e-5
    n_pos: int = N_POS
    n_tbuckets: int = N_TBUCKETS
    # self-attention layouts (causal / mtgr)
    offsets: Optional[np.ndarray] = None      # int32 [B+1]
    ts: Optional[np.ndarray] = None           # int64 [T]
    q: Optional[torch.Tensor] = None          # [T, H*d]
    k: Optional[torch.Tensor] = None
    v: Optional[torch.Tensor] = None
    u: Optional[torch.Tensor] = None
    n_static: Optional[np.ndarray] = None     # int32 [B] (mtgr)
    n_realtime: Optional[np.ndarray] = None   # int32 [B] (mtgr; history length for mfalcon_seq)
    grad: Optional[torch.Tensor] = None       # upstream gradient of o_pre [T, H*d]
    # M-FALCON layout
    hist_offsets: Optional[np.ndarray] = None
    hist_ts: Optional[np.ndarray] = None
    hist_k: Optional[torch.Tensor] = None
    hist_v: Optional[torch.Tensor] = None
    cand_offsets: Optional[np.ndarray] = None
    cand_ts: Optional[np.ndarray] = None
    cand_q: Optional[torch.Tensor] = None
    cand_k: Optional[torch.Tensor] = None
    cand_v: Optional[torch.Tensor] = None
    cand_u: Optional[torch.Tensor] = None
    b_m: int = 0
    # Group LayerNorm: gamma / beta are [n_groups, D] and token t uses row token_group[t]
    n_groups: int = 1
    token_group: Optional[np.ndarray] = None  # uint8 [T]
    meta: dict = field(default_factory=dict)

    @property
    def D(self) -> int:
        return self.H * self.d

    @property
    def B(self) -> int:
        off = self.offsets if self.offsets is not None else self.cand_offsets
        return len(off) - 1

    @property
    def T(self) -> int:
        off = self.offsets if self.offsets is not None else self.cand_offsets
        return int(off[-1])

    @property
    def lengths(self) -> np.ndarray:
        off = self.offsets if self.offsets is not None else self.cand_offsets
        return np.diff(off)

    @property
    def max_len(self) -> int:
        ln = self.lengths
        return int(ln.max()) if len(ln) else 0


# ----------------------------------------------------------------------------
# primitive draws
# ----------------------------------------------------------------------------

def _offsets(lengths) -> np.ndarray:
    off = np.zeros(len(lengths) + 1, dtype=np.int64)
    off[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    assert off[-1] < 2**31
    return off.astype(np.int32)


def increasing_ts(rng: np.random.Generator, n: int, start: int = T0) -> np.ndarray:
    """Strictly increasing int64 timestamps: gaps of 1 + floor(Exp(mean 3600))."""
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    gaps = 1 + np.floor(rng.exponential(GAP_MEAN, size=n)).astype(np.int64)
    gaps[0] = 0
    return start + np.cumsum(gaps)


def randn(gen: torch.Generator, shape, dtype: torch.dtype, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, dtype=torch.float32, device=gen.device)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def rab_tables(gen: torch.Generator, n_pos: int = N_POS, nb: int = N_TBUCKETS):
    return (randn(gen, (2 * n_pos - 1,), torch.float32, RAB_STD),
            randn(gen, (nb,), torch.float32, RAB_STD))


def ln_affine(gen: torch.Generator, D: int, random_affine: bool):
    if random_affine:
        g = 1.0 + randn(gen, (D,), torch.float32, 0.1)
        b = randn(gen, (D,), torch.float32, 0.1)
    else:
        g = torch.ones(D, dtype=torch.float32)
        b = torch.zeros(D, dtype=torch.float32)
    return g, b


# ----------------------------------------------------------------------------
# length distributions
# ----------------------------------------------------------------------------

def zipf_lengths(rng, B: int, exponent: float = 1.2, lo: int = 16, hi: int = 4096) -> np.ndarray:
    """P(L) proportional to L**-exponent on the integers [lo, hi]."""
    support = np.arange(lo, hi + 1, dtype=np.float64)
    p = support ** (-exponent)
    p /= p.sum()
    return rng.choice(np.arange(lo, hi + 1), size=B, p=p).astype(np.int64)


def stochastic_length_cap(n_max: int, sl_alpha: float) -> int:
    """Length kept by Stochastic Length: floor(N ** (alpha / 2))."""
    return int(np.floor(n_max ** (sl_alpha / 2.0)))


def stochastic_length_subsample(rng, ts: np.ndarray, cap: int) -> np.ndarray:
    """Keep a uniform random subset of ``cap`` events, in their original order."""
    if len(ts) <= cap:
        return ts
    keep = np.sort(rng.choice(len(ts), size=cap, replace=False))
    return ts[keep]


def lognormal_lengths(rng, total: int, median: float = 1024.0, sigma: float = 1.0,
                      lo: int = 32, hi: int = 8192) -> np.ndarray:
    out = []
    acc = 0
    while acc < total:
        L = int(np.clip(np.round(rng.lognormal(np.log(median), sigma)), lo, hi))
        if acc + L > total:
            L = total - acc
            if L < lo:
                break
        out.append(L)
        acc += L
    return np.asarray(out, dtype=np.int64)


# ----------------------------------------------------------------------------
# builders
# ----------------------------------------------------------------------------

def make_causal(lengths, H: int, d: int, dtype=torch.bfloat16, seed: int = 0,
                alpha: Optional[float] = None, ts_list=None, random_affine: bool = False,
                with_grad: bool = False, name: str = "causal") -> Workload:
    rng = np.random.Generator(np.random.PCG64(seed))
    gen = torch.Generator().manual_seed(seed)
    lengths = np.asarray(lengths, dtype=np.int64)
    if ts_list is None:
        ts_list = [increasing_ts(rng, int(L)) for L in lengths]
    offsets = _offsets(lengths)
    T = int(offsets[-1])
    D = H * d
    ts = np.concatenate(ts_list).astype(np.int64) if T else np.zeros(0, np.int64)
    q = randn(gen, (T, D), dtype)
    k = randn(gen, (T, D), dtype)
    v = randn(gen, (T, D), dtype)
    u = randn(gen, (T, D), dtype)
    rp, rt = rab_tables(gen)
    g, b = ln_affine(gen, D, random_affine)
    grad = randn(gen, (T, D), dtype) if with_grad else None
    if alpha is None:
        alpha = float(max(int(lengths.max()) if len(lengths) else 1, 1))
    return Workload(name=name, kind="causal", dtype=dtype, H=H, d=d, alpha=float(alpha),
                    rab_pos=rp, rab_time=rt, gamma=g, beta=b, offsets=offsets, ts=ts,
                    q=q, k=k, v=v, u=u, grad=grad)


def mtgr_user(rng, n_profile: int, n_long: int, n_rt: int, n_cand: int, start: int = T0):
    """Timestamps of one MTGR user-aggregated row.

    Layout: [profile (ts 0) | long-term behaviours | real-time behaviours | candidates].
    Candidate timestamps are drawn uniformly between the start of the real-time
    window (or one second after the last long-term event when there is none)
    and one hour after the last non-candidate event, in random order.
    """
    hist = increasing_ts(rng, n_long + n_rt, start)
    ts_prof = np.zeros(n_profile, dtype=np.int64)
    if n_rt > 0:
        lo = int(hist[n_long])
    else:
        lo = int(hist[-1]) + 1 if len(hist) else start
    last = int(hist[-1]) if len(hist) else start
    cand = rng.integers(lo, last + 3600 + 1, size=n_cand, dtype=np.int64)
    return np.concatenate([ts_prof, hist, cand])


def make_mtgr(n_profile, n_long, n_rt, n_cand, H: int, d: int, dtype=torch.bfloat16,
              seed: int = 0, alpha: Optional[float] = None, random_affine: bool = False,
              with_grad: bool = False, ts_list=None, name: str = "mtgr") -> Workload:
    rng = np.random.Generator(np.random.PCG64(seed))
    gen = torch.Generator().manual_seed(seed)
    n_profile = np.asarray(n_profile, dtype=np.int64)
    n_long = np.asarray(n_long, dtype=np.int64)
    n_rt = np.asarray(n_rt, dtype=np.int64)
    n_cand = np.asarray(n_cand, dtype=np.int64)
    lengths = n_profile + n_long + n_rt + n_cand
    if ts_list is None:
        ts_list = [mtgr_user(rng, int(a), int(b_), int(c), int(e))
                   for a, b_, c, e in zip(n_profile, n_long, n_rt, n_cand)]
    w = make_causal(lengths, H, d, dtype, seed + 1, alpha, ts_list, random_affine, with_grad, name)
    w.kind = "mtgr"
    w.n_static = (n_profile + n_long).astype(np.int32)
    w.n_realtime = n_rt.astype(np.int32)
    w.meta.update(n_profile=n_profile, n_long=n_long, n_cand=n_cand)
    return w


def make_mfalcon(n_hist, n_cand, H: int, d: int, dtype=torch.bfloat16, seed: int = 0,
                 b_m: int = 256, alpha: Optional[float] = None, random_affine: bool = False,
                 name: str = "mfalcon") -> Workload:
    """Cached history K/V per user plus candidates with request timestamps after it."""
    rng = np.random.Generator(np.random.PCG64(seed))
    gen = torch.Generator().manual_seed(seed)
    n_hist = np.asarray(n_hist, dtype=np.int64)
    n_cand = np.asarray(n_cand, dtype=np.int64)
    hist_ts, cand_ts = [], []
    for n, m in zip(n_hist, n_cand):
        h = increasing_ts(rng, int(n))
        last = int(h[-1]) if n > 0 else T0
        hist_ts.append(h)
        cand_ts.append(last + rng.integers(1, 3600 + 1, size=int(m), dtype=np.int64))
    ho, co = _offsets(n_hist), _offsets(n_cand)
    Th, Tc = int(ho[-1]), int(co[-1])
    D = H * d
    hk = randn(gen, (Th, D), dtype)
    hv = randn(gen, (Th, D), dtype)
    cq = randn(gen, (Tc, D), dtype)
    ck = randn(gen, (Tc, D), dtype)
    cv = randn(gen, (Tc, D), dtype)
    cu = randn(gen, (Tc, D), dtype)
    rp, rt = rab_tables(gen)
    g, b = ln_affine(gen, D, random_affine)
    if alpha is None:
        alpha = float(int(n_hist.max()) + 1 if len(n_hist) else 1)
    return Workload(name=name, kind="mfalcon", dtype=dtype, H=H, d=d, alpha=float(alpha),
                    rab_pos=rp, rab_time=rt, gamma=g, beta=b,
                    hist_offsets=ho, hist_ts=np.concatenate(hist_ts) if Th else np.zeros(0, np.int64),
                    hist_k=hk, hist_v=hv, cand_offsets=co,
                    cand_ts=np.concatenate(cand_ts) if Tc else np.zeros(0, np.int64),
                    cand_q=cq, cand_k=ck, cand_v=cv, cand_u=cu, b_m=b_m)


GLN_PROFILE, GLN_BEHAVIOUR, GLN_REALTIME, GLN_CANDIDATE = 0, 1, 2, 3


def with_group_norm(w: Workload, seed: int = 0, groups=None) -> Workload:
    """Group LayerNorm on a self-attention workload: one gamma/beta row per token
    source.  MTGR rows [profile | long-term behaviour | real-time | candidates] get
    groups 0..3 from their segment sizes; other workloads take `groups`, a uint8
    array [T] or a group count to draw uniform random ids from.  The affine rows are
    1 + N(0, 0.1) and N(0, 0.1) (distinct per group, so a routing error shows)."""
    gen = torch.Generator().manual_seed(seed + 505)
    if groups is None:
        assert w.kind == "mtgr", "token groups from segments need an MTGR workload"
        parts = []
        for b in range(w.B):
            L = int(w.offsets[b + 1] - w.offsets[b])
            npf = int(w.meta["n_profile"][b])
            S, R = int(w.n_static[b]), int(w.n_realtime[b])
            parts.append(np.concatenate([np.full(npf, GLN_PROFILE), np.full(S - npf, GLN_BEHAVIOUR),
                                         np.full(R, GLN_REALTIME), np.full(L - S - R, GLN_CANDIDATE)]))
        tg = np.concatenate(parts) if parts else np.zeros(0)
        G = 4
    elif np.isscalar(groups):
        G = int(groups)
        tg = np.random.Generator(np.random.PCG64(seed)).integers(0, G, size=w.T)
    else:
        tg = np.asarray(groups)
        G = int(tg.max()) + 1 if tg.size else 1
    w.n_groups = G
    w.token_group = tg.astype(np.uint8)
    w.gamma = 1.0 + randn(gen, (G, w.D), torch.float32, 0.1)
    w.beta = randn(gen, (G, w.D), torch.float32, 0.1)
    return w


def mfalcon_seq_from(w: Workload, seed: int = 0, name: str = "mfalcon_seq") -> Workload:
    """The same users as an M-FALCON workload, laid out as one jagged row per user:
    [history ; candidates].  History K/V and all candidate tensors are w's; the
    history Q and U (which the cached layout does not need) are drawn here."""
    gen = torch.Generator().manual_seed(seed)
    ho, co = np.asarray(w.hist_offsets, np.int64), np.asarray(w.cand_offsets, np.int64)
    n_hist, n_cand = np.diff(ho), np.diff(co)
    D = w.H * w.d
    hq = randn(gen, (int(ho[-1]), D), w.dtype)
    hu = randn(gen, (int(ho[-1]), D), w.dtype)
    rows_h = [np.arange(ho[b], ho[b + 1]) for b in range(len(n_hist))]
    rows_c = [np.arange(co[b], co[b + 1]) for b in range(len(n_cand))]

    def cat(hist, cand):
        parts = []
        for rh, rc in zip(rows_h, rows_c):
            parts.append(hist[torch.as_tensor(rh, dtype=torch.long)])
            parts.append(cand[torch.as_tensor(rc, dtype=torch.long)])
        return torch.cat(parts) if parts else hist[:0]

    ts = np.concatenate([np.concatenate([w.hist_ts[ho[b]:ho[b + 1]], w.cand_ts[co[b]:co[b + 1]]])
                         for b in range(len(n_hist))]) if len(n_hist) else np.zeros(0, np.int64)
    return Workload(name=name, kind="mfalcon_seq", dtype=w.dtype, H=w.H, d=w.d, alpha=w.alpha,
                    rab_pos=w.rab_pos, rab_time=w.rab_time, gamma=w.gamma, beta=w.beta,
                    offsets=_offsets(n_hist + n_cand).astype(np.int32), ts=ts.astype(np.int64),
                    q=cat(hq, w.cand_q), k=cat(w.hist_k, w.cand_k), v=cat(w.hist_v, w.cand_v),
                    u=cat(hu, w.cand_u), n_realtime=n_hist.astype(np.int32))


# ----------------------------------------------------------------------------
# the projections around the attention
# ----------------------------------------------------------------------------

@dataclass
class ProjWorkload:
    """Inputs of f1 (X -> U, V, Q, K) and f2 (O_pre -> out) and their upstream gradients.
    Weights are [out, in] with N(0, 1/fan_in) entries, so Z and out stay O(1); biases
    N(0, 0.1); activations and gradients N(0, 1); the residual is X (d_out = d_in)."""
    T: int
    d_in: int
    D: int
    d_out: int
    x: torch.Tensor          # [T, d_in]
    w1: torch.Tensor         # [4D, d_in]
    b1: torch.Tensor         # [4D] fp32
    o_pre: torch.Tensor      # [T, D]
    w2: torch.Tensor         # [d_out, D]
    b2: torch.Tensor         # [d_out] fp32
    dact: torch.Tensor       # [T, 4D]: gradients of U, V, Q, K side by side
    g_out: torch.Tensor      # [T, d_out]
    z: torch.Tensor          # [T, 4D]: a pre-activation input for the f1 backward
    name: str = "proj"


def make_projection(T: int, d_in: int, D: int, d_out: Optional[int] = None, seed: int = 0,
                    device: str = "cpu", dtype=torch.bfloat16, name: str = "proj") -> ProjWorkload:
    d_out = d_in if d_out is None else d_out
    gen = torch.Generator(device=device).manual_seed(seed + 606)
    return ProjWorkload(
        T=T, d_in=d_in, D=D, d_out=d_out,
        x=randn(gen, (T, d_in), dtype), w1=randn(gen, (4 * D, d_in), dtype, d_in ** -0.5),
        b1=randn(gen, (4 * D,), torch.float32, 0.1), o_pre=randn(gen, (T, D), dtype),
        w2=randn(gen, (d_out, D), dtype, D ** -0.5), b2=randn(gen, (d_out,), torch.float32, 0.1),
        dact=randn(gen, (T, 4 * D), dtype), g_out=randn(gen, (T, d_out), dtype),
        z=randn(gen, (T, 4 * D), dtype, 2.0), name=name)


@dataclass
class LayerWorkload:
    """Inputs of a whole HSTU layer: the attention workload (offsets, timestamps, masks, rab
    tables, LayerNorm affine) plus X [T, d_model], the f1 / f2 weights and dL/d out."""
    attn: Workload
    d_model: int
    x: torch.Tensor           # [T, d_model] bf16
    w1: torch.Tensor          # [4D, d_model] bf16
    b1: torch.Tensor          # [4D] fp32
    w2: torch.Tensor          # [d_model, D] bf16
    b2: torch.Tensor          # [d_model] fp32
    g_out: torch.Tensor       # [T, d_model] bf16


def make_layer(attn: Workload, d_model: int, seed: int = 0) -> LayerWorkload:
    """Adds layer inputs to an attention workload (its q, k, v, u are then produced by f1)."""
    gen = torch.Generator().manual_seed(seed + 707)
    D = attn.D
    return LayerWorkload(attn=attn, d_model=d_model, x=randn(gen, (attn.T, d_model), torch.bfloat16),
                         w1=randn(gen, (4 * D, d_model), torch.bfloat16, d_model ** -0.5),
                         b1=randn(gen, (4 * D,), torch.float32, 0.1),
                         w2=randn(gen, (d_model, D), torch.bfloat16, D ** -0.5),
                         b2=randn(gen, (d_model,), torch.float32, 0.1),
                         g_out=randn(gen, (attn.T, d_model), torch.bfloat16))


def projection_large(seed: int = 0, device: str = "cpu") -> ProjWorkload:
    """The large layer's projections: 262,144 tokens, d_model 1024 = 8 heads x 128."""
    return make_projection(262144, 1024, 1024, 1024, seed=seed, device=device, name="proj_T262144_d1024")


# ----------------------------------------------------------------------------
# the five named workloads
# ----------------------------------------------------------------------------

def tiny_fp32(seed: int = 0) -> Workload:
    """4 jagged sequences {17, 64, 100, 255}, 2 heads, d=32, fp32, causal, alpha = 255."""
    return make_causal([17, 64, 100, 255], H=2, d=32, dtype=torch.float32, seed=seed,
                       alpha=255.0, name="tiny_fp32_causal_B4_H2_d32")


def training_sl(seed: int = 0, B: int = 64, with_grad: bool = True) -> Workload:
    """64 Zipf(1.2) sequences in [16, 4096], Stochastic Length alpha=1.6 (cap 776),
    d_model 512 = 4 heads x 128, causal, bf16."""
    rng = np.random.Generator(np.random.PCG64(seed))
    raw = zipf_lengths(rng, B)
    cap = stochastic_length_cap(4096, 1.6)
    ts_list = [stochastic_length_subsample(rng, increasing_ts(rng, int(L)), cap) for L in raw]
    lengths = [len(t) for t in ts_list]
    w = make_causal(lengths, H=4, d=128, dtype=torch.bfloat16, seed=seed + 101, ts_list=ts_list,
                    with_grad=with_grad, name="training_sl_B64_H4_d128")
    w.meta.update(raw_lengths=raw, sl_cap=cap)
    return w


def mtgr_medium(seed: int = 0, B: int = 128) -> Workload:
    """128 MTGR users: 24 profile + U[200,3000] long-term (static), U{0..64} real-time,
    U{20..200} candidates; d_model 768 = 6 heads x 128, bf16."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n_long = rng.integers(200, 3000 + 1, size=B)
    n_rt = rng.integers(0, 64 + 1, size=B)
    n_cand = rng.integers(20, 200 + 1, size=B)
    return make_mtgr(np.full(B, 24), n_long, n_rt, n_cand, H=6, d=128, seed=seed + 202,
                     name="mtgr_medium_B128_H6_d128")


def mfalcon_ranking(seed: int = 0, users: int = 256, n: int = 2048, m: int = 1024,
                    b_m: int = 256) -> Workload:
    """256 users x 2048 cached history tokens, 1024 candidates each, b_m = 256,
    d_model 512 = 4 heads x 128, bf16, alpha = n + 1."""
    return make_mfalcon(np.full(users, n), np.full(users, m), H=4, d=128, seed=seed + 303,
                        b_m=b_m, alpha=float(n + 1), name="mfalcon_U256_n2048_m1024_bm256")


def large_layer(seed: int = 0, total: int = 262144, with_grad: bool = True) -> Workload:
    """Lognormal(median 1024, sigma 1) lengths in [32, 8192] summing to 256k tokens,
    d_model 1024 = 8 heads x 128, causal, bf16."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lengths = lognormal_lengths(rng, total)
    return make_causal(lengths, H=8, d=128, dtype=torch.bfloat16, seed=seed + 404,
                       with_grad=with_grad, name=f"large_layer_T{total}_H8_d128")
