"""Torch-facing binding of libhstu_b200: argument marshalling only.

Every function takes CUDA tensors, allocates outputs and workspace with torch
(unless the caller passes them), and calls one C-ABI entry point on the
current CUDA stream.  All computation runs in the library's kernels.

Layout (see include/hstu.h): q, k, v, u are jagged ``[T, H*d]`` row-major
tensors (bf16, or fp32 for the fp32 path), ``seq_offsets`` int32 ``[B+1]``,
``timestamps`` int64 ``[T]``, ``rab_pos`` fp32 ``[2P-1]``, ``rab_time`` fp32
``[nb]``, ``ln_gamma``/``ln_beta`` fp32 ``[H*d]``.
"""
from __future__ import annotations

import ctypes as C
from typing import Optional

import torch

from . import capi

_DTYPES = {torch.bfloat16: capi.HSTU_BF16, torch.float32: capi.HSTU_F32}


def _p(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def make_dims(T: int, B: int, H: int, d: int, dtype: torch.dtype, alpha: float, max_seq_len: int,
              n_pos: int = 256, n_tbuckets: int = 64, ln_eps: float = 1e-5) -> capi.HstuDims:
    return capi.HstuDims(B=B, T=T, H=H, d_qk=d, d_v=d, dtype=_DTYPES[dtype], n_pos=n_pos,
                         n_tbuckets=n_tbuckets, max_seq_len=max_seq_len, alpha=float(alpha),
                         ln_eps=float(ln_eps))


def make_mask(kind: str = "causal", n_static: Optional[torch.Tensor] = None,
              n_realtime: Optional[torch.Tensor] = None) -> capi.HstuMaskSpec:
    if kind == "causal":
        return capi.HstuMaskSpec(kind=capi.HSTU_MASK_CAUSAL, n_static=None, n_realtime=None)
    if kind == "mtgr":
        _need(n_static, "n_static", torch.int32)
        _need(n_realtime, "n_realtime", torch.int32)
        return capi.HstuMaskSpec(kind=capi.HSTU_MASK_MTGR, n_static=n_static.data_ptr(),
                                 n_realtime=n_realtime.data_ptr())
    if kind == "mfalcon_seq":
        # n_realtime[b] is the history length of row b; the rest of the row are candidates
        _need(n_realtime, "n_realtime", torch.int32)
        return capi.HstuMaskSpec(kind=capi.HSTU_MASK_MFALCON_SEQ, n_static=None,
                                 n_realtime=n_realtime.data_ptr())
    raise ValueError(f"unknown mask kind {kind!r}")


def attn_workspace_bytes(dims: capi.HstuDims, mask_kind: int, is_bwd: bool, n_groups: int = 1) -> int:
    if n_groups > 1:
        n = capi.LIB.hstu_attn_workspace_bytes_gln(C.byref(dims), mask_kind, n_groups, 1 if is_bwd else 0)
    else:
        n = capi.LIB.hstu_attn_workspace_bytes(C.byref(dims), mask_kind, 1 if is_bwd else 0)
    if n == 0:
        raise capi.HstuError(capi.HSTU_ERR_INVALID_ARG, "hstu_attn_workspace_bytes")
    return int(n)


def workspace(nbytes: int, device, zero: bool = True) -> torch.Tensor:
    """A byte buffer usable as workspace (torch allocations are 256-byte aligned); zeroed for
    the attention workspaces, whose control block must start clear."""
    if zero:
        return torch.zeros(nbytes, dtype=torch.uint8, device=device)
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


class Layer:
    """Holds the shapes, mask and workspace of one jagged HSTU attention layer.

    Reusing a Layer across steps keeps the workspace (and its status word)
    resident, so the forward/backward calls allocate only their outputs.
    """

    def __init__(self, seq_offsets: torch.Tensor, timestamps: torch.Tensor, H: int, d: int,
                 dtype: torch.dtype, alpha: float, max_seq_len: int, mask_kind: str = "causal",
                 n_static: Optional[torch.Tensor] = None, n_realtime: Optional[torch.Tensor] = None,
                 n_pos: int = 256, n_tbuckets: int = 64, ln_eps: float = 1e-5, n_groups: int = 1,
                 token_group: Optional[torch.Tensor] = None):
        """n_groups > 1 selects Group LayerNorm: token_group (uint8 [T]) names each token's
        group, and ln_gamma / ln_beta (and their gradients) are [n_groups, H*d]."""
        _need(seq_offsets, "seq_offsets", torch.int32)
        _need(timestamps, "timestamps", torch.int64)
        self.seq_offsets, self.timestamps = seq_offsets, timestamps
        self.B = seq_offsets.numel() - 1
        self.T = timestamps.numel()
        self.H, self.d, self.dtype = H, d, dtype
        self.n_static, self.n_realtime = n_static, n_realtime
        self.dims = make_dims(self.T, self.B, H, d, dtype, alpha, max_seq_len, n_pos, n_tbuckets, ln_eps)
        self.mask = make_mask(mask_kind, n_static, n_realtime)
        self.norm = None
        if n_groups > 1:
            _need(token_group, "token_group", torch.uint8)
            self.token_group = token_group
            self.norm = capi.HstuNormSpec(n_groups=int(n_groups), token_group=token_group.data_ptr())
        self.device = seq_offsets.device
        G = int(n_groups)
        n = attn_workspace_bytes(self.dims, self.mask.kind, False, G)
        if self.mask.kind != capi.HSTU_MASK_MFALCON_SEQ:   # the full-sequence M-FALCON mask is forward only
            n = max(n, attn_workspace_bytes(self.dims, self.mask.kind, True, G))
        self.ws = workspace(n, self.device)

    @property
    def D(self) -> int:
        return self.H * self.d

    def forward(self, q, k, v, u, rab_pos, rab_time, ln_gamma, ln_beta, out: Optional[dict] = None) -> dict:
        for t, n in ((q, "q"), (k, "k"), (v, "v"), (u, "u")):
            _need(t, n, self.dtype)
        for t, n in ((rab_pos, "rab_pos"), (rab_time, "rab_time"), (ln_gamma, "ln_gamma"), (ln_beta, "ln_beta")):
            _need(t, n, torch.float32)
        if out is None:
            out = dict(y=torch.empty_like(q), o_pre=torch.empty_like(q),
                       mean=torch.empty(self.T, dtype=torch.float32, device=self.device),
                       rstd=torch.empty(self.T, dtype=torch.float32, device=self.device))
        args = (_p(q), _p(k), _p(v), _p(u), _p(self.seq_offsets), _p(self.timestamps), _p(rab_pos), _p(rab_time),
                _p(ln_gamma), _p(ln_beta), _p(out["y"]), _p(out["o_pre"]), _p(out["mean"]), _p(out["rstd"]),
                _p(self.ws), self.ws.numel(), _stream())
        if self.norm is None:
            st = capi.LIB.hstu_attn_fwd(C.byref(self.dims), C.byref(self.mask), *args)
        else:
            st = capi.LIB.hstu_attn_fwd_gln(C.byref(self.dims), C.byref(self.mask), C.byref(self.norm), *args)
        capi.check(st, "hstu_attn_fwd")
        return out

    def backward(self, q, k, v, u, rab_pos, rab_time, ln_gamma, ln_beta, fwd: dict, d_o_pre,
                 out: Optional[dict] = None) -> dict:
        _need(d_o_pre, "d_o_pre", self.dtype)
        if out is None:
            out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                       du=torch.empty_like(u),
                       d_rab_pos=torch.empty_like(rab_pos), d_rab_time=torch.empty_like(rab_time),
                       d_gamma=torch.empty_like(ln_gamma), d_beta=torch.empty_like(ln_beta))
        args = (_p(q), _p(k), _p(v), _p(u), _p(self.seq_offsets), _p(self.timestamps), _p(rab_pos), _p(rab_time),
                _p(ln_gamma), _p(ln_beta), _p(fwd["y"]), _p(fwd["mean"]), _p(fwd["rstd"]), _p(d_o_pre),
                _p(out["dq"]), _p(out["dk"]), _p(out["dv"]), _p(out["du"]), _p(out["d_rab_pos"]),
                _p(out["d_rab_time"]), _p(out["d_gamma"]), _p(out["d_beta"]), _p(self.ws), self.ws.numel(),
                _stream())
        if self.norm is None:
            st = capi.LIB.hstu_attn_bwd(C.byref(self.dims), C.byref(self.mask), *args)
        else:
            st = capi.LIB.hstu_attn_bwd_gln(C.byref(self.dims), C.byref(self.mask), C.byref(self.norm), *args)
        capi.check(st, "hstu_attn_bwd")
        return out

    def backward_from_dy(self, q, k, v, rab_pos, rab_time, dy, out: Optional[dict] = None) -> dict:
        """Attention-only backward (hstu_attn_bwd_dy): dy = dL/dY in; dq, dk, dv and the
        bias-table gradients out."""
        _need(dy, "dy", self.dtype)
        if out is None:
            out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                       d_rab_pos=torch.empty_like(rab_pos), d_rab_time=torch.empty_like(rab_time))
        st = capi.LIB.hstu_attn_bwd_dy(C.byref(self.dims), C.byref(self.mask), _p(q), _p(k), _p(v),
                                       _p(self.seq_offsets), _p(self.timestamps), _p(rab_pos), _p(rab_time),
                                       _p(dy), _p(out["dq"]), _p(out["dk"]), _p(out["dv"]), _p(out["d_rab_pos"]),
                                       _p(out["d_rab_time"]), _p(self.ws), self.ws.numel(), _stream())
        capi.check(st, "hstu_attn_bwd_dy")
        return out

    def check_device_error(self) -> int:
        return int(capi.LIB.hstu_check_device_error(_p(self.ws), _stream()))


class HSTULayer:
    """One HSTU layer end to end on the library's kernels (Meta HSTU blog, section 3 formula):
        U, V, Q, K = Split(SiLU(X W1^T + b1))            (f1, phi1 = SiLU)
        Y = (SiLU(Q K^T + rab) * mask) V / alpha         (jagged pointwise attention)
        O_pre = Norm(Y) * U                              (LayerNorm or Group LayerNorm)
        out = O_pre W2^T + b2 (+ X when residual)        (f2)
    Parameters are passed per call as a dict: w1 [4D, d_model], b1 [4D] or None, w2 [d_model, D],
    b2 [d_model] or None, rab_pos, rab_time, ln_gamma, ln_beta (bf16 weights, fp32 the rest).
    Outputs and workspaces are allocated on the first call and reused by later calls, so the
    tensors a call returns are overwritten by the next call of the same kind."""

    def __init__(self, seq_offsets, timestamps, d_model: int, H: int, d: int, alpha: float, max_seq_len: int,
                 mask_kind: str = "causal", n_static=None, n_realtime=None, n_groups: int = 1, token_group=None,
                 residual: bool = True, n_pos: int = 256, n_tbuckets: int = 64, ln_eps: float = 1e-5):
        self.attn = Layer(seq_offsets, timestamps, H, d, torch.bfloat16, alpha, max_seq_len, mask_kind=mask_kind,
                          n_static=n_static, n_realtime=n_realtime, n_pos=n_pos, n_tbuckets=n_tbuckets,
                          ln_eps=ln_eps, n_groups=n_groups, token_group=token_group)
        self.d_model, self.D, self.residual = d_model, H * d, residual
        self._status = []
        self._buf = {}                                     # outputs reused from step to step

    def forward(self, x, params: dict) -> dict:
        """Returns out and the tensors the backward needs."""
        _need(x, "x", torch.bfloat16)
        b = self._buf
        f = b["f1"] = f1_fwd(x, params["w1"], params.get("b1"), self.D, out=b.get("f1"))
        a = b["attn"] = self.attn.forward(f["q"], f["k"], f["v"], f["u"], params["rab_pos"], params["rab_time"],
                                          params["ln_gamma"], params["ln_beta"], out=b.get("attn"))
        o = b["f2"] = f2_fwd(a["o_pre"], params["w2"], params.get("b2"), residual=x if self.residual else None,
                             out=b.get("f2"))
        self._status = [f["status"], o["status"]]
        return dict(out=o["out"], x=x, f1=f, attn=a)

    def backward(self, saved: dict, d_out, params: dict) -> dict:
        """Gradients of every input and parameter for d_out = dL/d out."""
        _need(d_out, "d_out", torch.bfloat16)
        f, a = saved["f1"], saved["attn"]
        b = self._buf
        g2 = b["b2"] = f2_bwd(a["o_pre"], params["w2"], d_out, out=b.get("b2"))
        ga = b["battn"] = self.attn.backward(f["q"], f["k"], f["v"], f["u"], params["rab_pos"], params["rab_time"],
                                             params["ln_gamma"], params["ln_beta"], a, g2["d_o_pre"],
                                             out=b.get("battn"))
        g1 = b["b1"] = f1_bwd(saved["x"], params["w1"], f["z"], ga["du"], ga["dv"], ga["dq"], ga["dk"],
                              dx_add=d_out if self.residual else None, out=b.get("b1"))
        self._status += [g2["status"], g1["status"]]
        return dict(dx=g1["dx"], dw1=g1["dw1"], db1=g1["db1"], dw2=g2["dw2"], db2=g2["db2"],
                    d_rab_pos=ga["d_rab_pos"], d_rab_time=ga["d_rab_time"], d_ln_gamma=ga["d_gamma"],
                    d_ln_beta=ga["d_beta"], d_o_pre=g2["d_o_pre"], dq=ga["dq"], dk=ga["dk"], dv=ga["dv"],
                    du=ga["du"])

    def check_device_error(self) -> int:
        """0, or the first nonzero status of the attention workspace or the projections' words."""
        st = self.attn.check_device_error()
        if st != 0:
            return st
        for t in self._status:
            v = int(t.item())
            if v != 0:
                return capi.HSTU_ERR_DEVICE_TIMEOUT if v & 2 else capi.HSTU_ERR_DEVICE_BOUNDS
        return 0


class MFalcon:
    """M-FALCON candidate scoring against cached history K/V (microbatch b_m)."""

    def __init__(self, hist_offsets, hist_ts, cand_offsets, cand_ts, H: int, d: int, alpha: float,
                 b_m: int, max_hist_len: int, max_cand_len: int, n_pos: int = 256, n_tbuckets: int = 64,
                 ln_eps: float = 1e-5):
        for t, n, dt in ((hist_offsets, "hist_offsets", torch.int32), (cand_offsets, "cand_offsets", torch.int32),
                         (hist_ts, "hist_ts", torch.int64), (cand_ts, "cand_ts", torch.int64)):
            _need(t, n, dt)
        self.hist_offsets, self.hist_ts, self.cand_offsets, self.cand_ts = hist_offsets, hist_ts, cand_offsets, cand_ts
        self.B = cand_offsets.numel() - 1
        self.b_m = int(b_m)
        self.H, self.d = H, d
        self.dims = capi.HstuMfalconDims(B=self.B, T_hist=hist_ts.numel(), T_cand=cand_ts.numel(), H=H, d_qk=d,
                                         d_v=d, dtype=capi.HSTU_BF16, n_pos=n_pos, n_tbuckets=n_tbuckets,
                                         max_hist_len=max_hist_len, max_cand_len=max_cand_len,
                                         alpha=float(alpha), ln_eps=float(ln_eps))
        n = capi.LIB.hstu_mfalcon_workspace_bytes(C.byref(self.dims), self.b_m)
        if n == 0:
            raise capi.HstuError(capi.HSTU_ERR_INVALID_ARG, "hstu_mfalcon_workspace_bytes")
        self.ws = workspace(int(n), cand_offsets.device)

    def score(self, hist_k, hist_v, cand_q, cand_k, cand_v, cand_u, rab_pos, rab_time, ln_gamma, ln_beta,
              out: Optional[dict] = None) -> dict:
        for t, n in ((hist_k, "hist_k"), (hist_v, "hist_v"), (cand_q, "cand_q"), (cand_k, "cand_k"),
                     (cand_v, "cand_v"), (cand_u, "cand_u")):
            _need(t, n, torch.bfloat16)
        if out is None:
            out = dict(y=torch.empty_like(cand_q), o_pre=torch.empty_like(cand_q))
        st = capi.LIB.hstu_mfalcon_score(
            C.byref(self.dims), _p(hist_k), _p(hist_v), _p(self.hist_offsets), _p(self.hist_ts), _p(cand_q),
            _p(cand_k), _p(cand_v), _p(cand_u), _p(self.cand_offsets), _p(self.cand_ts), _p(rab_pos),
            _p(rab_time), _p(ln_gamma), _p(ln_beta), self.b_m, _p(out["y"]), _p(out["o_pre"]), _p(self.ws),
            self.ws.numel(), _stream())
        capi.check(st, "hstu_mfalcon_score")
        return out

    def check_device_error(self) -> int:
        return int(capi.LIB.hstu_check_device_error(_p(self.ws), _stream()))


# ----------------------------------------------------------------------------
# the projections around the attention: f1 (X -> U, V, Q, K with SiLU) and f2
# ----------------------------------------------------------------------------

def _status(dev):
    return torch.empty(1, dtype=torch.int32, device=dev)    # the entry points set it to 0 first


def f1_fwd(x, w1, b1, D: int, save_z: bool = True, out: Optional[dict] = None) -> dict:
    """U, V, Q, K = split(SiLU(x @ w1.T + b1)), each [T, D]; z (pre-activation) kept for
    the backward when save_z.  w1 is [4D, d_in]; b1 fp32 [4D] or None."""
    _need(x, "x", torch.bfloat16)
    _need(w1, "w1", torch.bfloat16)
    T, d_in = x.shape
    if out is None:
        out = {n: torch.empty(T, D, dtype=torch.bfloat16, device=x.device) for n in ("u", "v", "q", "k")}
        out["z"] = torch.empty(T, 4 * D, dtype=torch.bfloat16, device=x.device) if save_z else None
        out["status"] = _status(x.device)
    st = capi.LIB.hstu_f1_fwd(T, d_in, D, _p(x), _p(w1), _p(b1), _p(out["u"]), _p(out["v"]), _p(out["q"]),
                              _p(out["k"]), _p(out.get("z")), _p(out.get("status")), _stream())
    capi.check(st, "hstu_f1_fwd")
    return out


def f2_fwd(o_pre, w2, b2=None, residual=None, out: Optional[dict] = None) -> dict:
    """out = o_pre @ w2.T + b2 (+ residual); w2 is [d_out, D]."""
    _need(o_pre, "o_pre", torch.bfloat16)
    _need(w2, "w2", torch.bfloat16)
    T, D = o_pre.shape
    d_out = w2.shape[0]
    if out is None:
        out = dict(out=torch.empty(T, d_out, dtype=torch.bfloat16, device=o_pre.device),
                   status=_status(o_pre.device))
    st = capi.LIB.hstu_f2_fwd(T, D, d_out, _p(o_pre), _p(w2), _p(b2), _p(residual), _p(out["out"]),
                              _p(out.get("status")), _stream())
    capi.check(st, "hstu_f2_fwd")
    return out


def f1_bwd(x, w1, z, du, dv, dq, dk, out: Optional[dict] = None, dx_add=None) -> dict:
    """dx [T, d_in] (bf16; plus dx_add when given), dw1 [4D, d_in] and db1 [4D] (fp32) of f1 for
    the U, V, Q, K gradients."""
    T, d_in = x.shape
    D = du.shape[1]
    if out is None:
        n = capi.LIB.hstu_f1_bwd_workspace_bytes(T, D)
        out = dict(dx=torch.empty_like(x), dw1=torch.empty(4 * D, d_in, dtype=torch.float32, device=x.device),
                   db1=torch.empty(4 * D, dtype=torch.float32, device=x.device), ws=workspace(n, x.device, False),
                   status=_status(x.device))
    st = capi.LIB.hstu_f1_bwd(T, d_in, D, _p(x), _p(w1), _p(z), _p(du), _p(dv), _p(dq), _p(dk), _p(dx_add),
                              _p(out["dx"]),
                              _p(out["dw1"]), _p(out["db1"]), _p(out["ws"]), out["ws"].numel(),
                              _p(out.get("status")), _stream())
    capi.check(st, "hstu_f1_bwd")
    return out


def f2_bwd(o_pre, w2, g, out: Optional[dict] = None) -> dict:
    """d_o_pre [T, D] (bf16), dw2 [d_out, D] and db2 [d_out] (fp32) of f2 for g = dL/d out."""
    T, D = o_pre.shape
    d_out = w2.shape[0]
    if out is None:
        n = capi.LIB.hstu_f2_bwd_workspace_bytes(T, d_out)
        out = dict(d_o_pre=torch.empty_like(o_pre), dw2=torch.empty(d_out, D, dtype=torch.float32, device=g.device),
                   db2=torch.empty(d_out, dtype=torch.float32, device=g.device), ws=workspace(n, g.device, False),
                   status=_status(g.device))
    st = capi.LIB.hstu_f2_bwd(T, D, d_out, _p(o_pre), _p(w2), _p(g), _p(out["d_o_pre"]), _p(out["dw2"]),
                              _p(out["db2"]), _p(out["ws"]), out["ws"].numel(), _p(out.get("status")), _stream())
    capi.check(st, "hstu_f2_bwd")
    return out


# ----------------------------------------------------------------------------
# the data step: Stochastic Length sampling, row gathers, token-balanced bins
# ----------------------------------------------------------------------------

def sl_sample(seq_offsets, cap: int, seed: int, out_capacity: Optional[int] = None) -> dict:
    """Stochastic Length: sequences longer than cap keep a uniform random subset of cap events
    in order.  Returns offsets [B+1], gather (input token index per output token, int32) and
    status (device int32, nonzero for an invalid batch or too small a capacity)."""
    _need(seq_offsets, "seq_offsets", torch.int32)
    B = seq_offsets.numel() - 1
    T = int(seq_offsets[-1].item())
    cap_out = T if out_capacity is None else int(out_capacity)
    dev = seq_offsets.device
    out = dict(offsets=torch.empty(B + 1, dtype=torch.int32, device=dev),
               gather=torch.empty(max(cap_out, 1), dtype=torch.int32, device=dev), status=_status(dev))
    st = capi.LIB.hstu_sl_sample(B, T, _p(seq_offsets), int(cap), C.c_uint64(int(seed) & (2**64 - 1)), cap_out,
                                 _p(out["offsets"]), _p(out["gather"]), _p(out["status"]), _stream())
    capi.check(st, "hstu_sl_sample")
    return out


def gather_rows(src: torch.Tensor, idx: torch.Tensor, n_rows: Optional[int] = None,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out[r] = src[idx[r]] for the first n_rows indices (rows of any contiguous tensor)."""
    if not src.is_cuda or not src.is_contiguous():
        raise ValueError("src must be a contiguous CUDA tensor")
    _need(idx, "idx", torch.int32)
    n = idx.numel() if n_rows is None else int(n_rows)
    if out is None:
        out = torch.empty((n,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    row_bytes = src[0].numel() * src.element_size() if src.shape[0] > 0 else out[0].numel() * out.element_size()
    st = capi.LIB.hstu_gather_rows(n, row_bytes, _p(src), src.shape[0], _p(idx), _p(out), _stream())
    capi.check(st, "hstu_gather_rows")
    return out


def pack_balanced(seq_offsets, n_bins: int) -> dict:
    """Token-balanced contiguous bins of sequences and their gradient weights."""
    _need(seq_offsets, "seq_offsets", torch.int32)
    B = seq_offsets.numel() - 1
    dev = seq_offsets.device
    out = dict(bin_seq_start=torch.empty(n_bins + 1, dtype=torch.int32, device=dev),
               bin_tokens=torch.empty(n_bins, dtype=torch.int32, device=dev),
               bin_weight=torch.empty(n_bins, dtype=torch.float32, device=dev))
    st = capi.LIB.hstu_pack_balanced(B, _p(seq_offsets), int(n_bins), _p(out["bin_seq_start"]),
                                     _p(out["bin_tokens"]), _p(out["bin_weight"]), _stream())
    capi.check(st, "hstu_pack_balanced")
    return out


def mfalcon_cache_history(seq_offsets, timestamps, n_history, k, v, hist_rows: Optional[int] = None,
                          out: Optional[dict] = None) -> dict:
    """KV cache for MFalcon.score from a full-sequence M-FALCON batch: the first
    n_history[b] rows of every user's [history ; candidates] row of k, v and
    timestamps, packed, with their offsets.  hist_rows (rows to allocate) defaults
    to sum(n_history), read on the host.  out["status"] (device int32) is nonzero
    when the batch was invalid or did not fit; nothing else is written then."""
    _need(seq_offsets, "seq_offsets", torch.int32)
    _need(timestamps, "timestamps", torch.int64)
    _need(n_history, "n_history", torch.int32)
    if k.dtype != v.dtype or k.shape != v.shape or k.dim() != 2 or not k.is_contiguous() or not v.is_contiguous():
        raise ValueError("k and v must be contiguous [T, H*d] tensors of one dtype")
    B = seq_offsets.numel() - 1
    if hist_rows is None:
        hist_rows = int(n_history.sum().item()) if B > 0 else 0
    dev = k.device
    if out is None:
        out = dict(hist_offsets=torch.empty(B + 1, dtype=torch.int32, device=dev),
                   hist_ts=torch.empty(hist_rows, dtype=torch.int64, device=dev),
                   hist_k=torch.empty(hist_rows, k.shape[1], dtype=k.dtype, device=dev),
                   hist_v=torch.empty(hist_rows, k.shape[1], dtype=k.dtype, device=dev),
                   status=torch.zeros(1, dtype=torch.int32, device=dev))
    st = capi.LIB.hstu_mfalcon_cache_history(
        B, k.shape[0], k.shape[1], _DTYPES[k.dtype], _p(seq_offsets), _p(timestamps), _p(n_history), _p(k),
        _p(v), out["hist_k"].shape[0], _p(out["hist_offsets"]), _p(out["hist_ts"]), _p(out["hist_k"]),
        _p(out["hist_v"]), _p(out["status"]), _stream())
    capi.check(st, "hstu_mfalcon_cache_history")
    return out


def debug_indices(seq_offsets, timestamps, mask_kind: str = "causal", n_static=None, n_realtime=None,
                  n_pos: int = 256, n_tbuckets: int = 64):
    """Per-pair (mask, rab_pos index, time bucket) from the kernels' own device functions."""
    _need(seq_offsets, "seq_offsets", torch.int32)
    _need(timestamps, "timestamps", torch.int64)
    L = (seq_offsets[1:] - seq_offsets[:-1]).to(torch.int64)
    po = torch.zeros(L.numel() + 1, dtype=torch.int64, device=seq_offsets.device)
    po[1:] = torch.cumsum(L * L, 0)
    n = int(po[-1].item())
    m = torch.zeros(n, dtype=torch.uint8, device=seq_offsets.device)
    pi = torch.zeros(n, dtype=torch.int16, device=seq_offsets.device)
    tb = torch.zeros(n, dtype=torch.int8, device=seq_offsets.device)
    kind = {"causal": capi.HSTU_MASK_CAUSAL, "mtgr": capi.HSTU_MASK_MTGR,
            "mfalcon_seq": capi.HSTU_MASK_MFALCON_SEQ}[mask_kind]
    st = capi.LIB.hstu_debug_indices(L.numel(), kind, _p(seq_offsets), _p(timestamps), _p(n_static),
                                     _p(n_realtime), n_pos, n_tbuckets, _p(po), _p(m), _p(pi), _p(tb), _stream())
    capi.check(st, "hstu_debug_indices")
    return m, pi, tb, po
