"""hstu_attn_fwd_noalloc (the forward with the library's built-in scratch) against
hstu_attn_fwd (caller workspace) on the same inputs, through the C ABI, on two
calls in a row.  Collected last so that it also runs after every other GPU test."""
import ctypes as C

import pytest
import torch

from hstu_jagged_pointwise_b200 import capi, ops
from hstu_jagged_pointwise_b200 import workloads as W
from parity import dev

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _outputs(d, T):
    return dict(y=torch.empty_like(d["q"]), o_pre=torch.empty_like(d["q"]),
                mean=torch.empty(T, dtype=torch.float32, device="cuda"),
                rstd=torch.empty(T, dtype=torch.float32, device="cuda"))


def _args(d, o):
    return [_p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["u"]), _p(d["offsets"]), _p(d["ts"]),
            _p(d["rab_pos"]), _p(d["rab_time"]), _p(d["gamma"]), _p(d["beta"]),
            _p(o["y"]), _p(o["o_pre"]), _p(o["mean"]), _p(o["rstd"])]


def _case(kind, dtype):
    if kind == "causal":
        return W.make_causal([1, 127, 129, 300, 700], H=2, d=128, seed=31, random_affine=True, dtype=dtype)
    return W.make_mtgr([24, 2, 60], [100, 190, 40], [10, 0, 5], [20, 70, 9], H=2, d=64, seed=32,
                       random_affine=True, dtype=dtype)


@pytest.mark.parametrize("kind,dtype", [("causal", torch.bfloat16), ("mtgr", torch.bfloat16),
                                        ("causal", torch.float32)])
def test_fwd_noalloc_matches_workspace_entry_point(kind, dtype):
    w = _case(kind, dtype)
    d = dev(w)
    T = int(w.offsets[-1])
    dims = ops.make_dims(T, len(w.offsets) - 1, w.H, w.d, w.dtype, w.alpha, max(w.max_len, 1),
                         w.n_pos, w.n_tbuckets, w.eps)
    mask = ops.make_mask(w.kind, d.get("n_static"), d.get("n_realtime"))
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)

    # the existing entry point with a caller workspace
    ws = ops.workspace(ops.attn_workspace_bytes(dims, mask.kind, False), "cuda")
    ref = _outputs(d, T)
    st = capi.LIB.hstu_attn_fwd(C.byref(dims), C.byref(mask), *_args(d, ref), _p(ws), ws.numel(), stream)
    assert st == capi.HSTU_OK, capi.status_string(st)
    assert capi.LIB.hstu_check_device_error(_p(ws), stream) == capi.HSTU_OK

    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = _outputs(d, T)
        for t in out.values():
            t.fill_(float("nan"))
        status.fill_(-1)
        st = capi.LIB.hstu_attn_fwd_noalloc(C.byref(dims), C.byref(mask), *_args(d, out), _p(status), stream)
        assert st == capi.HSTU_OK, capi.status_string(st)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        # the same kernels on the same inputs, and no step of the forward depends on the
        # order of atomics: the results are the same bits
        for name in ("y", "o_pre", "mean", "rstd"):
            assert torch.equal(out[name], ref[name]), f"{name} (call {call}) differs from hstu_attn_fwd"


def test_fwd_noalloc_rejects_problems_beyond_its_scratch():
    """A problem whose work list does not fit the built-in scratch is refused before any
    launch with HSTU_ERR_WORKSPACE (the caller then needs hstu_attn_fwd and a workspace)."""
    w = _case("causal", torch.bfloat16)
    d = dev(w)
    T = int(w.offsets[-1])
    big = ops.make_dims(40_000_000, 1, 8, 128, torch.bfloat16, w.alpha, 1000, w.n_pos, w.n_tbuckets, w.eps)
    mask = ops.make_mask(w.kind, None, None)
    assert ops.attn_workspace_bytes(big, mask.kind, False) > capi.NOALLOC_SCRATCH_BYTES
    out = _outputs(d, T)
    for t in out.values():
        t.fill_(7.0)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = capi.LIB.hstu_attn_fwd_noalloc(C.byref(big), C.byref(mask), *_args(d, out), _p(status), stream)
    assert st == capi.HSTU_ERR_WORKSPACE, capi.status_string(st)
    torch.cuda.synchronize()
    assert int(status.item()) == -1                      # nothing ran
    assert all(bool((t == 7.0).all()) for t in out.values())
