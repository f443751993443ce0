"""Bounded device waits (the failure path of the pipelined kernels), exercised
without a fault.  Every main-loop wait of the tcgen05 attention forward and
backward, the M-FALCON scorer and the projection GEMM gives up after a limit,
records the timeout bit in the status word, drains what its CTA issued, frees
the tensor memory and returns.  The test hook hstu_debug_set_wait_fault sets a
short limit (about a millisecond) and makes each CTA's TMA producer withhold its
first tile load, so the waits for that tile run out.  The call must report
HSTU_ERR_DEVICE_TIMEOUT, and the next normal call on the same context must be
correct against the oracle and clean."""
import numpy as np
import pytest
import torch

import oracle
from hstu_jagged_pointwise_b200 import capi, ops
from hstu_jagged_pointwise_b200 import workloads as W
from parity import assert_bf16, dev, run_mfalcon, storage_bwd, storage_fwd, storage_mfalcon

pytestmark = pytest.mark.gpu

LIMIT = 2_000_000          # SM cycles (about 1 ms at 1.9 GHz)


def _layer(w, d):
    return ops.Layer(d["offsets"], d["ts"], w.H, w.d, w.dtype, w.alpha, max(w.max_len, 1))


def _fwd(layer, d):
    return layer.forward(d["q"], d["k"], d["v"], d["u"], d["rab_pos"], d["rab_time"], d["gamma"], d["beta"])


def _bwd(layer, d, f):
    return layer.backward(d["q"], d["k"], d["v"], d["u"], d["rab_pos"], d["rab_time"], d["gamma"], d["beta"], f,
                          d["grad"])


def test_attention_forward_and_backward_waits_run_out_and_recover():
    w = W.make_causal([300, 129, 700], H=2, d=128, seed=51, random_affine=True, with_grad=True)
    d = dev(w)
    layer = _layer(w, d)
    with capi.wait_fault(LIMIT):
        _fwd(layer, d)
        assert layer.check_device_error() == capi.HSTU_ERR_DEVICE_TIMEOUT
    assert layer.check_device_error() == capi.HSTU_OK                # read and cleared
    f = _fwd(layer, d)
    torch.cuda.synchronize()
    assert layer.check_device_error() == capi.HSTU_OK
    y, o, _, _ = oracle.layer_fwd(w)
    st = storage_fwd(w)
    assert_bf16(f["y"], y, "y after a timed-out forward", st["y"])
    assert_bf16(f["o_pre"], o, "o_pre after a timed-out forward", st["o_pre"])

    with capi.wait_fault(LIMIT):
        _bwd(layer, d, f)
        assert layer.check_device_error() == capi.HSTU_ERR_DEVICE_TIMEOUT
    g = _bwd(layer, d, f)
    torch.cuda.synchronize()
    assert layer.check_device_error() == capi.HSTU_OK
    ref = oracle.layer_bwd(w)
    sb = storage_bwd(w)
    for k in ("dq", "dk", "dv", "du", "d_rab_pos", "d_rab_time"):
        assert_bf16(g[k], ref[k], f"{k} after a timed-out backward", sb[k])


def test_wait_limit_alone_changes_nothing():
    """A limit far above any real wait, with no load withheld: clean, and the same bits."""
    w = W.make_causal([200, 64], H=2, d=64, seed=52)
    d = dev(w)
    layer = _layer(w, d)
    ref = {k: t.clone() for k, t in _fwd(layer, d).items()}
    with capi.wait_fault(4_000_000_000, withhold=False):
        got = _fwd(layer, d)
        torch.cuda.synchronize()
        assert layer.check_device_error() == capi.HSTU_OK
    for k in ("y", "o_pre"):
        assert torch.equal(got[k], ref[k]), k


def test_mfalcon_scorer_wait_runs_out_and_recovers():
    w = W.make_mfalcon([200, 300], [130, 5], H=2, d=128, seed=53, alpha=301.0)
    d = dev(w)
    lm, lc = int(np.diff(w.hist_offsets).max()), int(np.diff(w.cand_offsets).max())
    m = ops.MFalcon(d["hist_offsets"], d["hist_ts"], d["cand_offsets"], d["cand_ts"], w.H, w.d, w.alpha, w.b_m,
                    lm, lc)
    args = (d["hist_k"], d["hist_v"], d["cand_q"], d["cand_k"], d["cand_v"], d["cand_u"], d["rab_pos"],
            d["rab_time"], d["gamma"], d["beta"])
    with capi.wait_fault(LIMIT):
        m.score(*args)
        assert m.check_device_error() == capi.HSTU_ERR_DEVICE_TIMEOUT
    out, _ = run_mfalcon(w, d=d)
    y, o = oracle.mfalcon_layer(w)
    st = storage_mfalcon(w)
    assert_bf16(out["y"], y, "y after a timed-out scorer", st["y"])
    assert_bf16(out["o_pre"], o, "o_pre after a timed-out scorer", st["o_pre"])


def test_projection_gemm_wait_runs_out_and_recovers():
    w = W.make_projection(300, 224, 64, 224, seed=54)
    c = {n: getattr(w, n).cuda() for n in ("x", "w1", "b1")}
    with capi.wait_fault(LIMIT):
        f = ops.f1_fwd(c["x"], c["w1"], c["b1"], w.D)
        torch.cuda.synchronize()
        assert int(f["status"].item()) & 2, "the GEMM did not report its timed-out wait"
    f = ops.f1_fwd(c["x"], c["w1"], c["b1"], w.D)
    torch.cuda.synchronize()
    assert int(f["status"].item()) == 0
    z, u, v, q, k = oracle.f1_fwd(w.x, w.w1, w.b1, w.D)
    from parity import bf16
    for name, ref in (("z", z), ("u", u), ("v", v), ("q", q), ("k", k)):
        assert_bf16(f[name], ref, name, bf16(ref))
