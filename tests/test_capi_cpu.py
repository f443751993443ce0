"""Host-side checks of the C-ABI library that need no GPU: it loads, exports every
symbol include/hstu.h declares, and rejects bad arguments before any launch."""
import ctypes as C
import os
import re

import pytest

from conftest import ROOT

capi = pytest.importorskip("hstu_jagged_pointwise_b200.capi")


def header_functions():
    src = open(os.path.join(ROOT, "include", "hstu.h")).read()
    return sorted(set(re.findall(r"HSTU_API\s+[\w\s\*]+?\b(hstu_\w+)\s*\(", src)))


def test_exports_match_header():
    names = header_functions()
    assert len(names) == 28, names
    assert set(names) == set(capi.EXPORTS)
    for n in names:
        assert hasattr(capi.LIB, n), n


def test_no_host_symbols_leak():
    out = os.popen(f"nm -D --defined-only {capi.LIB_PATH}").read().split("\n")
    exported = {l.split()[-1] for l in out if " T " in l}
    assert exported == set(capi.EXPORTS), exported - set(capi.EXPORTS)


def test_status_strings_and_version():
    assert capi.LIB.hstu_version().decode() == "0.1.0"
    for s in range(-6, 1):
        assert capi.status_string(s) != "unknown status"
    assert capi.status_string(-99) == "unknown status"


def dims(**kw):
    base = dict(B=4, T=436, H=2, d_qk=32, d_v=32, dtype=capi.HSTU_F32, n_pos=256, n_tbuckets=64,
                max_seq_len=255, alpha=255.0, ln_eps=1e-5)
    base.update(kw)
    return capi.HstuDims(**base)


def test_workspace_query():
    d = dims()
    n_f = capi.LIB.hstu_attn_workspace_bytes(C.byref(d), 0, 0)
    n_b = capi.LIB.hstu_attn_workspace_bytes(C.byref(d), 0, 1)
    assert n_f > 0 and n_b > n_f and n_f % 256 == 0
    assert capi.LIB.hstu_attn_workspace_bytes(None, 0, 0) == 0
    for bad in (dict(d_qk=48, d_v=48), dict(H=0), dict(alpha=0.0), dict(alpha=float("nan")),
                dict(n_pos=0), dict(n_pos=1025), dict(n_tbuckets=65), dict(d_qk=32, d_v=64),
                dict(dtype=7), dict(max_seq_len=-1)):
        assert capi.LIB.hstu_attn_workspace_bytes(C.byref(dims(**bad)), 0, 0) == 0, bad
    # bf16 supports 64 / 128 only
    assert capi.LIB.hstu_attn_workspace_bytes(C.byref(dims(dtype=capi.HSTU_BF16)), 0, 0) == 0
    assert capi.LIB.hstu_attn_workspace_bytes(C.byref(dims(dtype=capi.HSTU_BF16, d_qk=128, d_v=128)), 0, 0) > 0
    assert capi.LIB.hstu_attn_workspace_bytes(C.byref(dims()), 5, 0) == 0


def test_fwd_rejects_bad_arguments_before_launch():
    d = dims()
    m = capi.HstuMaskSpec(kind=0, n_static=None, n_realtime=None)
    nulls = [None] * 15
    # null dims / mask
    assert capi.LIB.hstu_attn_fwd(None, C.byref(m), *nulls, 0, None) == capi.HSTU_ERR_INVALID_ARG
    assert capi.LIB.hstu_attn_fwd(C.byref(d), None, *nulls, 0, None) == capi.HSTU_ERR_INVALID_ARG
    # unsupported width
    d2 = dims(d_qk=48, d_v=48)
    assert capi.LIB.hstu_attn_fwd(C.byref(d2), C.byref(m), *nulls, 0, None) == capi.HSTU_ERR_UNSUPPORTED
    # fp32 rows wider than 4096 (LayerNorm rows are held in registers)
    d3 = dims(dtype=capi.HSTU_F32, H=33, d_qk=128, d_v=128)
    assert capi.LIB.hstu_attn_fwd(C.byref(d3), C.byref(m), *nulls, 0, None) == capi.HSTU_ERR_UNSUPPORTED
    # MTGR without segment arrays
    m2 = capi.HstuMaskSpec(kind=1, n_static=None, n_realtime=None)
    assert capi.LIB.hstu_attn_fwd(C.byref(d), C.byref(m2), *nulls, 0, None) == capi.HSTU_ERR_INVALID_ARG
    # missing / small / misaligned workspace
    assert capi.LIB.hstu_attn_fwd(C.byref(d), C.byref(m), *nulls, 0, None) == capi.HSTU_ERR_WORKSPACE
    buf = (C.c_uint8 * 4096)()
    base = C.addressof(buf)
    aligned = (base + 255) // 256 * 256
    args = [None] * 14 + [C.c_void_p(aligned)]
    assert capi.LIB.hstu_attn_fwd(C.byref(d), C.byref(m), *args, 16, None) == capi.HSTU_ERR_WORKSPACE
    args = [None] * 14 + [C.c_void_p(aligned + 8)]
    assert capi.LIB.hstu_attn_fwd(C.byref(d), C.byref(m), *args, 2048, None) == capi.HSTU_ERR_WORKSPACE
    # enough workspace but null tensors
    args = [None] * 14 + [C.c_void_p(aligned)]
    assert capi.LIB.hstu_attn_fwd(C.byref(d), C.byref(m), *args, 2048, None) == capi.HSTU_ERR_INVALID_ARG
    # T == 0 is a no-op
    d0 = dims(B=0, T=0)
    assert capi.LIB.hstu_attn_fwd(C.byref(d0), C.byref(m), *args, 2048, None) == capi.HSTU_OK


def test_bwd_rejects_bad_arguments_before_any_cuda_call():
    """hstu_attn_bwd and hstu_attn_bwd_dy check every argument before their first CUDA call,
    so on a machine without a GPU each bad call returns its own status, not a CUDA error."""
    d = dims()
    m = capi.HstuMaskSpec(kind=0, n_static=None, n_realtime=None)
    nulls23, nulls14 = [None] * 23, [None] * 14
    assert capi.LIB.hstu_attn_bwd(None, C.byref(m), *nulls23, 0, None) == capi.HSTU_ERR_INVALID_ARG
    assert capi.LIB.hstu_attn_bwd(C.byref(d), None, *nulls23, 0, None) == capi.HSTU_ERR_INVALID_ARG
    assert capi.LIB.hstu_attn_bwd_dy(None, C.byref(m), *nulls14, 0, None) == capi.HSTU_ERR_INVALID_ARG
    d2 = dims(d_qk=48, d_v=48)
    assert capi.LIB.hstu_attn_bwd(C.byref(d2), C.byref(m), *nulls23, 0, None) == capi.HSTU_ERR_UNSUPPORTED
    m2 = capi.HstuMaskSpec(kind=1, n_static=None, n_realtime=None)
    assert capi.LIB.hstu_attn_bwd(C.byref(d), C.byref(m2), *nulls23, 0, None) == capi.HSTU_ERR_INVALID_ARG
    # missing or small workspace
    assert capi.LIB.hstu_attn_bwd(C.byref(d), C.byref(m), *nulls23, 0, None) == capi.HSTU_ERR_WORKSPACE
    need = capi.LIB.hstu_attn_workspace_bytes(C.byref(d), 0, 1)
    ws = (C.c_uint8 * (need + 256))()
    wsa = C.c_void_p((C.addressof(ws) + 255) // 256 * 256)
    assert capi.LIB.hstu_attn_bwd(C.byref(d), C.byref(m), *nulls23[:22], wsa, need - 256, None) == capi.HSTU_ERR_WORKSPACE
    # enough workspace: missing gradient outputs, then missing inputs (T > 0)
    assert capi.LIB.hstu_attn_bwd(C.byref(d), C.byref(m), *nulls23[:22], wsa, need, None) == capi.HSTU_ERR_INVALID_ARG
    grads = (C.c_float * 1024)()
    g = C.c_void_p((C.addressof(grads) + 15) // 16 * 16)
    args = [None] * 18 + [g, g, g, g] + [wsa]
    assert capi.LIB.hstu_attn_bwd(C.byref(d), C.byref(m), *args, need, None) == capi.HSTU_ERR_INVALID_ARG
    args_dy = [None] * 11 + [g, g] + [wsa]
    assert capi.LIB.hstu_attn_bwd_dy(C.byref(d), C.byref(m), *args_dy, need, None) == capi.HSTU_ERR_INVALID_ARG


def test_full_sequence_mfalcon_mask_is_forward_only():
    """The [history ; candidates] mask has a forward workspace, no backward, and needs n_realtime."""
    d = dims()
    assert capi.LIB.hstu_attn_workspace_bytes(C.byref(d), capi.HSTU_MASK_MFALCON_SEQ, 0) > 0
    assert capi.LIB.hstu_attn_workspace_bytes(C.byref(d), capi.HSTU_MASK_MFALCON_SEQ, 1) == 0
    buf = (C.c_int32 * 8)()
    m = capi.HstuMaskSpec(kind=capi.HSTU_MASK_MFALCON_SEQ, n_static=None, n_realtime=C.addressof(buf))
    nulls = [None] * 23
    assert capi.LIB.hstu_attn_bwd(C.byref(d), C.byref(m), *nulls, 0, None) == capi.HSTU_ERR_UNSUPPORTED
    # without the history lengths the forward is refused before any launch
    m0 = capi.HstuMaskSpec(kind=capi.HSTU_MASK_MFALCON_SEQ, n_static=None, n_realtime=None)
    assert capi.LIB.hstu_attn_fwd(C.byref(d), C.byref(m0), *([None] * 15), 0, None) == \
        capi.HSTU_ERR_INVALID_ARG
    assert capi.LIB.hstu_debug_indices(1, capi.HSTU_MASK_MFALCON_SEQ, C.addressof(buf), C.addressof(buf), None,
                                       None, 256, 64, C.addressof(buf), C.addressof(buf), C.addressof(buf),
                                       C.addressof(buf), None) == capi.HSTU_ERR_INVALID_ARG


def test_cache_producer_rejects_bad_arguments_before_launch():
    f = capi.LIB.hstu_mfalcon_cache_history
    buf = (C.c_int64 * 64)()
    a = C.addressof(buf)
    ok = [a] * 5   # seq_offsets, timestamps, n_history, k, v
    outs = [a] * 5  # hist_offsets, hist_ts, hist_k, hist_v, device_status
    assert f(-1, 0, 64, capi.HSTU_BF16, *ok, 0, *outs, None) == capi.HSTU_ERR_INVALID_ARG
    assert f(1, 4, 64, 7, *ok, 4, *outs, None) == capi.HSTU_ERR_INVALID_ARG            # dtype
    assert f(1, 4, 4, capi.HSTU_BF16, *ok, 4, *outs, None) == capi.HSTU_ERR_UNSUPPORTED  # 8-byte rows
    assert f(1, 4, 64, capi.HSTU_BF16, *ok, 4, a, a, a, a, None, None) == capi.HSTU_ERR_INVALID_ARG  # no status
    assert f(1, 4, 64, capi.HSTU_BF16, a, a, a, a + 8, a, 4, *outs, None) == capi.HSTU_ERR_INVALID_ARG  # k misaligned
    assert f(1, 4, 64, capi.HSTU_BF16, a, a, a, a, a, -1, *outs, None) == capi.HSTU_ERR_INVALID_ARG


def test_projections_reject_bad_arguments_before_launch():
    buf = (C.c_uint8 * 4096)()
    a = (C.addressof(buf) + 255) // 256 * 256          # 256-byte aligned host address (never dereferenced)
    f1 = capi.LIB.hstu_f1_fwd
    assert f1(-1, 64, 64, *([a] * 10), None) == capi.HSTU_ERR_INVALID_ARG
    assert f1(4, 60, 64, *([a] * 10), None) == capi.HSTU_ERR_UNSUPPORTED       # d_in not a multiple of 8
    assert f1(4, 64, 96, *([a] * 10), None) == capi.HSTU_ERR_UNSUPPORTED       # D not a multiple of 64
    assert f1(4, 64, 64, a, a, a + 8, *([a] * 7), None) == capi.HSTU_ERR_INVALID_ARG   # misaligned bias
    assert f1(4, 64, 64, None, *([a] * 7), None, None, None) == capi.HSTU_ERR_INVALID_ARG  # no x
    f2 = capi.LIB.hstu_f2_fwd
    assert f2(4, 64, 48, *([a] * 7)) == capi.HSTU_ERR_UNSUPPORTED             # d_out not a multiple of 32
    assert capi.LIB.hstu_f1_bwd_workspace_bytes(4, 48) == 0
    assert capi.LIB.hstu_f1_bwd_workspace_bytes(4, 4096) == 0                 # 4D above 8192
    assert capi.LIB.hstu_f1_bwd_workspace_bytes(4, 64) > 0
    assert capi.LIB.hstu_f2_bwd_workspace_bytes(4, 64) > 0
    assert capi.LIB.hstu_f1_bwd(4, 64, 64, *([a] * 12), 16, None, None) == capi.HSTU_ERR_WORKSPACE
    assert capi.LIB.hstu_f2_bwd(4, 64, 64, *([a] * 7), 16, None, None) == capi.HSTU_ERR_WORKSPACE


def test_data_step_rejects_bad_arguments_before_launch():
    buf = (C.c_uint8 * 4096)()
    a = (C.addressof(buf) + 255) // 256 * 256
    f = capi.LIB.hstu_sl_sample
    assert f(-1, 0, a, 8, 1, 0, a, a, a, None) == capi.HSTU_ERR_INVALID_ARG
    assert f(1, 4, a, 0, 1, 4, a, a, a, None) == capi.HSTU_ERR_INVALID_ARG      # cap < 1
    assert f(1, 4, a, 8, 1, 4, a, a, None, None) == capi.HSTU_ERR_INVALID_ARG   # no status word
    assert f(1, 4, a + 2, 8, 1, 4, a, a, a, None) == capi.HSTU_ERR_INVALID_ARG  # misaligned offsets
    g = capi.LIB.hstu_gather_rows
    assert g(-1, 16, a, 4, a, a, None) == capi.HSTU_ERR_INVALID_ARG
    assert g(4, 0, a, 4, a, a, None) == capi.HSTU_ERR_INVALID_ARG
    assert g(0, 16, None, 0, None, None, None) == capi.HSTU_OK                  # nothing to gather
    p = capi.LIB.hstu_pack_balanced
    assert p(4, a, 0, a, a, a, None) == capi.HSTU_ERR_INVALID_ARG               # no bins
    assert p(4, a, 2, a, None, a, None) == capi.HSTU_ERR_INVALID_ARG


def test_mfalcon_rejects_bad_arguments():
    d = capi.HstuMfalconDims(B=2, T_hist=10, T_cand=4, H=2, d_qk=128, d_v=128, dtype=capi.HSTU_BF16,
                             n_pos=256, n_tbuckets=64, max_hist_len=8, max_cand_len=4, alpha=9.0,
                             ln_eps=1e-5)
    assert capi.LIB.hstu_mfalcon_workspace_bytes(C.byref(d), 256) > 0
    assert capi.LIB.hstu_mfalcon_workspace_bytes(C.byref(d), 0) == 0
    nulls = [None] * 14
    assert capi.LIB.hstu_mfalcon_score(C.byref(d), *nulls, 0, None, None, None, 0, None) == \
        capi.HSTU_ERR_INVALID_ARG
    d.dtype = capi.HSTU_F32
    assert capi.LIB.hstu_mfalcon_score(C.byref(d), *nulls, 4, None, None, None, 0, None) == \
        capi.HSTU_ERR_UNSUPPORTED


def test_debug_indices_rejects_bad_arguments():
    assert capi.LIB.hstu_debug_indices(1, 0, None, None, None, None, 256, 64, None, None, None, None,
                                       None) == capi.HSTU_ERR_INVALID_ARG
    assert capi.LIB.hstu_debug_indices(1, 3, None, None, None, None, 256, 64, None, None, None, None,
                                       None) == capi.HSTU_ERR_INVALID_ARG
    assert capi.LIB.hstu_debug_indices(0, 0, None, None, None, None, 256, 64, None, None, None, None,
                                       None) == capi.HSTU_OK


def test_fwd_noalloc_rejects_oversized_problems_on_the_host():
    """The built-in scratch has a fixed size; larger problems are refused before any launch."""
    from hstu_jagged_pointwise_b200 import ops
    import torch
    dims = ops.make_dims(T=1 << 30, B=1, H=8, d=128, dtype=torch.bfloat16, alpha=1.0, max_seq_len=1 << 18)
    mask = ops.make_mask("causal")
    need = capi.LIB.hstu_attn_workspace_bytes(C.byref(dims), capi.HSTU_MASK_CAUSAL, 0)
    assert need > capi.NOALLOC_SCRATCH_BYTES
    st = capi.LIB.hstu_attn_fwd_noalloc(C.byref(dims), C.byref(mask), *([None] * 15), None)
    assert st == capi.HSTU_ERR_WORKSPACE
    st = capi.LIB.hstu_attn_fwd_noalloc(None, C.byref(mask), *([None] * 15), None)
    assert st == capi.HSTU_ERR_INVALID_ARG


def test_binding_fails_loudly_without_the_library(tmp_path):
    """No CPU fallback: with the shared library absent, importing the binding or the ops layer
    raises and names the missing file."""
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "hstu_jagged_pointwise_b200"
    pkg.mkdir()
    for f in ("__init__.py", "capi.py", "ops.py", "shard.py", "workloads.py"):
        shutil.copy(os.path.join(ROOT, "hstu_jagged_pointwise_b200", f), pkg / f)
    for mod in ("hstu_jagged_pointwise_b200.capi", "hstu_jagged_pointwise_b200.ops"):
        r = subprocess.run([sys.executable, "-c", f"import {mod}"], cwd=tmp_path, capture_output=True, text=True,
                           env={**os.environ, "PYTHONPATH": str(tmp_path)})
        assert r.returncode != 0 and "libhstu_b200.so is missing" in r.stderr, r.stderr[-800:]


def test_debug_wait_fault_checks_its_arguments():
    assert capi.LIB.hstu_debug_set_wait_fault(-1, 0) == capi.HSTU_ERR_INVALID_ARG
    assert capi.LIB.hstu_debug_set_wait_fault(1000, 2) == capi.HSTU_ERR_INVALID_ARG
    assert capi.LIB.hstu_debug_set_wait_fault(0, 0) == capi.HSTU_OK
    with capi.wait_fault(1000):
        pass                                   # host-side setting only: nothing launches
    assert capi.LIB.hstu_debug_set_wait_fault(0, 0) == capi.HSTU_OK
