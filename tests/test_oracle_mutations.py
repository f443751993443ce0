"""The pins must catch plausible mistakes in the oracle.

Each case plants one mistake in a copy of the C oracle (a flipped sign, an off-by-one, a
dropped term, a transposed operand, a wrong mask or position rule), builds the copy in a
temporary directory and swaps it in for the oracle's library.  At least one pin of
``test_oracle_pins`` must then fail.  The oracle's own source and build are never touched.
"""
import ctypes as C
import inspect
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

# (name, text in the oracle's source, the planted mistake)
MUTATIONS = [
    ("pos_delta_sign", "int64_t dp = pos_j - pos_i;", "int64_t dp = pos_i - pos_j;"),
    ("bucket_off_by_one", "return b < nb - 1 ? b : nb - 1;", "return b < nb - 1 ? b + (b > 40) : nb - 1;"),
    ("realtime_excludes_self", "if (ci == 1) return cj == 0 || (cj == 1 && j <= i);",
     "if (ci == 1) return cj == 0 || (cj == 1 && j < i);"),
    ("candidate_filter_not_strict", "return cj != 2 && ts[j] < ts[i];", "return cj != 2 && ts[j] <= ts[i];"),
    ("full_sequence_candidates_see_candidates", "if (kind == ORACLE_MFSEQ) return cj != 2;",
     "if (kind == ORACLE_MFSEQ) return 1;"),
    ("full_sequence_candidate_misses_itself", "if (j == i) return 1;", "if (j == i) return kind != ORACLE_MFSEQ;"),
    ("candidate_position_own_index", "if ((kind == ORACLE_MTGR || kind == ORACLE_MFSEQ) && i >= S + R) return S + R;",
     "if ((kind == ORACLE_MTGR || kind == ORACLE_MFSEQ) && i >= S + R) return i;"),
    ("full_sequence_position_rule_dropped",
     "if ((kind == ORACLE_MTGR || kind == ORACLE_MFSEQ) && i >= S + R) return S + R;",
     "if (kind == ORACLE_MTGR && i >= S + R) return S + R;"),
    ("alpha_dropped_forward", "for (int c = 0; c < dv; c++) out[c] /= alpha;", ";"),
    ("silu_grad_wrong", "return s * (1.0 + z * (1.0 - s));", "return s * (1.0 + z * s);"),
    ("alpha_dropped_backward", "double a = operand(silu(z)) / alpha;", "double a = operand(silu(z));"),
    ("dk_transposed_operand", "dkj[c] += dzo * (double)qi[c];", "dkj[c] += dzo * (double)kj[c];"),
    ("bf16_model_dz_not_rounded", "double dzo = operand(dz);", "double dzo = dz;"),
    ("bf16_model_rounds_rab_sums", "lp[pi] += dz;", "lp[pi] += dzo;"),
    ("unbiased_variance",
     "        var /= D;\n        double rs = 1.0 / sqrt(var + eps);\n        for (int c = 0; c < D; c++) {\n            double ln",
     "        var /= (D - 1);\n        double rs = 1.0 / sqrt(var + eps);\n        for (int c = 0; c < D; c++) {\n            double ln"),
    ("layer_norm_grad_term_dropped", "dy[r * D + c] = rs * (gx[c] - m1 - xh[c] * m2);", "dy[r * D + c] = rs * (gx[c] - m1);"),
    ("time_grad_scaled", "lt[ti] += dz;", "lt[ti] += dz * 1.0001;"),
    ("mfalcon_positions_swapped", "z += (double)rab_pos[pos_index(n, j, P)];",
     "z += (double)rab_pos[pos_index(j, n, P)];"),
    ("mfalcon_self_term_dropped", "for (int64_t j = 0; j <= n; j++) {", "for (int64_t j = 0; j < n; j++) {"),
    ("mfalcon_self_value_from_history", ": cand_v + c * ldv + h * dv;", ": hist_v + h0 * ldv + h * dv;"),
    ("mfalcon_alpha_dropped", "for (int e = 0; e < dv; e++) out[e] /= alpha;", ";"),
    ("pos_grad_scaled", "lp[pi] += dz;", "lp[pi] += 0.5 * dz;"),
    ("static_sees_realtime", "if (ci == 0) return cj == 0;", "if (ci == 0) return cj <= 1;"),
]


def _pin_calls():
    """Every pin as a no-argument call; the slowest last, so a caught mistake ends early."""
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        if name == "test_backward_finite_differences":
            calls += [(f"{name}[{k}]", (lambda f=fn, k=k: f(k))) for k in ("causal", "mtgr")]
        else:
            calls.append((name, fn))
    calls.sort(key=lambda c: c[0] == "test_group_layer_norm_matches_torch_autograd")
    return calls


def _build_copy(src: str, d) -> C.CDLL:
    c_path, so_path = d / "hstu_oracle.c", d / "libhstu_oracle_mut.so"
    c_path.write_text(src)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                           "-fno-fast-math", "-o", str(so_path), str(c_path), "-lm"])
    lib = C.CDLL(str(so_path))
    oracle._declare(lib)
    return lib


def test_unmutated_copy_passes_every_pin(tmp_path, monkeypatch):
    """Control: a copy built the same way but left as it is passes every pin, so a failure
    below comes from the planted mistake and not from the swap."""
    monkeypatch.setattr(oracle, "_lib", _build_copy(open(oracle._SRC).read(), tmp_path))
    for name, call in _pin_calls():
        call()


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(name, old, new, tmp_path, monkeypatch):
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"the text to mutate for {name} is not unique in the oracle"
    monkeypatch.setattr(oracle, "_lib", _build_copy(src.replace(old, new), tmp_path))
    for pin_name, call in _pin_calls():
        try:
            call()
        except AssertionError:
            return
    pytest.fail(f"no pin caught the planted mistake {name}")


# ----------------------------------------------------------------------------
# the oracle's Python functions (Group LayerNorm, projections, Stochastic Length, packer)
# ----------------------------------------------------------------------------

PY_MUTATIONS = [
    ("gln_forward_one_affine_row", "o[r], mu[r], rs[r] = ln_mul_fwd(y[r], u[r], g[k], b[k], eps)",
     "o[r], mu[r], rs[r] = ln_mul_fwd(y[r], u[r], g[0], b[0], eps)"),
    ("gln_backward_one_affine_row", "dy[r], du[r], dg[k], db[k] = ln_mul_bwd(y[r], u[r], g[k], b[k], gr[r], eps)",
     "dy[r], du[r], dg[k], db[k] = ln_mul_bwd(y[r], u[r], g[0], b[0], gr[r], eps)"),
    ("norm_ignores_groups", 'if getattr(w, "n_groups", 1) > 1:\n        return gln_mul_fwd',
     'if False:\n        return gln_mul_fwd'),
    ("f1_split_q_k_swapped", "return z, a[:, :D], a[:, D:2 * D], a[:, 2 * D:3 * D], a[:, 3 * D:]",
     "return z, a[:, :D], a[:, D:2 * D], a[:, 3 * D:], a[:, 2 * D:3 * D]"),
    ("f1_bias_dropped", "z = z + _as_f64(b1)", "z = z"),
    ("f1_silu_grad_wrong", "* s * (1 + z * (1 - s))", "* s * (1 + z * s)"),
    ("f2_residual_dropped", "o = o + _as_f64(residual)", "o = o"),
    ("f2_bias_grad_mean", "return g @ _as_f64(w2), g.T @ _as_f64(o_pre), g.sum(0)",
     "return g @ _as_f64(w2), g.T @ _as_f64(o_pre), g.mean(0)"),
    ("splitmix64_constant", "np.uint64(0xBF58476D1CE4E5B9)", "np.uint64(0xBF58476D1CE4E5B8)"),
    ("sl_kept_events_out_of_order", "keep = np.sort(order[:cap])", "keep = order[:cap]"),
    ("pack_bin_by_start", "mid2 = 2 * off[b] + (off[b + 1] - off[b])", "mid2 = 2 * off[b]"),
    ("pack_weights_by_tokens", "weights = np.array([(start[r + 1] - start[r]) / B if B else 0.0",
     "weights = np.array([(tokens[r]) / T if B else 0.0"),
]


def _mutated_module(src: str):
    import types
    mod = types.ModuleType("oracle_mutated")
    mod.__file__ = oracle.__file__
    exec(compile(src, oracle.__file__, "exec"), mod.__dict__)
    mod._lib = oracle.lib()
    return mod


def test_unmodified_python_copy_passes_every_pin(monkeypatch):
    monkeypatch.setattr(pins, "oracle", _mutated_module(open(oracle.__file__).read()))
    for name, call in _pin_calls():
        call()


@pytest.mark.parametrize("name,old,new", PY_MUTATIONS, ids=[m[0] for m in PY_MUTATIONS])
def test_pins_catch_planted_python_mistake(name, old, new, monkeypatch):
    src = open(oracle.__file__).read()
    assert src.count(old) == 1, f"the text to mutate for {name} is not unique in the oracle"
    monkeypatch.setattr(pins, "oracle", _mutated_module(src.replace(old, new)))
    for pin_name, call in _pin_calls():
        try:
            call()
        except Exception:
            return
    pytest.fail(f"no pin caught the planted mistake {name}")
