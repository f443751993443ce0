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
    ("alpha_dropped_backward", "double a = silu(z) / alpha;", "double a = silu(z);"),
    ("dk_transposed_operand", "dkj[c] += dz * (double)qi[c];", "dkj[c] += dz * (double)kj[c];"),
    ("unbiased_variance",
     "        var /= D;\n        double rs = 1.0 / sqrt(var + eps);\n        for (int c = 0; c < D; c++) {\n            double ln",
     "        var /= (D - 1);\n        double rs = 1.0 / sqrt(var + eps);\n        for (int c = 0; c < D; c++) {\n            double ln"),
    ("layer_norm_grad_term_dropped", "dy[r * D + c] = rs * (gx[c] - m1 - xh[c] * m2);", "dy[r * D + c] = rs * (gx[c] - m1);"),
    ("time_grad_scaled", "lt[ti] += dz;", "lt[ti] += dz * 1.0001;"),
    ("mfalcon_positions_swapped", "z += (double)rab_pos[pos_index(n, j, P)];",
     "z += (double)rab_pos[pos_index(j, n, P)];"),
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
