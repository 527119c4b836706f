"""Plausible mistakes planted in a copy of the oracle each fail at least one
of its pins.

Each case copies oracle/ttt_oracle.c and oracle/ttt_oracle.py into a
temporary directory, changes one thing (a sign, a dropped term, a transposed
index, a state read at the wrong moment, a dropped stride, a gate without
tanh, the reverse pass on the wrong input), builds that copy with gcc and
runs the pins of tests/test_oracle_pins.py against it.  The unchanged copy
passes them all (the same pins run on the real oracle in that file).
"""
import importlib.util
import os
import re
import shutil

import pytest

import test_oracle_pins as P

ORACLE_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle")


def _in_function(src: str, fname: str, old: str, new: str, all_in_body: bool = False) -> str:
    """Replace `old` by `new` inside the body of C function `fname` (first
    occurrence, or every occurrence in that body)."""
    m = re.search(r"\n[\w ]+\b" + re.escape(fname) + r"\(", src)
    assert m, fname
    start = src.index("{", m.end())
    depth, i = 0, start
    while True:   # the matching closing brace
        depth += {"{": 1, "}": -1}.get(src[i], 0)
        if depth == 0:
            break
        i += 1
    body = src[start:i + 1]
    pat = re.escape(old).replace(r"\ ", r"\s+").replace(r"\n", r"\s*")
    new_body, n = re.subn(pat, new, body, count=0 if all_in_body else 1)
    assert n >= 1, (fname, old)
    return src[:start] + new_body + src[i + 1:]


def _py(old: str, new: str):
    def f(src):
        assert src.count(old) == 1, old
        return src.replace(old, new)
    return f


C_MISTAKES = {
    "GELU' without the a*phi(a) term": ("ttt_ref_gelu_prime", "return Phi + a * phi;", "return Phi;"),
    "GELU with tanh in place of erf": ("ttt_ref_gelu", "erf(a / sqrt(2.0))", "tanh(a / sqrt(2.0))"),
    "dl/dW2 without its factor 2": ("ttt_ref_inner_loss_grad", "2.0 * e[j] * g[i]", "e[j] * g[i]"),
    "transposed W2 in the backward pass": ("ttt_ref_inner_loss_grad", "W2[(size_t)j * m + i]",
                                           "W2[(size_t)i * d + j]"),
    "per-token update with the wrong sign": ("ttt_ref_scan_per_token", "W2[p] -= eta * G2[p];",
                                             "W2[p] += eta * G2[p];"),
    "chunk update with the wrong sign": ("ttt_ref_scan_chunked", "W1[p] -= eta * G1[p];", "W1[p] += eta * G1[p];"),
    "chunk gradients at the running state": ("ttt_ref_scan_chunked", "ttt_ref_inner_loss_grad(d, m, W1c, W2c,",
                                             "ttt_ref_inner_loss_grad(d, m, W1, W2,"),
    "z read with the chunk-start state (before the update at b = 1)": (
        "ttt_ref_scan_chunked", "if (zmode == 0) ttt_ref_mlp_apply(d, m, W1, W2,",
        "if (zmode == 0) ttt_ref_mlp_apply(d, m, W1c, W2c,"),
    "reverse walk ignored in the chunk form": ("ttt_ref_scan_chunked", "const int t = reverse ? (T - 1 - n) : n;",
                                               "const int t = n;"),
    "head stride of K dropped in the multi-head driver": ("ttt_ref_scan_heads", "K + h * sT", "K"),
}

PY_MISTAKES = {
    "gate without tanh": _py("np.tanh(_f64(alpha)) * _f64(Z)", "_f64(alpha) * _f64(Z)"),
    "reverse pass on X instead of X'": _py('''        out["Xp"] = Xp
        src = Xp
    else:
        src = _f64(X)
    Zr, W1r, W2r = direction(''', '''        out["Xp"] = Xp
        src = _f64(X)
    else:
        src = _f64(X)
    Zr, W1r, W2r = direction('''),
    "per-head projection transposed": _py('np.einsum("hed,htd->hte", theta, X)', 'np.einsum("hde,htd->hte", theta, X)'),
    "full-width projection transposed": _py("_f64(X[r0:r0 + row_block]) @ theta.T",
                                            "_f64(X[r0:r0 + row_block]) @ theta"),
}

PINS = [
    P.test_gelu_matches_normal_cdf_table,
    P.test_gelu_and_derivative_against_library_and_fd,
    lambda: P.test_inner_gradient_central_differences(2),
    P.test_inner_gradient_matches_autograd,
    lambda: P.test_scan_matches_autograd_brute_force(1, 7),
    lambda: P.test_scan_matches_autograd_brute_force(3, 7),
    lambda: P.test_primal_matches_dual_form(4, 37),
    P.test_chunk_of_one_is_the_per_token_rule,
    P.test_eta_zero_closed_form,
    P.test_heads_equal_single_head_runs,
    P.test_gate_identity_at_alpha_zero_and_init_value,
    P.test_bidirectional_is_forward_then_reverse_on_gated_output,
    P.test_full_mode_with_block_diagonal_theta_equals_per_head_mode,
]


def _oracle_copy(tmp_path, name, c_edit=None, py_edit=None):
    d = tmp_path / name
    d.mkdir()
    c_src = open(os.path.join(ORACLE_DIR, "ttt_oracle.c")).read()
    py_src = open(os.path.join(ORACLE_DIR, "ttt_oracle.py")).read()
    if c_edit:
        c_src = c_edit(c_src)
    if py_edit:
        py_src = py_edit(py_src)
    (d / "ttt_oracle.c").write_text(c_src)
    (d / "ttt_oracle.py").write_text(py_src)
    spec = importlib.util.spec_from_file_location("ttt_oracle_" + name, str(d / "ttt_oracle.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def _failing_pins(mod) -> int:
    saved = P.O
    P.O = mod
    try:
        failed = 0
        for pin in PINS:
            try:
                with pytest.MonkeyPatch.context():
                    pin()
            except (AssertionError, ValueError, FloatingPointError):
                failed += 1
                break   # one is enough
        return failed
    finally:
        P.O = saved


@pytest.fixture(scope="module")
def gcc():
    if not shutil.which("gcc"):
        pytest.skip("gcc not found")


def test_unchanged_copy_passes_every_pin(tmp_path, gcc):
    assert _failing_pins(_oracle_copy(tmp_path, "unchanged")) == 0


@pytest.mark.parametrize("what", sorted(C_MISTAKES))
def test_planted_mistake_in_the_c_recurrence_fails_a_pin(tmp_path, gcc, what):
    fname, old, new = C_MISTAKES[what]
    mod = _oracle_copy(tmp_path, "c%d" % sorted(C_MISTAKES).index(what),
                       c_edit=lambda s: _in_function(s, fname, old, new, all_in_body=True))
    assert _failing_pins(mod) >= 1, what


@pytest.mark.parametrize("what", sorted(PY_MISTAKES))
def test_planted_mistake_in_the_layer_logic_fails_a_pin(tmp_path, gcc, what):
    mod = _oracle_copy(tmp_path, "p%d" % sorted(PY_MISTAKES).index(what), py_edit=PY_MISTAKES[what])
    assert _failing_pins(mod) >= 1, what
