"""The oracle's pins catch plausible mistakes in the oracle.

Each case plants one mistake in a copy of the oracle: a dropped term, a wrong sign, a wrong
index or operand, the wrong weight, or the wrong order of the apply and update steps. It
then runs the pins of test_oracle_pins.py against the copy, cheapest first, and requires
that at least one of them fails. The C++ per-token evolver is copied, edited and built in a
temporary folder. The numpy In-Place oracle and the PyTorch TTT-MLP oracle are edited as
source text and loaded as a separate module. The files under oracle/ are never modified.
"""
import os
import subprocess
import types

import pytest

import oracle
import test_oracle_pins as pins

ORACLE_DIR = os.path.dirname(os.path.abspath(oracle.__file__))
CPP = os.path.join(ORACLE_DIR, "ttt_oracle.cpp")
PY = os.path.join(ORACLE_DIR, "__init__.py")
COMBOS = pins.COMBOS

# --------------------------------------------------------------------------- pin batteries
FWD_PINS = (
    [("golden scalar chunks", pins.test_golden_scalar_worked_examples),
     ("golden vector-decay chunk", pins.test_golden_vector_decay_worked_example)]
    + [(f"dual form {l}/{a} C={C} decay={d}",
        lambda l=l, a=a, C=C, d=d: pins.test_oracle_matches_chunk_dual_form(l, a, C, d))
       for l, a in COMBOS for C in (1, 4) for d in (False, True)]
    + [("delta rule", lambda: pins.test_c1_is_the_delta_rule(True)),
       ("decayed Hebbian", pins.test_c1_inner_product_is_decayed_hebbian_attention),
       ("affine transition", pins.test_affine_state_transition)]
    + [(f"eta = 0 {l}/{a}", lambda l=l, a=a: pins.test_eta_zero_only_decays(l, a))
       for l, a in COMBOS]
    + [(f"vector dual form {l}/{a}", lambda l=l, a=a: pins.test_vector_decay_matches_its_dual_form(l, a, 4))
       for l, a in COMBOS]
    + [("vector zero factor", pins.test_vector_decay_zero_clears_exactly_one_row)]
)
BWD_PINS = (
    [("golden scalar backward", pins.test_golden_scalar_backward)]
    + [(f"finite differences {l}/{a}", lambda l=l, a=a: pins.test_backward_matches_finite_differences(l, a))
       for l, a in COMBOS]
    + [(f"vector finite differences {l}/{a}",
        lambda l=l, a=a: pins.test_vector_decay_backward_matches_finite_differences(l, a))
       for l, a in COMBOS]
)
INPLACE_PINS = [
    ("golden In-Place and NTP target", pins.test_golden_inplace_and_target_worked_examples),
    ("associative update", pins.test_inplace_final_state_is_associative),
    ("plain GEMM cases", pins.test_inplace_single_chunk_and_zero_lr_are_plain_gemm),
    ("In-Place dual form", pins.test_inplace_dual_form),
    ("document resets", pins.test_inplace_document_resets),
    ("In-Place finite differences", pins.test_inplace_backward_matches_finite_differences),
    ("In-Place single-chunk backward", pins.test_inplace_backward_single_chunk_closed_form),
    ("NTP target special cases", pins.test_inplace_target_special_cases),
    ("NTP target finite differences", pins.test_inplace_target_backward_matches_finite_differences),
]
MLP_PINS = (
    [("golden TTT-MLP", pins.test_golden_ttt_mlp_worked_example)]
    + [(f"TTT-MLP dual form {l}/{a} C={C}",
      lambda l=l, a=a, C=C: pins.test_ttt_mlp_matches_its_dual_form(l, a, C))
     for l, a in COMBOS for C in (2, 4)]
    + [("TTT-MLP without learning", pins.test_ttt_mlp_without_learning_only_decays)]
)


def _first_failing(battery):
    for name, pin in battery:
        try:
            pin()
        except (AssertionError, ValueError, FloatingPointError):
            return name
    return None


def _edit(text, old, new):
    assert old in text, f"mutation site not found: {old!r}"
    return text.replace(old, new)


# ---------------------------------------------------------------- C++ per-token evolver
# (description, text to replace, replacement): every occurrence is replaced
CPP_MUTANTS = [
    ("gradient at the running state instead of the chunk-start W0",
     "train_view<R, In>(sh, kt, v + t * dv, W0.data(), z.data(), g.data());",
     "train_view<R, In>(sh, kt, v + t * dv, W.data(), z.data(), g.data());"),
    ("chunk-start weight never refreshed",
     "    W0 = W;  // chunk-start weight",
     "    // W0 = W;  chunk-start weight"),
    ("decay applied to the write as well",
     "wrow[j] = gam * wrow[j] - eki * g[j];",
     "wrow[j] = gam * (wrow[j] - eki * g[j]);"),
    ("gradient ascent (wrong sign of the write)",
     "- eki * g[j];", "+ eki * g[j];"),
    ("learning rate without its factor 2",
     "const R eta = R(2) * sigmoid_(R(beta[t]) + R(sh.lr_bias));",
     "const R eta = sigmoid_(R(beta[t]) + R(sh.lr_bias));"),
    ("MSE write signal with the wrong sign",
     "vh - R(vt[j])", "R(vt[j]) - vh"),
    ("SiLU derivative missing its second term",
     "return s * (R(1) + z * (R(1) - s));", "return s;"),
    ("readout with the key instead of the query",
     "const R qi = R(qt[i]);", "const R qi = R(kt[i]);"),
    ("vector decay indexed by the first feature only",
     "return R(sh.gvec ? gamma[t * sh.dk + i] : gamma[t]);",
     "return R(sh.gvec ? gamma[t * sh.dk] : gamma[t]);"),
    ("backward drops the K^T dz route into the chunk-start adjoint",
     "wh0row[j] += ki * dz[j];", "(void)ki;"),
    ("backward forgets to decay the adjoint",
     "for (int j = 0; j < dv; ++j) Wh[(size_t)i * dv + j] *= gam;", "(void)gam;"),
    ("backward SiLU second derivative wrong",
     "return s * (R(1) - s) * (R(2) + z * (R(1) - R(2) * s));", "return s * (R(1) - s);"),
    ("backward dbeta without the sigmoid derivative",
     "dbeta[t] = deta * eta * (R(1) - eta / R(2));", "dbeta[t] = deta * eta;"),
    ("decay gradient against the state after the token",
     "const R* wp = Wprev.data() + (size_t)s * WS;", "const R* wp = Ws.data();"),
]


@pytest.mark.parametrize("what,old,new", CPP_MUTANTS, ids=[m[0] for m in CPP_MUTANTS])
def test_cpp_oracle_mutant_is_caught(what, old, new, tmp_path, monkeypatch):
    src = tmp_path / "ttt_oracle.cpp"
    src.write_text(_edit(open(CPP).read(), old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["g++", "-O1", "-std=c++17", "-fPIC", "-shared", str(src), "-o", str(lib)],
                   check=True)
    monkeypatch.setattr(oracle, "_lib", oracle.open_library(str(lib)))
    caught = _first_failing(FWD_PINS + BWD_PINS)
    assert caught is not None, f"no pin catches: {what}"


def test_cpp_oracle_batteries_pass_unmutated():
    # the batteries are meaningful only if the real oracle passes them
    assert _first_failing(FWD_PINS + BWD_PINS) is None


# ------------------------------------------------------- numpy / PyTorch oracle functions
PY_MUTANTS = [
    ("In-Place updates before it applies",
     "        o[i * C:(i + 1) * C] = zi @ w.T          # apply with the current fast weight\n"
     "        w += lr * (vh[i * C:(i + 1) * C].T @ zi)  # then update it with this chunk\n",
     "        w += lr * (vh[i * C:(i + 1) * C].T @ zi)\n"
     "        o[i * C:(i + 1) * C] = zi @ w.T\n", INPLACE_PINS),
    ("In-Place document start keeps the running weight",
     "            w = w0.copy()  # a new document starts from the initial fast weight\n",
     "            pass\n", INPLACE_PINS),
    ("In-Place backward drops the update's route into dZ",
     "            dz[sl] = do[sl] @ applied[i] + lr * (vh[sl] @ wh)\n",
     "            dz[sl] = do[sl] @ applied[i]\n", INPLACE_PINS),
    ("NTP target reads past tokens instead of future ones",
     "        y[: T - j] += w[j] * x[j:]\n", "        y[j:] += w[j] * x[: T - j]\n", INPLACE_PINS),
    ("NTP target backward shifts the wrong way",
     "        dx[j:] += w[j] * dy[: T - j]\n", "        dx[: T - j] += w[j] * dy[j:]\n",
     INPLACE_PINS),
    ("TTT-MLP hidden gradient at the running second layer",
     "                    g1 = (B0 @ g2) * d1\n", "                    g1 = (Bw @ g2) * d1\n",
     MLP_PINS),
    ("TTT-MLP second layer not decayed",
     "                    Bw = gam * Bw - eta * torch.outer(a, g2)\n",
     "                    Bw = Bw - eta * torch.outer(a, g2)\n", MLP_PINS),
    ("TTT-MLP readout before the token's write",
     "                    orows.append(_act_t(act, qt @ A) @ Bw)\n",
     "                    orows.append(_act_t(act, qt @ A0) @ B0)\n", MLP_PINS),
]


def _mutant_module(text):
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = PY  # its C++ part still loads the real build
    exec(compile(text, PY, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("what,old,new,battery", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_python_oracle_mutant_is_caught(what, old, new, battery, monkeypatch):
    monkeypatch.setattr(pins, "oracle", _mutant_module(_edit(open(PY).read(), old, new)))
    assert _first_failing(battery) is not None, f"no pin catches: {what}"


def test_python_oracle_batteries_pass_unmutated(monkeypatch):
    monkeypatch.setattr(pins, "oracle", _mutant_module(open(PY).read()))
    assert _first_failing(INPLACE_PINS + MLP_PINS) is None
