"""The oracle's pins catch plausible mistakes: each case below plants one
mistake in a copy of the C oracle (a dropped term, a wrong sign, index or
operand, a swapped role), builds the copy, points the oracle's front end at it
and runs the pins of ``test_oracle_pins.py``; at least one pin must fail.  The
two rules written in the Python front end (the slot count a skip rate asks for
and the quantile mapping to tau) get the same treatment on a rewritten copy of
the function.

The planted mistakes stay in index range, so a mutant can give wrong numbers
but never read or write outside its arrays.  Everything runs on the CPU.
"""
import importlib.util
import inspect
import os
import subprocess

import pytest

import oracle
import oracle.build as oracle_build
import oracle.oracle as oracle_front

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "ace_oracle.c")


def _pins():
    spec = importlib.util.spec_from_file_location("_oracle_pins", os.path.join(HERE, "test_oracle_pins.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    calls = {}
    for name, fn in inspect.getmembers(mod, inspect.isfunction):
        if not name.startswith("test_") or fn.__module__ != mod.__name__:
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if marks:
            argname, values = marks[0].args[0], marks[0].args[1]
            for v in values:
                calls[f"{name}[{v}]"] = (lambda f=fn, a=argname, v=v: f(**{a: v}))
        else:
            calls[name] = fn
    return calls


# (name, text in the oracle, replacement, the pins expected to catch it first)
MUTANTS = [
    ("rmsnorm: sum instead of mean", "sqrt(ss / d + eps_rms)", "sqrt(ss + eps_rms)",
     ["test_rmsnorm_closed_form_and_scale_invariance"]),
    ("rmsnorm: gamma dropped", "x[(long)t * d + i] = xb * gamma[i];", "x[(long)t * d + i] = xb;",
     ["test_rmsnorm_closed_form_and_scale_invariance"]),
    ("rmsnorm: eps dropped", "sqrt(ss / d + eps_rms)", "sqrt(ss / d)",
     ["test_rmsnorm_closed_form_and_scale_invariance"]),
    ("silu: wrong sign in the exponent", "a / (1.0 + exp(-a))", "a / (1.0 + exp(a))",
     ["test_swiglu_closed_form_ln3"]),
    ("swiglu: SiLU on the up projection", "h[j] = silu(a) * b;", "h[j] = a * silu(b);",
     ["test_swiglu_closed_form_ln3"]),
    ("swiglu: W^down read transposed",
     "for (int j = 0; j < m; ++j) s += h[j] * (double)wd[(long)i * m + j];",
     "for (int j = 0; j < m; ++j) s += h[j] * (double)wd[(long)j * d + i];",
     ["test_swiglu_upper_bound_spectral", "test_swiglu_linear_regime_matches_relu_bilinear"]),
    ("router: bias subtracted", "if (c->bias) s += (double)c->bias[e];",
     "if (c->bias) s -= (double)c->bias[e];",
     ["test_router_topk_matches_library_sort_and_softmax"]),
    ("router: ties go to the higher index", "if (best < 0 || l[e] > l[best]) best = e;",
     "if (best < 0 || l[e] >= l[best]) best = e;", ["test_router_tie_break_lower_index_first"]),
    ("router: gates not renormalised", "c->gate[t * k + r] = c->renorm ? p / ztop : p;",
     "c->gate[t * k + r] = p;", ["test_router_topk_matches_library_sort_and_softmax"]),
    ("router: softmax over the top-k only",
     "for (int e = 0; e < E; ++e) Z += exp(l[e] - lmax);",
     "for (int e = 0; e < k; ++e) Z += exp(l[sel[e]] - lmax);",
     ["test_router_topk_matches_library_sort_and_softmax"]),
    ("gsp: gamma dropped from the down product", "      p *= gamma[i];\n", "\n",
     ["test_gsp_frobenius_products_match_library_and_gram_identity"]),
    ("gsp: gamma dropped from a factor norm", "double v = gamma[i] * (double)w[(long)j * d + i];",
     "double v = (double)w[(long)j * d + i];", ["test_gsp_closed_form_scaled_identities"]),
    ("gsp: eps dropped from the normalisation",
     "a_tilde[e] = sqrt(a_up[e] * a_gate[e]);\n    mean += a_tilde[e];\n  }\n  mean /= E;\n"
     "  for (int e = 0; e < E; ++e) A[e] = a_tilde[e] / (mean + eps);",
     "a_tilde[e] = sqrt(a_up[e] * a_gate[e]);\n    mean += a_tilde[e];\n  }\n  mean /= E;\n"
     "  for (int e = 0; e < E; ++e) A[e] = a_tilde[e] / mean;",
     ["test_gsp_frobenius_products_match_library_and_gram_identity"]),
    ("gsp: a^up paired with the wrong product",
     "a_up[e] = norms[e * 4 + 0] * norms[e * 4 + 1];",
     "a_up[e] = norms[e * 4 + 0] * norms[e * 4 + 3];",
     ["test_gsp_closed_form_scaled_identities", "test_gsp_exact_scaling_laws[wg]"]),
    ("gsp: arithmetic instead of geometric mean",
     "a_tilde[e] = sqrt(a_up[e] * a_gate[e]);", "a_tilde[e] = 0.5 * (a_up[e] + a_gate[e]);",
     ["test_gsp_closed_form_unequal_views"]),
    ("gsp: no layer normalisation",
     "a_tilde[e] = sqrt(a_up[e] * a_gate[e]);\n    mean += a_tilde[e];\n  }\n  mean /= E;\n"
     "  for (int e = 0; e < E; ++e) A[e] = a_tilde[e] / (mean + eps);",
     "a_tilde[e] = sqrt(a_up[e] * a_gate[e]);\n    mean += a_tilde[e];\n  }\n  mean /= E;\n"
     "  for (int e = 0; e < E; ++e) A[e] = a_tilde[e];",
     ["test_gsp_closed_form_scaled_identities"]),
    ("gsp spectral: square of sigma returned", "return sqrt(n); }", "return n; }",
     ["test_power_iteration_matches_svd_with_gap"]),
    ("rcr: router rows not centred", "double wt = (double)wr[(long)e * d + i] - mean_w[i];",
     "double wt = (double)wr[(long)e * d + i];", ["test_rcr_translation_invariance_and_scaling"]),
    ("rcr: centred on the sum of the rows", "  for (int i = 0; i < d; ++i) mean_w[i] /= E;\n", "\n",
     ["test_rcr_translation_invariance_and_scaling"]),
    ("rcr: norm instead of RMS", "double rms = sqrt(ss / d);", "double rms = sqrt(ss);",
     ["test_rcr_prototype_rms_is_rho"]),
    ("rcr: rho dropped", "/ (rms + eps) * rho;", "/ (rms + eps);",
     ["test_rcr_prototype_rms_is_rho"]),
    ("rcr: gamma not applied to the prototype", "z[i] = q[i] * c->gamma[i];", "z[i] = q[i];",
     ["test_rcr_closed_form_ln3"]),
    ("rcr: output norm not divided by the prototype norm",
     "a_tilde[e] = fnorm[e] / (norm2(d, q + (long)e * d) + eps);", "a_tilde[e] = fnorm[e];",
     ["test_rcr_closed_form_ln3"]),
    ("mask: min instead of max",
     "default: c[s] = s_gsp[s] > s_rcr[s] ? s_gsp[s] : s_rcr[s]; break;",
     "default: c[s] = s_gsp[s] < s_rcr[s] ? s_gsp[s] : s_rcr[s]; break;", ["test_mask_rules"]),
    ("mask: top-1 not protected", "keep[s] = (unsigned char)(rank == 0 || !skip);",
     "keep[s] = (unsigned char)(!skip);", ["test_mask_rules"]),
    ("mask: a score equal to tau skipped", "int skip = (c[s] < tau);", "int skip = (c[s] <= tau);",
     ["test_tau_quantile_skips_exactly_n"]),
    ("mask: mean rule without the half", "case 2: c[s] = 0.5 * (s_gsp[s] + s_rcr[s]); break;",
     "case 2: c[s] = (s_gsp[s] + s_rcr[s]); break;", ["test_fusion_ablation_rules"]),
    ("compaction: skipped slots listed", "if (keep[s] && idx[s] == e) {", "if (idx[s] == e) {",
     ["test_compaction_order_and_bijection"]),
    ("compaction: ranks reversed", "slot_rank[S] = r;", "slot_rank[S] = k - 1 - r;",
     ["test_compaction_order_and_bijection"]),
    ("combine: gate dropped", "for (int i = 0; i < d; ++i) y[i] += c->gate[s] * o[i];",
     "for (int i = 0; i < d; ++i) y[i] += o[i];",
     ["test_zero_skip_is_dense_topk_and_k_equals_E_is_softmax_mixture"]),
    ("combine: skipped slots kept", "    if (!c->keep[s]) continue;\n", "\n",
     ["test_skipped_slots_drop_out_without_renormalisation"]),
]


@pytest.fixture(scope="module")
def pins():
    return _pins()


def _build_mutant(tmpdir, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"anchor not unique in the oracle: {old!r}"
    path = os.path.join(tmpdir, "ace_oracle_mutant.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(tmpdir, "libace_oracle_mutant.so")
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-o", lib,
                    path, "-lm", "-lpthread"], check=True)
    return lib


@pytest.mark.parametrize("name,old,new,first", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_a_planted_mistake_fails_a_pin(name, old, new, first, pins, tmp_path, monkeypatch):
    lib = _build_mutant(str(tmp_path), old, new)
    monkeypatch.setattr(oracle_build, "build", lambda force=False: lib)
    monkeypatch.setattr(oracle_front, "_lib", None)
    order = first + [p for p in sorted(pins) if p not in first]
    caught = None
    for p in order:
        try:
            pins[p]()
        except Exception as e:  # an assertion, or numpy refusing the wrong numbers
            caught = (p, type(e).__name__)
            break
    assert caught is not None, f"no pin fails with the planted mistake: {name}"


# (name, front-end function, text in it, replacement)
PY_MUTANTS = [
    ("tau: one candidate too low", "tau_quantile", "return float(cand[n_skip])",
     "return float(cand[n_skip - 1])"),
    ("tau: top-1 slots among the candidates", "tau_quantile", "cand = np.sort(c[:, 1:].reshape(-1))",
     "cand = np.sort(c.reshape(-1))"),
    ("slot count: rounded down", "n_skip_for", "int(math.floor(rate * total + 0.5))",
     "int(math.floor(rate * total))"),
    ("slot count: the two bases swapped", "n_skip_for",
     'total = T * k if of == "slots" else T * (k - 1)', 'total = T * (k - 1) if of == "slots" else T * k'),
]


@pytest.mark.parametrize("name,fn,old,new", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_a_planted_mistake_in_the_front_end_fails_a_pin(name, fn, old, new, pins, monkeypatch):
    src = inspect.getsource(getattr(oracle_front, fn))
    assert src.count(old) == 1, f"anchor not unique in {fn}: {old!r}"
    scope = dict(vars(oracle_front))
    exec(compile(src.replace(old, new), f"<mutant {fn}>", "exec"), scope)
    monkeypatch.setattr(oracle_front, fn, scope[fn])
    monkeypatch.setattr(oracle, fn, scope[fn])
    caught = None
    for p in sorted(pins):
        try:
            pins[p]()
        except Exception as e:
            caught = (p, type(e).__name__)
            break
    assert caught is not None, f"no pin fails with the planted mistake: {name}"
