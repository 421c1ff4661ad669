"""Plant one plausible mistake at a time in a copy of the oracle (on the CPU)
and check that the pin suite rejects every broken copy."""
import os

import pytest

import oracle
import oracle_pins as pins

MUTANTS = {
    "dropped process noise": ("a * a * P_prev + p;", "a * a * P_prev;"),
    "a instead of a^2 in predict": ("a * a * P_prev + p;", "a * P_prev + p;"),
    "mean not propagated by a": ("const double m_pred = a * m_prev;",
                                 "const double m_pred = m_prev;"),
    "evidence precision subtracted": ("*lam_out = 1.0 / P_pred + phi;",
                                      "*lam_out = 1.0 / P_pred - phi;"),
    "prior information inverted": ("*eta_out = m_pred / P_pred + b;",
                                   "*eta_out = m_pred * P_pred + b;"),
    "token information subtracted": ("*eta_out = m_pred / P_pred + b;",
                                     "*eta_out = m_pred / P_pred - b;"),
    "mu = eta * lambda": ("mu[i] = eta_t / lam_t;", "mu[i] = eta_t * lam_t;"),
    "var = lambda": ("var[i] = 1.0 / lam_t;", "var[i] = lam_t;"),
    "prior variance = lambda_0": ("double P = 1.0 / lam0;", "double P = lam0;"),
    "prior mean = eta_0": ("double m = eta0 / lam0;", "double m = eta0;"),
    "carried mean = eta": ("        m = eta_t / lam_t;", "        m = eta_t;"),
    "carried variance = prior variance": ("        P = 1.0 / lam_t;",
                                          "        P = 1.0 / (lam_t - phi[i]);"),
    "p and phi transposed": ("kf_token(a[i], p[i], phi[i], b[i],",
                             "kf_token(a[i], phi[i], p[i], b[i],"),
    "wrong batch stride": ("const int64_t base = bi * T * HN + hn;",
                           "const int64_t base = bi * HN + hn;"),
    "prior of channel 0 for all": ("lam0[ch], eta0[ch],", "lam0[0], eta0[0],"),
    "decode step: state read as variance": ("const double P = 1.0 / lam_state[ch];",
                                            "const double P = lam_state[ch];"),
    "decode step: eta not written": ("        eta_state[ch] = eta_t;", "        (void)eta_t;"),
    # the reverse-mode gradients
    "backward: later variance gradient dropped": ("+ gP_next;", ";"),
    "backward: later mean gradient dropped": ("+ gm_next;", ";"),
    "backward: var term sign": ("- g_v / (lam * lam) - g_m", "+ g_v / (lam * lam) - g_m"),
    "backward: mu -> eta uses lambda": ("+ g_m / lam;", "+ g_m * lam;"),
    "backward: mean path dropped from P-": ("- g_e * m_pred / (P_pred * P_pred);", ";"),
    "backward: d(a^2)/da = a": ("g_Pp * 2.0 * at * P_prev", "g_Pp * at * P_prev"),
    "backward: mean term of a dropped": ("+ g_mp * m_prev;", ";"),
    "backward: variance carried by a": ("gP_next = g_Pp * at * at;", "gP_next = g_Pp * at;"),
    "backward: mean carried without a": ("gm_next = g_mp * at;", "gm_next = g_mp;"),
    "backward: prior mean term dropped": ("- gm_next * eta0 / (lam0 * lam0);", ";"),
    "backward: prior information gradient": ("*g_eta0 = gm_next / lam0;", "*g_eta0 = gm_next;"),
    "backward: phi and b gradients swapped": ("gphi[i] = g_l;\n        gb[i] = g_e;",
                                               "gphi[i] = g_e;\n        gb[i] = g_l;"),
    "backward: wrong batch stride": ("(bi * T) * HN + hn;", "bi * HN + hn;"),
    "backward: prior variance = lambda_0": ("double P = 1.0 / lam0, m", "double P = lam0, m"),
    "backward: recomputed state carries the variance only": ("m = m_out;", "m = m_out * 0.0 + m;"),
    "backward: recomputed mean not divided": ("m_out = eta_t / lam_t;", "m_out = eta_t;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    with open(oracle.SOURCE) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation site for {name!r} not found exactly once"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = oracle.build(str(path), str(tmp_path / "libmutant.so"), force=True)
    orc = oracle.Oracle.load(os.path.abspath(lib))
    failures = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError, FloatingPointError, ZeroDivisionError) as e:
            failures.append((pin.__name__, str(e)[:80]))
    assert failures, f"no pin caught mutant {name!r}"


# Mistakes planted in the layer function of the oracle package (Python source).
LAYER_MUTANTS = {
    "layer: phi = k w": ("phi = kk * kk * ww", "phi = kk * ww"),
    "layer: information without the value precision": ("info = kk * ww * vv", "info = kk * vv"),
    "layer: variance readout with q, not q^2": ("np.sum(qq * qq * var, axis=4)", "np.sum(qq * var, axis=4)"),
    "layer: readout of eta": ('mu = out["mu"].reshape(shape5)', 'mu = out["eta"].reshape(shape5)'),
    "layer: final state from the first token": ('lam_T = out["lam"][:, T - 1]', 'lam_T = out["lam"][:, 0]'),
    "layer: k read out instead of q": ("qq = q[:, :, :, None, :]", "qq = k[:, :, :, None, :]"),
    "layer: a and p swapped": ("self.forward(flat(aa), flat(pp),", "self.forward(flat(pp), flat(aa),"),
    "layer backward: dk without the factor 2": ("g_phi * 2.0 * kk * ww", "g_phi * kk * ww"),
    "layer backward: dw with k, not k^2": ("g_phi * kk * kk + g_b * kk * vv", "g_phi * kk + g_b * kk * vv"),
    "layer backward: dq without the variance term": (
        "np.sum(g_y[..., None] * mu + 2.0 * g_s[..., None] * qq * var, axis=3)",
        "np.sum(g_y[..., None] * mu, axis=3)"),
    "layer backward: da from the first batch row": ('"a": np.sum(gr["a"].reshape(shape5), axis=(0, 1)),',
                                                    '"a": np.sum(gr["a"].reshape(shape5), axis=1)[0],'),
    "layer backward: final precision gradient dropped": ("g_lam[:, T - 1] = _f64(g_lam_T)", "pass"),
    "layer backward: variance readout gradient with q": ("g_var = g_s[..., None] * qq * qq",
                                                          "g_var = g_s[..., None] * qq"),
}


# Mistakes planted in the attention weights and the convolutional form.
ATTENTION_MUTANTS = {
    "attention: gate with the precision after the token": (
        "lam_before = np.concatenate([lam0[:, None], out[\"lam\"][:, :T - 1]], axis=1)",
        "lam_before = out[\"lam\"]"),
    "attention: gate with a^2 on top": ("gate = a / (a * a + p * lam_before)",
                                        "gate = a * a / (a * a + p * lam_before)"),
    "attention: product includes the source token": (
        "np.cumprod(gate[:, start + j + 1:start + n_valid], axis=1)",
        "np.cumprod(gate[:, start + j:start + n_valid - 1], axis=1)"),
    "attention: process noise dropped from the gate": ("gate = a / (a * a + p * lam_before)",
                                                       "gate = a / (a * a + lam_before)"),
    "attention: windows not offset by t0": ("start = t0 + w * W", "start = w * W"),
}

LTI_MUTANTS = {
    "lti: precision kernel a^-1": ("kappa = np.power(a[..., None], -2.0 * m)",
                                   "kappa = np.power(a[..., None], -m)"),
    "lti: prior decayed one step short": ("lam[:, t] = kappa[..., t + 1] * lam0", "lam[:, t] = kappa[..., t] * lam0"),
    "lti: kernel not reversed": ('np.einsum("bhns,bshn->bhn", kappa[..., t::-1], phi[:, :t + 1])',
                                 'np.einsum("bhns,bshn->bhn", kappa[..., :t + 1], phi[:, :t + 1])'),
    "lti: mean kernel squared": ("nu = np.power(a[..., None], -m)", "nu = np.power(a[..., None], -2.0 * m)"),
    "lti: mu = eta lambda": ('return {"lam": lam, "eta": eta, "mu": eta / lam,',
                             'return {"lam": lam, "eta": eta, "mu": eta * lam,'),
}


def _python_mutant_caught(old, new, name, pin_list):
    import importlib.util
    path = os.path.join(os.path.dirname(oracle.SOURCE), "__init__.py")
    src = open(path).read()
    assert src.count(old) == 1, f"mutation site for {name!r} not found exactly once"
    spec = importlib.util.spec_from_loader("oracle_py_mutant", loader=None, origin=path)
    mod = importlib.util.module_from_spec(spec)
    mod.__file__ = path
    exec(compile(src.replace(old, new), path, "exec"), mod.__dict__)
    orc = mod.Oracle.load(oracle.build())
    failures = []
    for pin in pin_list:
        try:
            pin(orc)
        except (AssertionError, ValueError, FloatingPointError, ZeroDivisionError) as e:
            failures.append((pin.__name__, str(e)[:80]))
    assert failures, f"no pin caught mutant {name!r}"


@pytest.mark.parametrize("name", sorted(ATTENTION_MUTANTS))
def test_attention_mutant_is_caught(name):
    _python_mutant_caught(*ATTENTION_MUTANTS[name], name, pins.ATTENTION_PINS)


@pytest.mark.parametrize("name", sorted(LTI_MUTANTS))
def test_lti_mutant_is_caught(name):
    _python_mutant_caught(*LTI_MUTANTS[name], name, pins.LTI_PINS)


@pytest.mark.parametrize("name", sorted(LAYER_MUTANTS))
def test_layer_mutant_is_caught(name):
    import importlib.util
    old, new = LAYER_MUTANTS[name]
    path = os.path.join(os.path.dirname(oracle.SOURCE), "__init__.py")
    src = open(path).read()
    assert src.count(old) == 1, f"mutation site for {name!r} not found exactly once"
    spec = importlib.util.spec_from_loader("oracle_layer_mutant", loader=None, origin=path)
    mod = importlib.util.module_from_spec(spec)
    mod.__file__ = path
    exec(compile(src.replace(old, new), path, "exec"), mod.__dict__)
    orc = mod.Oracle.load(oracle.build())
    failures = []
    for pin in pins.LAYER_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError, FloatingPointError, ZeroDivisionError) as e:
            failures.append((pin.__name__, str(e)[:80]))
    assert failures, f"no pin caught mutant {name!r}"
