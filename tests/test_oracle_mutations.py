"""The oracle's pins must catch plausible mistakes.

Each case compiles a copy of the oracle's C source with one deliberate mistake planted
(a dropped term, a wrong sign, a transposed operand, a wrong state) into a temporary
directory, on the CPU, and checks that at least one pin of ``test_oracle_pins`` fails on
it.  The committed oracle is never modified.
"""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "kla_oracle.c")


def _forward_pins(mod):
    yield lambda: pins.test_golden_hand_example(mod)
    yield lambda: pins.test_hard_projection_every_step(mod)
    for eps in (0.0, 1e-6, 0.5):
        yield lambda eps=eps: pins.test_relaxed_interpolation(mod, eps)
    yield lambda: pins.test_line_search(mod)
    for eta, eps in ((0.4, 0.0), (0.9, 1e-3), (0.25, 2.0)):
        yield lambda eta=eta, eps=eps: pins.test_proximal_form(mod, eta, eps)
    yield lambda: pins.test_classical_kaczmarz_min_norm(mod)
    yield lambda: pins.test_table6_product_form(mod, True)
    yield lambda: pins.test_eta_zero_pure_decay(mod)
    yield lambda: pins.test_exact_rational_bruteforce(mod)


def _backward_pins(mod):
    for T, ck, eps in ((7, 3, 1e-2), (12, 64, 0.3), (5, 1, 1e-6)):
        yield lambda T=T, ck=ck, eps=eps: pins.test_backward_finite_differences(mod, T, ck, eps)


def _direct_pins(mod):
    yield lambda: pins.test_direct_mode_with_kaczmarz_eta_equals_kaczmarz_mode(mod)
    yield lambda: pins.test_direct_mode_inverse_norm_beta_projects(mod)


def _direct_backward_pins(mod):
    for T, ck in ((7, 3), (5, 64)):
        yield lambda T=T, ck=ck: pins.test_direct_backward_finite_differences(mod, T, ck)


def _diag_forward_pins(mod):
    for eps in (1e-6, 0.5):
        yield lambda eps=eps: pins.test_diag_relaxed_interpolation(mod, eps)
    for C in (3, 8):
        yield lambda C=C: pins.test_diag_chunk_form_matches_token_form(mod, C)


def _diag_backward_pins(mod):
    for beta, eps in (("kaczmarz", 1e-2), ("direct", 0.0)):
        yield lambda beta=beta, eps=eps: pins.test_diag_backward_finite_differences(mod, beta, eps)
    yield lambda: pins.test_diag_uniform_channels_equal_scalar_gating(mod, "kaczmarz")


def _diag_chunk_pins(mod):
    yield lambda: pins.test_diag_uniform_channels_equal_scalar_gating(mod, "kaczmarz")
    for C in (3, 8):
        yield lambda C=C: pins.test_diag_chunk_form_matches_token_form(mod, C)


def _chunk_pins(mod):
    for C in (2, 3, 8, 64):
        yield lambda C=C: pins.test_chunk_form_matches_token_form(mod, C)


MUTATIONS = [
    # (name, original text, mutated text, which pins must catch it)
    ("residual_ignores_decay", "e[j] = v[j] - s;", "e[j] = v[j] - s / alpha;", _forward_pins),
    ("eps_dropped", "double den = knorm2 + eps;", "double den = knorm2;", _forward_pins),
    ("write_sign_flipped", "for (int j = 0; j < Dv; ++j) S[(size_t)i * Dv + j] += beta * k[i] * e[j];",
     "for (int j = 0; j < Dv; ++j) S[(size_t)i * Dv + j] -= beta * k[i] * e[j];", _forward_pins),
    ("readout_transposed", "for (int i = 0; i < Dk; ++i) s += S[(size_t)i * Dv + j] * q[i];",
     "for (int i = 0; i < Dk; ++i) s += S[(size_t)j * Dk + i] * q[i];", _forward_pins),
    ("beta_uses_norm_not_square", "double beta = kaczmarz_beta(eta, n, eps, direct);",
     "double beta = kaczmarz_beta(eta, sqrt(n), eps, direct);", _forward_pins),
    ("direct_mode_normalises_anyway", "    if (direct) return eta;",
     "    if (direct) return eta / (knorm2 + 1.0);", _direct_pins),
    ("bwd_direct_deta_halved", "                        detat = dbeta;\n",
     "                        detat = 0.5 * dbeta;\n", _direct_backward_pins),
    ("bwd_direct_keeps_norm_term", "                        detat = dbeta;\n",
     "                        detat = dbeta;\n                        dn = -dbeta * beta / den;\n",
     _direct_backward_pins),
    ("bwd_dk_drops_norm_term", "dkt[i] = beta * s - Sbde[i] + 2.0 * kt[i] * dn;",
     "dkt[i] = beta * s - Sbde[i];", _backward_pins),
    ("bwd_dg_drops_alpha", "dgt *= alpha;", "dgt *= 1.0;", _backward_pins),
    ("bwd_dq_uses_previous_state", "for (int j = 0; j < Dv; ++j) s += Scur[(size_t)i * Dv + j] * dot[j];",
     "for (int j = 0; j < Dv; ++j) s += Sprev[(size_t)i * Dv + j] * dot[j];", _backward_pins),
    ("bwd_de_drops_beta", "de[j] = beta * s;", "de[j] = s;", _backward_pins),
    ("diag_one_channel_decay_for_all", "        const double ar = exp(gvec[r]);",
     "        const double ar = exp(gvec[0]);", _diag_forward_pins),
    ("diag_bwd_dg_drops_alpha", "dg[IDX_TOK(b, t, h, r, T, H, Dk)] = ar * acc;",
     "dg[IDX_TOK(b, t, h, r, T, H, Dk)] = acc;", _diag_backward_pins),
    ("diag_bwd_state_gradient_not_decayed", "                        Lam[x] = ar * dsd;",
     "                        Lam[x] = dsd;", _diag_backward_pins),
    ("diag_chunk_ratio_inverted",
     "aij += ki[r] * kj[r] * exp(Gc[(size_t)i * Dk + r] - Gc[(size_t)j * Dk + r]);",
     "aij += ki[r] * kj[r] * exp(Gc[(size_t)j * Dk + r] - Gc[(size_t)i * Dk + r]);", _diag_chunk_pins),
    ("chunk_decay_ratio_inverted", "val = bet[i] * (gam[i] / gam[j]) * kk;",
     "val = bet[i] * (gam[j] / gam[i]) * kk;", _chunk_pins),
    ("chunk_substitution_sign", "U[(size_t)i * Dv + c2] -= l * U[(size_t)j * Dv + c2];",
     "U[(size_t)i * Dv + c2] += l * U[(size_t)j * Dv + c2];", _chunk_pins),
    ("chunk_state_drops_decay", "double s = gC * S[(size_t)x * Dv + c2];",
     "double s = S[(size_t)x * Dv + c2];", _chunk_pins),
]


@pytest.mark.parametrize("name,old,new,detectors", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(tmp_path, name, old, new, detectors):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "kla_oracle_mut.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libkla_oracle_mut.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    str(mutated), "-o", str(lib), "-lm"], check=True)
    mod = oracle.OracleLib(str(lib))
    caught = 0
    for check in detectors(mod):
        try:
            check()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught the planted mistake {name}"
