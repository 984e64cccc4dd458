"""Planted mistakes in the oracle must fail its pins.

Each test swaps one oracle function for a copy with a plausible mistake (a dropped
term, a wrong sign, an off-by-one index, a wrong tie rule), on the CPU, and runs
the pin that guards it: the pin has to fail.  This is what makes the pins evidence
that the oracle is right rather than a restatement of it.
"""

import numpy as np
import pytest
import torch

import test_oracle_diagnostics as diag_pins
import test_oracle_pins as pins
import test_oracle_precision as prec_pins
from oracle import compress, diagnostics, factored, precision, recurrences
from workloads import FORM_GDN


def _fails(check, *args):
    with pytest.raises(AssertionError):
        check(*args)


def test_dropped_erase_term_in_the_new_value_column(monkeypatch):
    real = factored.step

    def planted(form, a, U, V, vbar, q, k, v, alpha, beta):
        a2, U2, V2, o = real(form, a, U, V, vbar, q, k, v, alpha, beta)
        omega, eps = factored.split_value(v, vbar)
        V2 = V2.copy()
        V2[:, :, -1] = np.asarray(beta)[:, None] * eps          # beta eps, no - g V U^T k
        return a2, U2, V2, o
    monkeypatch.setattr(factored, "step", planted)
    _fails(pins.test_lemma2_factored_step_is_exact, FORM_GDN)


def test_wrong_sign_in_the_sink_update(monkeypatch):
    real = factored.step

    def planted(form, a, U, V, vbar, q, k, v, alpha, beta):
        a2, U2, V2, o = real(form, a, U, V, vbar, q, k, v, alpha, beta)
        g = np.asarray(alpha)[:, None]
        ka = np.einsum("ni,ni->n", k, a)[:, None]
        a2 = a2 + 2 * np.asarray(beta)[:, None] * g * ka * k     # + g k^T a instead of -
        return a2, U2, V2, o
    monkeypatch.setattr(factored, "step", planted)
    _fails(pins.test_lemma2_factored_step_is_exact, FORM_GDN)
    _fails(pins.test_lemma1_sink_follows_its_own_recurrence, FORM_GDN)


def test_decay_applied_after_the_write_in_the_dense_step(monkeypatch):
    def planted(S, k, v, g, beta):
        b = np.asarray(beta, dtype=np.float64)[:, None, None]
        kS = np.einsum("ni,nij->nj", k, S)
        S2 = S - b * np.einsum("ni,nj->nij", k, kS) + b * np.einsum("ni,nj->nij", k, v)
        return np.asarray(g, dtype=np.float64)[:, None, None] * S2   # g also scales the write
    monkeypatch.setattr(recurrences, "gdn_step", planted)
    _fails(pins.test_gdn_step_closed_form_on_key_and_complement)


def test_off_by_one_singular_triplets_in_the_truncation(monkeypatch):
    def planted(U, V, R):
        A = np.einsum("nir,njr->nij", U, V)
        X, s, Yt = np.linalg.svd(A, full_matrices=False)
        sq = np.sqrt(s[:, 1:R + 1])                              # skips the largest triplet
        Up = X[:, :, 1:R + 1] * sq[:, None, :]
        Vp = np.swapaxes(Yt[:, 1:R + 1, :], 1, 2) * sq[:, None, :]
        return Up, Vp, s
    monkeypatch.setattr(compress, "truncate_product", planted)
    _fails(pins.test_truncation_of_a_known_spectrum)


def test_ties_away_from_zero_in_the_16bit_rounding(monkeypatch):
    def planted(x, fmt):
        x = np.asarray(x, dtype=np.float64)
        step = precision.ulp(x, fmt)
        r = np.floor(np.abs(x) / step + 0.5) * step               # ties away from zero
        r = np.where(r > precision.max_finite(fmt), np.inf, r)
        return np.copysign(r, x)
    monkeypatch.setattr(precision, "round_nearest", planted)
    _fails(prec_pins.test_rounding_equals_torch_conversion, "bf16", torch.bfloat16, -140, 128)
    _fails(prec_pins.test_closed_forms)


def test_wrong_sign_of_the_cross_energy(monkeypatch):
    real = diagnostics.energies

    def planted(a, U, V, vbar):
        e = real(a, U, V, vbar)
        e[:, 2] = -e[:, 2]
        return e
    monkeypatch.setattr(diagnostics, "energies", planted)
    _fails(diag_pins.test_parts_add_up_to_the_energy_of_the_reconstructed_state)


def test_core_without_the_transpose_in_the_qr_route(monkeypatch):
    def planted(U, V, R):
        Qu, Ru = np.linalg.qr(U)
        Qv, Rv = np.linalg.qr(V)
        M = Ru @ Rv                                              # R_u R_v instead of R_u R_v^T
        X, s, Yt = np.linalg.svd(M, full_matrices=False)
        sq = np.sqrt(s[:, :R])
        return Qu @ X[:, :, :R] * sq[:, None, :], Qv @ np.swapaxes(Yt[:, :R, :], 1, 2) * sq[:, None, :], s
    monkeypatch.setattr(compress, "truncate_qr_core", planted)
    _fails(pins.test_qr_core_route_equals_product_svd)


def test_sink_projection_without_the_norm(monkeypatch):
    def planted(S, vbar):
        return np.einsum("nij,nj->ni", S, vbar)                  # S vbar, not S vbar / |vbar|^2
    monkeypatch.setattr(factored, "sink_coefficient", planted)
    import oracle.convert as oconv
    monkeypatch.setattr(oconv, "sink_coefficient", planted)
    _fails(pins.test_conversion_recovers_a_known_sink_and_content)


def test_mamba2_with_the_erase_left_on(monkeypatch):
    real = factored.step

    def planted(form, a, U, V, vbar, q, k, v, alpha, beta):
        if form == pins.FORM_MAMBA2:                             # GDN's update with Delta as beta
            return real(pins.FORM_GDN, a, U, V, vbar, q, k, v, alpha, beta)
        return real(form, a, U, V, vbar, q, k, v, alpha, beta)
    monkeypatch.setattr(factored, "step", planted)
    _fails(pins.test_mamba2_is_the_general_update_with_erase_off)


def test_kda_decay_applied_after_the_erase(monkeypatch):
    def planted(S, k, v, alpha, beta):
        b = np.asarray(beta, dtype=np.float64)[:, None, None]
        kS = np.einsum("ni,nij->nj", k, S)
        E = S - b * np.einsum("ni,nj->nij", k, kS)
        return alpha[:, :, None] * E + b * np.einsum("ni,nj->nij", k, v)   # Diag(alpha) (I - b k k^T) S
    monkeypatch.setattr(recurrences, "kda_step", planted)
    _fails(pins.test_kda_closed_form_and_gdn_special_case)

