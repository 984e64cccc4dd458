"""Whole oracle trajectories for a sample of units (test infrastructure).

Per unit (request b, layer l, head h), following SEED figures & tables
(thelatestinai.com), Figure 1 and Table 1:
  1. dense prefill of n_prefill tokens from S_0 = 0 (``recurrences``),
  2. conversion to sink + rank R (``convert``), leaving c = R columns,
  3. n_decode exact factored steps with read-out (``factored.step``); each step
     appends one column pair,
  4. after the step that brings the column count to R + W, the factors are
     compressed back to rank R (``compress.truncate_qr_core``): with decode steps
     counted from 1 this is after steps W, 2W, 3W, ... (every W steps); a
     request that joined j steps earlier (ragged schedules) is j steps ahead.
An open-loop dense shadow S_t^exact runs the dense recurrence on the same inputs
from the uncompressed prefill state, for Lemma 1 and Corollary 4 checks.
"""

from __future__ import annotations

import numpy as np

from workloads import philox

from . import compress, convert, factored, recurrences


def run_units(cfg, b, l, h, n_prefill=None, n_decode=None, keep_shadow=True, lead_in=0):
    """Run the sampled units (1-D arrays b, l, h) and return a dict of trajectories.

    With lead_in = j > 0 the units first take j lead-in decode steps (inputs of
    philox.PHASE_LEADIN, t = 0 .. j-1, outputs not kept), as a request that joined
    the batch j steps before the others; the trajectories below start after them.

    Keys: o (T, n, d_v); a_t (T, n, d_k); ncols (T,) after each step;
    comp_steps (list of 1-based steps after which a compression ran);
    sigma (n_comp, n, R) kept singular values; gap (n_comp, n) relative gap at R;
    tail (n_comp + 1, n) discarded tail norm (conversion first); S_conv the state
    right after the conversion;
    a, U, V final factors; S final reconstructed state; S0 the prefill state;
    and, with keep_shadow, S_exact (final open-loop dense state),
    err_open (T, n) ||S~_t - S_t^exact||_F and sink_dev (T, n) max |a_t - sink(S_t^exact)|.
    """
    if not 0 <= lead_in < cfg.W:
        raise ValueError("lead_in must lie in [0, W)")
    b, l, h = (np.atleast_1d(np.asarray(x, dtype=np.int64)) for x in (b, l, h))
    T = cfg.n_decode if n_decode is None else n_decode
    S0 = recurrences.dense_prefill(cfg, b, l, h, n_prefill)
    vb = philox.vbar(cfg, l, h).astype(np.float64)
    a, U, V, s0 = convert.convert(S0, vb, cfg.R)
    out = {"S0": S0, "vbar": vb, "conv_sigma": s0[:, :cfg.R].copy(),
           "conv_gap": compress.rel_gap(s0, cfg.R), "S_conv": factored.reconstruct(a, U, V, vb)}
    tails = [compress.tail_norm(s0, cfg.R)]
    S_exact = S0.copy()
    o_all, a_all, ncols_all, sig, gaps, comp_steps = [], [], [], [], [], []
    err_open, sink_dev = [], []
    ncols = cfg.R
    # ragged schedules: a request that joined `lead_in` steps before the others has
    # taken that many decode steps (inputs of the lead-in phase) before step 0, so
    # it holds R + lead_in columns and compresses after steps W - lead_in, 2W - lead_in, ...
    for j in range(lead_in):
        inp = recurrences.f64(philox.token_inputs(cfg, b, l, h, j, philox.PHASE_LEADIN))
        a, U, V, _ = factored.step(cfg.form, a, U, V, vb, inp["q"], inp["k"], inp["v"],
                                   inp["alpha"], inp["beta"])
        ncols += 1
        if keep_shadow:
            S_exact = recurrences.dense_step(cfg.form, S_exact, inp["k"], inp["v"],
                                             inp["alpha"], inp["beta"])
    for t in range(T):
        inp = recurrences.f64(philox.token_inputs(cfg, b, l, h, t, philox.PHASE_DECODE))
        a, U, V, o = factored.step(cfg.form, a, U, V, vb, inp["q"], inp["k"], inp["v"],
                                   inp["alpha"], inp["beta"])
        ncols += 1
        if ncols == cfg.R + cfg.W:
            U, V, s = compress.truncate_qr_core(U, V, cfg.R)
            sig.append(s[:, :cfg.R].copy())
            gaps.append(compress.rel_gap(s, cfg.R))
            tails.append(compress.tail_norm(s, cfg.R))
            comp_steps.append(t + 1)
            ncols = cfg.R
        o_all.append(o)
        a_all.append(a.copy())
        ncols_all.append(ncols)
        if keep_shadow:
            S_exact = recurrences.dense_step(cfg.form, S_exact, inp["k"], inp["v"],
                                             inp["alpha"], inp["beta"])
            S_t = factored.reconstruct(a, U, V, vb)
            err_open.append(np.sqrt(np.sum((S_t - S_exact) ** 2, axis=(1, 2))))
            sink_dev.append(np.max(np.abs(a - factored.sink_coefficient(S_exact, vb)), axis=1))
    out.update(
        o=np.array(o_all), a_t=np.array(a_all), ncols=np.array(ncols_all, dtype=np.int64),
        comp_steps=comp_steps,
        sigma=np.array(sig) if sig else np.zeros((0, b.size, cfg.R)),
        gap=np.array(gaps) if gaps else np.zeros((0, b.size)),
        tail=np.array(tails), a=a, U=U, V=V, S=factored.reconstruct(a, U, V, vb))
    if keep_shadow:
        out.update(S_exact=S_exact, err_open=np.array(err_open), sink_dev=np.array(sink_dev))
    return out
