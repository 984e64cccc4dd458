"""fp64 CPU oracle for SEED's shallow-in-representation recurrent state.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
NumPy float64 restatement of what the decode hot path computes.  Only the test
suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it.  It shares no code with the CUDA library and never imports it; the
one module both sides use is ``workloads`` (seeded input generation only).

Sources (each function cites the passage it follows), all pages about the paper
"Shallow Encoding Emits Deep Memories" (SEED):
  SEED summary (picx.dev)           - Methodology: "SEED Architecture",
                                      "Exact Update (Lemma 2)", "Open-Loop Error
                                      Bound (Corollary 4)"; Implications: Lemma 1
  SEED figures & tables (thelatestinai.com) - Figure 1(b), Table 1, Table 2,
                                      Table 17
  SEED commentary (sungsoo.github.io) - "2. Exact factored update"

Modules:
  recurrences  dense GDN / KDA / Mamba-2 steps, read-out, dense prefill
  factored     sink decomposition (Lemma 1) and the exact factored step (Lemma 2)
  compress     rank-R truncation: plain SVD of U V^T, and the QR + core-SVD route
  convert      end-of-prefill conversion of a dense state
  bytes_model  the analytical byte account (Table 17) behind Table 2
  precision    rounding to the 16-bit factor formats (Table 9)
  diagnostics  sink and content energies (Figures 3 and 12)
  run          whole trajectories (prefill, convert, decode, compress) for sampled units

Parity pins: every function above is pinned in tests/test_oracle_pins.py to a
fact the pages or the mathematics fix (Lemma 2 exactness against the dense
recurrence, Lemma 1's sink recurrence, Eckart-Young by brute force, Corollary 4,
the delta-rule write, closed-form unrolled sums, Table 2's byte values).
"""

from . import bytes_model, compress, convert, diagnostics, factored, precision, recurrences, run  # noqa: F401
