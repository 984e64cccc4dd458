"""Algorithmic byte accounting of the decode step (host logic for measurement).

Per head-step (one unit, one decode step, c columns held before the step), fp32
(with 16-bit factors, fb = 2 bytes per U and V value instead of 4; the sink, the
scales and the dense state stay fp32):

  lazy (the layout libseed uses)
    GDN, Mamba-2  4 [ d_k + (d_k + d_v + 1) c + d_k + d_k + d_v + (c + 1) ]
                  read a, the c columns of U and V and their c decay scales;
                  write a, one U column, one V column and c + 1 scales
    KDA           4 [ d_k + (d_k + d_v) c + d_k + d_k + d_v + 2 d_k ]
                  the per-channel decay product P (d_k) is read and written
                  instead of the column scales
  explicit        4 [ d_k + (d_k + d_v) c + d_k + d_k c + d_k + d_v ]
                  (U rewritten in full every step)
  table2          2 * 4 [ d_k + (d_k + d_v) (R + W/2) ]  (every state read and
                  written in full at the mean column count, the Table 2 traffic
                  convention of "Shallow Encoding Emits Deep Memories")
  dense           2 * 4 d_k d_v

The shared v̄ is not counted (Table 17 of the same page), nor are the per-step
inputs q, k, v, alpha, beta and the output o, nor the 8 bytes of the per-unit
column counter.
"""

from __future__ import annotations

FORM_KDA = 1


def lazy_bytes(form: int, d_k: int, d_v: int, c: float, fb: int = 4) -> float:
    """a read and written (4 d_k each), the c stored columns of U and V read and one
    new pair written (fb bytes a value), and the decay state read and written."""
    factors = fb * ((d_k + d_v) * c + d_k + d_v)
    if form == FORM_KDA:
        return factors + 4.0 * (2 * d_k + 2 * d_k)
    return factors + 4.0 * (2 * d_k + c + (c + 1))


def explicit_bytes(d_k: int, d_v: int, c: float, fb: int = 4) -> float:
    return fb * ((d_k + d_v) * c + d_k * c + d_k + d_v) + 4.0 * 2 * d_k


def table2_bytes(d_k: int, d_v: int, R: int, W: int, fb: int = 4) -> float:
    return 2 * (4.0 * d_k + fb * (d_k + d_v) * (R + W / 2))


def dense_bytes(d_k: int, d_v: int) -> float:
    return 2 * 4.0 * d_k * d_v


def io_bytes(form: int, d_k: int, d_v: int) -> float:
    """Per-step inputs and output of one unit: q, k, v, alpha, beta, o."""
    alpha = d_k if form == FORM_KDA else 1
    return 4.0 * (2 * d_k + 2 * d_v + alpha + 1)


def mean_columns(R: int, W: int) -> float:
    """Mean column count before a step over one compression window: R + (W - 1) / 2."""
    return R + (W - 1) / 2.0


def compress_flops(d_k: int, d_v: int, R: int, W: int, sweeps: float) -> float:
    """Floating-point operations of one unit's compression by the QR route (the
    truncation of Figure 1(b) of the SEED figures & tables page), m = R + W:

      Gram matrices of U and V           2 (d_k + d_v) m^2
      two Cholesky factorisations        2 m^3 / 3
      core M = R_u R_v^T (triangular)    2 m^3 / 3
      one-sided Jacobi, per sweep        m (m - 1) / 2 pairs x 6 m
                                         (a dot product and a rotation of two m-columns)
      left vectors and small factors     6 m^2 R
      U' and V' from the stored panels   2 (d_k + d_v) m R
    """
    m = R + W
    return (2.0 * (d_k + d_v) * m * m + 4.0 * m ** 3 / 3.0 + sweeps * (m * (m - 1) / 2.0) * 6.0 * m
            + 6.0 * m * m * R + 2.0 * (d_k + d_v) * m * R)


def fp32_peak_tflops(sm_mhz: float, sms: int = 148) -> float:
    """FP32 FMA peak of the CUDA cores: SMs x 128 lanes x 2 flops x clock."""
    return sms * 128 * 2 * sm_mhz * 1e6 / 1e12
