"""Error measures shared by the parity tests (numpy only, no GPU, no torch).

The layer's output gate bounds max |y - y_ref| by 1.5e-2 * RMS(y_ref), where
y_ref is the fp64 oracle.  y is bf16, whose unit roundoff is 2^-8: a value of
4 RMS carries up to 4 * 2^-8 = 1.6e-2 RMS of rounding error even when it is
computed exactly.  The measures here separate the two parts:

* ``raw_error``   max |y - y_ref| / RMS, the literal reading;
* ``gate_error``  max(|y - y_ref| - half_ulp(y_ref)) / RMS, the computation's
                  error on top of one correct rounding to the output format
                  (a correctly rounded exact result scores <= 0);
* ``vs_rounded``  max |y - RNE(y_ref)| / RMS and how many outputs differ from
                  the correctly rounded reference at all.
"""

from __future__ import annotations

import numpy as np

_MANT = {"bf16": 8, "fp16": 11}           # significant bits, implicit bit included
_TINY = {"bf16": 2.0 ** -133, "fp16": 2.0 ** -25}


def rms(a) -> float:
    return float(np.sqrt(np.mean(np.square(a))))


def round_to(ref: np.ndarray, fmt: str) -> np.ndarray:
    """fp64 -> nearest value of the format (ties to even), exactly: with
    ref = m * 2^e and m in [0.5, 1), the format keeps rint(m * 2^p) * 2^(e-p)
    for p significant bits (np.rint rounds half to even).  Normal range only,
    which covers every output of the seeded workloads."""
    p = _MANT[fmt]
    m, e = np.frexp(np.asarray(ref, np.float64))
    return np.ldexp(np.rint(np.ldexp(m, p)), e - p)


def half_ulp(ref: np.ndarray, fmt: str) -> np.ndarray:
    """Half a unit in the last place of |ref| in the output format: the error a
    correctly rounded result may carry on top of the computation's own."""
    mant = _MANT[fmt]
    e = np.floor(np.log2(np.maximum(np.abs(ref), 1e-300)))
    return np.maximum(2.0 ** (e - mant), _TINY[fmt])


def gate_error(got: np.ndarray, ref: np.ndarray, fmt: str) -> float:
    """max(|got - ref| - half_ulp(ref)) / RMS(ref); the gate is <= 1.5e-2.
    A value that is exact but for its final rounding scores <= 0."""
    excess = np.abs(got - ref) - half_ulp(ref, fmt)
    return float(np.max(excess) / max(rms(ref), 1e-30))


def raw_error(got: np.ndarray, ref: np.ndarray) -> float:
    """max |got - ref| / RMS(ref), the gate's literal reading."""
    return float(np.max(np.abs(got - ref)) / max(rms(ref), 1e-30))


def vs_rounded(got: np.ndarray, ref: np.ndarray, fmt: str):
    """(max |got - RNE(ref)| / RMS(ref), fraction of outputs != RNE(ref))."""
    rr = round_to(ref, fmt)
    diff = np.abs(got - rr)
    return float(np.max(diff) / max(rms(ref), 1e-30)), float(np.mean(diff != 0))
