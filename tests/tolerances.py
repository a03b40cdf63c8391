"""Parity criteria between the CUDA path and the fp64 oracle.

The bars are the stated tolerances of the workloads:
  * norms (n, g): 1e-3 relative for bf16 modules, 1e-5 relative for fp32;
  * bf16 compose outputs and gradients: within 2 bf16 ulps of the oracle
    value, or within 1e-2 relative;
  * fp32 compose outputs and gradients: within 1e-5 relative.
Near exact cancellation (y close to 0 while base and lora are not) no
relative bar can hold for a value computed in fp32, so every elementwise check
adds the fp32 evaluation bound of the expression being checked: 8 * 2^-24
times the sum of the magnitudes of its terms.  dm sums T signed products in
fp32; its bound is 1e-5 of sum_t |dy (base + s lora)| / n_c (a partial sum of
at most a few hundred terms per thread, then a fixed-order tree) plus 1e-6
relative.
"""
import numpy as np

U32 = 2.0 ** -24


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def check_bf16(got, ref, term_mag, what: str):
    """got: values read back from bf16; ref: fp64 oracle; term_mag: sum of the
    magnitudes of the terms that formed each value (for the cancellation floor)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    floor = 8 * U32 * np.asarray(term_mag, dtype=np.float64)
    ok = (err <= 2 * bf16_ulp(ref) + floor) | (err <= 1e-2 * np.abs(ref) + floor)
    if not ok.all():
        i = np.argmax(~ok.ravel())
        raise AssertionError(
            f"{what}: {int((~ok).sum())} of {ok.size} outside 2 bf16 ulps / 1e-2 rel; first at "
            f"flat {i}: got {got.ravel()[i]!r} ref {ref.ravel()[i]!r}")


def check_f32(got, ref, term_mag, what: str, rtol: float = 1e-5):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    ok = err <= rtol * np.abs(ref) + 8 * U32 * np.asarray(term_mag, dtype=np.float64)
    if not ok.all():
        i = np.argmax(~ok.ravel())
        raise AssertionError(
            f"{what}: {int((~ok).sum())} of {ok.size} outside {rtol} rel; first at flat {i}: "
            f"got {got.ravel()[i]!r} ref {ref.ravel()[i]!r}")


def check_rel(got, ref, rtol: float, what: str):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    ok = err <= rtol * np.abs(ref)
    if not ok.all():
        i = np.argmax(~ok.ravel())
        raise AssertionError(
            f"{what}: {int((~ok).sum())} of {ok.size} beyond {rtol} relative; worst "
            f"{float(np.max(err / np.maximum(np.abs(ref), 1e-300))):.3e}; first at {i}: "
            f"got {got.ravel()[i]!r} ref {ref.ravel()[i]!r}")


def check_dm(got, ref, abs_sum, what: str):
    """abs_sum: sum_t |dy (base + s lora)| / n_c per column."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    ok = err <= 1e-6 * np.abs(ref) + 1e-5 * np.asarray(abs_sum, dtype=np.float64)
    if not ok.all():
        i = np.argmax(~ok.ravel())
        raise AssertionError(f"{what}: {int((~ok).sum())} of {ok.size} columns off; first {i}: "
                             f"got {got.ravel()[i]!r} ref {ref.ravel()[i]!r}")
