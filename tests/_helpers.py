"""Shared helpers for the parity tests: moving data between torch and the oracle's numpy form,
and the comparison rules.

Parity rules:
  * codes and scale bytes: bit-exact, scale bytes compared in canonical (unswizzled) form;
  * GEMM outputs: max over (m, n) of |Y_gpu - Y_ref| / (||x_m||_2 ||w_n||_2) <= 2e-3, the norms
    taken over the original bf16 rows of X and W (the Cauchy-Schwarz scale of an output).
"""
import numpy as np
import torch

import oracle as O

GEMM_TOL = 2e-3


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bits -> CUDA bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def gpu_codes(q, rows: int) -> np.ndarray:
    kp = O.kpad(q.k_aug)
    return q.codes[: rows * kp // 2].cpu().numpy().reshape(rows, kp // 2)


def gpu_sf_canonical(q, rows: int) -> np.ndarray:
    kp = O.kpad(q.k_aug)
    return O.sf_unswizzle(q.sf.cpu().numpy(), rows, kp // 16)


def gpu_sf_swizzled(q, rows: int) -> np.ndarray:
    kp = O.kpad(q.k_aug)
    return q.sf[: O.sf_swizzled_bytes(rows, kp // 16)].cpu().numpy()


def assert_codes_equal(got, want, what="codes"):
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        m, k = bad[0]
        raise AssertionError(f"{what}: {len(bad)} mismatching bytes, first at row {m} byte {k}: "
                             f"got {got[m, k]:#04x} want {want[m, k]:#04x}")


def row_norms(bits: np.ndarray) -> np.ndarray:
    f = O.bf16_bits_to_f32(bits).astype(np.float64)
    return np.sqrt((f * f).sum(axis=1))


def normalized_gemm_error(y_gpu_bits: np.ndarray, y_ref: np.ndarray, xnorm: np.ndarray, wnorm: np.ndarray,
                          with_add: bool = False) -> float:
    """max |Y_gpu - Y_ref| / (||x_m|| ||w_n||). With a residual add in the epilogue the output is
    one bf16 rounding of (product + add), whose size is set by the add term, not by the product:
    that rounding (at most 2^-8 |Y_ref|) is taken off before normalising."""
    y = O.bf16_bits_to_f32(y_gpu_bits).astype(np.float64)
    den = np.outer(xnorm, wnorm)
    den = np.where(den > 0, den, 1.0)
    diff = np.abs(y - y_ref)
    if with_add:
        diff = np.maximum(diff - 2.0 ** -8 * np.abs(y_ref), 0.0)
    return float(np.max(diff / den))
