"""Helpers shared by the tests: bit views between torch and the oracle's
numpy arrays, and the comparison metrics the parity bar is stated in."""

import numpy as np
import torch

import oracle


def bits(t: torch.Tensor) -> np.ndarray:
    """BF16 tensor (any device) -> uint16 numpy bit patterns."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def codes(t: torch.Tensor) -> np.ndarray:
    """FP8 tensor (any device) -> uint8 numpy codes."""
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def from_bits(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def from_codes(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).view(torch.float8_e4m3fn).to(device)


def scalar(v: float, device) -> torch.Tensor:
    return torch.tensor([v], dtype=torch.float32, device=device)


def ordinal(c: np.ndarray) -> np.ndarray:
    """Position of an E4M3 code on the number line (+-0 both 0)."""
    c = c.astype(np.int32)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def code_step_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    return np.abs(ordinal(a) - ordinal(b))


def is_nan_code(c: np.ndarray) -> np.ndarray:
    return (c & 0x7F) == 0x7F


def rel_fro(y_bits: np.ndarray, ref_bits: np.ndarray) -> float:
    y = oracle.bf16_to_f64(y_bits)
    r = oracle.bf16_to_f64(ref_bits)
    return float(np.linalg.norm(y - r) / max(np.linalg.norm(r), 1e-300))


def gemm_elementwise_bound_ok(y_bits, ref_bits, abssum_bits, K):
    """|y - ref| <= 2^-7 |ref| + K * 2^-21 * sum_k |x_k w_k| * scale: one BF16
    rounding step plus a worst-case fp32 accumulation error (with slack for a
    tensor-core accumulator a few bits short of fp32)."""
    y = oracle.bf16_to_f64(y_bits)
    r = oracle.bf16_to_f64(ref_bits)
    a = np.abs(oracle.bf16_to_f64(abssum_bits))
    bound = 2.0 ** -7 * np.abs(r) + K * 2.0 ** -21 * a * 1.01 + 1e-30
    return np.abs(y - r) <= bound


# The parity bars (floating point tolerances come from the stated requirement):
GEMM_REL_FRO = 1e-2          # GEMM and MLP BF16 outputs, relative Frobenius
SWIGLU_MAX_STEP = 1          # SwiGLU-quant codes: at most one E4M3 step apart ...
SWIGLU_MAX_FRAC = 1e-4       # ... on at most this fraction of elements


def stratified_rows(M: int, seed: int, block: int = 128, extra: int = 4) -> np.ndarray:
    """Rows of an [M, ...] output for a sampled oracle check that reach every
    place a tile-level fault could hide: one row in every `block`-row slab
    (128 = one CTA's half of a CTA-pair tile, so both CTAs of every pair tile
    are covered), cycling through the four 32-row epilogue-warp quarters of
    the slab from one slab to the next, plus the first and last rows (the last
    one lies in the ragged final tile when M is not a multiple of the tile)
    and `extra` uniformly drawn rows.  Sorted, without repeats."""
    rng = np.random.default_rng(seed)
    rows = {0, M - 1}
    for i, b0 in enumerate(range(0, M, block)):
        lo = b0 + (i % 4) * 32
        hi = min(lo + 32, M)
        if lo >= M:
            lo, hi = b0, min(b0 + block, M)
        rows.add(int(rng.integers(lo, hi)))
    rows.update(int(r) for r in rng.choice(M, min(extra, M), replace=False))
    return np.array(sorted(rows), dtype=np.int64)
