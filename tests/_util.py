"""Test helpers: moving bf16 bit patterns between numpy and the GPU, and the
parity tolerance.  The tolerance is the one stated for this layer pair:
max|gpu - oracle| <= 2e-2 * RMS(oracle) and ||gpu - oracle||_F / ||oracle||_F <= 5e-3."""
import numpy as np

import synthetic as syn

MAX_REL_RMS = 2e-2
FROB_REL = 5e-3


def to_dev(bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device)


def from_dev(t) -> np.ndarray:
    return t.detach().cpu().contiguous().view(__import__("torch").int16).numpy().view(np.uint16)


def f64(bits) -> np.ndarray:
    return syn.bf16_bits_to_f64(bits)


def errors(gpu_bits: np.ndarray, ref: np.ndarray):
    g = f64(gpu_bits)
    ref = np.asarray(ref, dtype=np.float64)
    d = g - ref
    rms = float(np.sqrt(np.mean(ref * ref)))
    max_rel = float(np.max(np.abs(d)) / rms) if rms > 0 else float(np.max(np.abs(d)))
    frob = float(np.linalg.norm(d) / np.linalg.norm(ref)) if np.linalg.norm(ref) > 0 else float(np.linalg.norm(d))
    return max_rel, frob


def assert_rounded_once(gpu_bits: np.ndarray, ref: np.ndarray, what: str = "", floor: float = 4e-3):
    """Bound for an intermediate that the kernel rounds once to bf16 (e.g. the
    attention output O, whose values are heavy-tailed: a query with one dominant
    key returns about that key's V row, many times RMS(O)).  Each element may be
    off by one bf16 rounding, |d| <= 2^-8 |ref|, plus fp32/fp16 arithmetic
    upstream of the rounding, bounded by `floor` * RMS(ref); the Frobenius
    bound of the layer outputs still applies."""
    g = f64(gpu_bits)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values in GPU output"
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    excess = np.abs(g - ref) - (2.0 ** -8 * np.abs(ref) + floor * rms)
    frob = float(np.linalg.norm(g - ref) / np.linalg.norm(ref))
    assert np.max(excess) <= 0 and frob <= FROB_REL, (
        f"{what}: worst excess over 2^-8|ref|+{floor}*rms = {np.max(excess):.3e}, frob={frob:.3e}")


def assert_parity(gpu_bits: np.ndarray, ref: np.ndarray, what: str = ""):
    assert np.all(np.isfinite(f64(gpu_bits))), f"{what}: non-finite values in GPU output"
    max_rel, frob = errors(gpu_bits, ref)
    print(f"[parity] {what}: max|d|/rms={max_rel:.4e} frob={frob:.4e}")
    assert max_rel <= MAX_REL_RMS and frob <= FROB_REL, (
        f"{what}: max|d|/rms={max_rel:.3e} (<= {MAX_REL_RMS}), frob={frob:.3e} (<= {FROB_REL})")
    return max_rel, frob
