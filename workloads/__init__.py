"""Seeded synthetic activation tensors for the five quantization workloads.

This module is shared by the CPU oracle tests, the GPU parity tests and the
benchmark.  It draws random numbers and casts them to bf16 — nothing else: it
holds none of the quantizer's arithmetic (no scales, no rounding to FP4, no
Hadamard, no normalisation).

Every tensor is drawn in float64 with ``numpy.random.default_rng(seed)`` and
cast once to bf16 with round-to-nearest-even (torch's float64 -> bfloat16
conversion).  Tensors are returned as ``uint16`` arrays holding the bf16 bit
patterns, row-major ``[M, K]`` (M tokens x K channels), so that both sides of a
parity test receive exactly the same bytes.

The workloads stand in for the LLM activations the pages quantize (Qwen-7B's
hidden size 4096 on the FP4Quant page; the 7B-70B LLaMA/Qwen layers on the
ARCQuant page).  No dataset is involved.

  nvfp4_outliers   : N(0,1), 1 % of the entries (distinct uniform positions) x20
  mxfp4_student_t  : 0.5 * Student-t(df=3)
  hadamard_channels: N(0,1), 64 fixed channels x50
  arc_activations  : N(0,1), 256 outlier channels x30, gamma ~ U(0.5, 1.5),
                     channel order from a separate 512-row calibration draw
  dual_gain        : N(0,1) x per-token gain exp(N(0,1)) (LogNormal(0,1))
  random_payload   : uniform random code bytes and scale bytes (a dequantizer
                     input that needs no quantizer run to produce)
  random_signs     : a seeded +-1 pattern (bit mask) for a random-sign rotation
"""
from __future__ import annotations

import numpy as np
import torch

__all__ = [
    "to_bf16_bits",
    "bf16_bits_to_torch",
    "nvfp4_outliers",
    "mxfp4_student_t",
    "hadamard_channels",
    "arc_activations",
    "dual_gain",
    "random_payload",
    "random_signs",
    "WORKLOADS",
]

# Full sizes (M tokens x K channels) and seeds of the five workloads.
WORKLOADS = {
    "nvfp4_256x1024": dict(M=256, K=1024, seed=1),
    "mxfp4_4096x4096": dict(M=4096, K=4096, seed=2),
    "hadamard_nvfp4_8192x4096": dict(M=8192, K=4096, seed=3),
    "arc_8192x4096": dict(M=8192, K=4096, seed=4, S=256),
    "dual_fwht512_32768x4096": dict(M=32768, K=4096, seed=5),
}


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Cast float64 values to bf16 (round to nearest even), return the bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_torch(bits: np.ndarray) -> torch.Tensor:
    """View a uint16 array of bf16 bit patterns as a torch bfloat16 CPU tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _chunked_rows(M: int, K: int, draw, chunk_rows: int = 2048) -> np.ndarray:
    out = np.empty((M, K), dtype=np.uint16)
    for r0 in range(0, M, chunk_rows):
        r1 = min(M, r0 + chunk_rows)
        out[r0:r1] = to_bf16_bits(draw(r1 - r0))
    return out


def nvfp4_outliers(M: int = 256, K: int = 1024, seed: int = 1, frac: float = 0.01,
                   gain: float = 20.0) -> np.ndarray:
    """N(0,1) with round(frac*M*K) distinct uniformly chosen entries multiplied by `gain`."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    n = int(round(frac * M * K))
    if n:
        idx = rng.choice(M * K, n, replace=False)
        x.reshape(-1)[idx] *= gain
    return to_bf16_bits(x)


def mxfp4_student_t(M: int = 4096, K: int = 4096, seed: int = 2, df: float = 3.0,
                    scale: float = 0.5) -> np.ndarray:
    """scale * Student-t(df), heavy tailed."""
    rng = np.random.default_rng(seed)
    return _chunked_rows(M, K, lambda m: scale * rng.standard_t(df, size=(m, K)))


def hadamard_channels(M: int = 8192, K: int = 4096, seed: int = 3, n_chan: int = 64,
                      gain: float = 50.0) -> np.ndarray:
    """N(0,1) with `n_chan` fixed, seeded channels (columns) multiplied by `gain`."""
    rng = np.random.default_rng(seed)
    chans = rng.choice(K, min(n_chan, K), replace=False)
    g = np.ones(K)
    g[chans] = gain
    return _chunked_rows(M, K, lambda m: rng.standard_normal((m, K)) * g)


def arc_activations(M: int = 8192, K: int = 4096, seed: int = 4, S: int = 256,
                    gain: float = 30.0, calib_rows: int = 512):
    """Activations for the fused reorder + RMSNorm + residual path.

    Returns ``(x_bits [M,K] uint16, gamma_bits [K] uint16, perm [K] int32,
    outliers [S] int32)``.

    * ``x``: N(0,1) with ``S`` seeded channels multiplied by ``gain``.
    * ``gamma``: U(0.5, 1.5) per channel, stored as bf16.
    * ``perm``: channel order for the reorder step, from a separate calibration
      draw of ``calib_rows`` rows of the same distribution: channels sorted by
      descending calibration statistic max_rows |x_calib[:, c]| * gamma[c]
      (stable, ties to the lower channel index).  ``perm[p]`` is the original
      channel placed at position ``p``.
    * ``outliers``: positions 0..S-1 of the reordered channel axis (the S
      channels with the largest calibration statistic).
    """
    rng = np.random.default_rng(seed)
    chans = rng.choice(K, min(S, K), replace=False)
    g = np.ones(K)
    g[chans] = gain
    gamma64 = rng.uniform(0.5, 1.5, size=K)
    gamma_bits = to_bf16_bits(gamma64)
    gamma_vals = (gamma_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    x_calib = rng.standard_normal((calib_rows, K)) * g
    stat = np.max(np.abs(x_calib), axis=0) * gamma_vals
    perm = np.argsort(-stat, kind="stable").astype(np.int32)
    outliers = np.arange(min(S, K), dtype=np.int32)
    x = _chunked_rows(M, K, lambda m: rng.standard_normal((m, K)) * g)
    return x, gamma_bits, perm, outliers


def dual_gain(M: int = 32768, K: int = 4096, seed: int = 5) -> np.ndarray:
    """N(0,1) times a per-token (row) gain drawn from LogNormal(0, 1)."""
    rng = np.random.default_rng(seed)
    return _chunked_rows(
        M, K, lambda m: rng.standard_normal((m, K)) * np.exp(rng.standard_normal((m, 1))))


def random_payload(M: int, K: int, fmt: str, seed: int = 6):
    """Uniform random bytes in the storage layout of a quantized [M, K] tensor.

    Returns ``(codes [M, K/2] uint8, scales uint8, scale)``: every code byte in
    0..255 (two E2M1 codes); scale bytes E4M3 in 0x08..0x6f (NVFP4 / dual) or
    E8M0 in 100..139 (MXFP4); ``scale`` a float32 tensor scale (NVFP4, INT4),
    a [M, K/128] float32 array drawn from U(1e-3, 1) (dual) or None (MXFP4).
    INT4 code bytes hold two 4-bit two's complement integers (every nibble,
    -8 included, is a valid input to a dequantizer)."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    if fmt == "mxfp4":
        return codes, rng.integers(100, 140, size=(M, K // 32), dtype=np.uint8), None
    scales = rng.integers(0x08, 0x70, size=(M, K // 16), dtype=np.uint8)
    if fmt in ("nvfp4", "int4"):
        return codes, scales, np.float32(rng.uniform(1e-3, 1.0))
    if fmt == "dual":
        return codes, scales, rng.uniform(1e-3, 1.0, size=(M, K // 128)).astype(np.float32)
    raise ValueError(fmt)


def random_signs(period: int, seed: int = 8) -> np.ndarray:
    """A uniformly random sign pattern of `period` channels as uint32 words:
    bit j (word j // 32, bit j % 32) set means channel j is negated."""
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2, size=period).astype(np.uint64)
    words = np.zeros((period + 31) // 32, np.uint32)
    for j in range(period):
        words[j // 32] |= np.uint32(int(bits[j]) << (j % 32))
    return words
