"""When block-sparse attention is switched on during denoising.

The tutorial's "Quantized and sparse attention" section keeps the first
denoising steps dense and switches Sol-Attention on below a noise-level
cutoff (``disabled_until_timestep``).  Its worked figures: with the packed
time-shift schedule alpha = 6.93, a cutoff of 0.96 keeps the first 12 of 50
steps dense for the base model and the first 4 of 16 for the distilled one,
and a cutoff of 0.94 gives the recommended 16 dense steps of 50.

Reading: step t of n has the noise level sigma_t = 1 - t / n (t = 0 .. n-1,
the usual linear flow-matching grid) shifted to

    s_t = alpha * sigma_t / (1 + (alpha - 1) * sigma_t),

and step t runs dense attention while s_t >= cutoff.  The three worked
figures above hold under this reading.
"""

from __future__ import annotations


def shifted_sigma(step: int, num_steps: int, alpha: float) -> float:
    """Noise level of denoising step ``step`` (0-based) of ``num_steps``."""
    if num_steps < 1 or not 0 <= step < num_steps:
        raise ValueError("need 0 <= step < num_steps")
    sigma = 1.0 - step / num_steps
    return alpha * sigma / (1.0 + (alpha - 1.0) * sigma)


def sparse_active(step: int, num_steps: int, alpha: float, cutoff: float) -> bool:
    """True when step ``step`` runs block-sparse attention (its shifted
    noise level is below ``cutoff``)."""
    return shifted_sigma(step, num_steps, alpha) < cutoff


def dense_steps(num_steps: int, alpha: float, cutoff: float) -> int:
    """Number of initial steps that stay dense."""
    return sum(not sparse_active(t, num_steps, alpha, cutoff) for t in range(num_steps))
