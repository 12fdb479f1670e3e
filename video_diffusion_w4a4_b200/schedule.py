"""Timestep-aware cube sizes (DeltaQuant note, training-strategy section and
the ablation table): the high-noise early denoising steps, which decide most of
the image quality, use small cubes (16 tokens, t x h x w = 4 x 1 x 4) and the
remaining steps large ones (64 tokens, 4 x 2 x 8), the early share being a
quarter to 30 % of the steps.

A policy for the caller: the cube is an argument of every forward call, so a
denoising loop asks this module which cube to pass at each step.  No arithmetic
of the layer lives here.
"""
from __future__ import annotations

EARLY_CUBE = (4, 1, 4)
LATE_CUBE = (4, 2, 8)


def cube_for_step(step: int, num_steps: int, early_fraction: float = 0.3,
                  early=EARLY_CUBE, late=LATE_CUBE) -> tuple[int, int, int]:
    """The cube for denoising step `step` (0-based) of `num_steps`: `early` for the
    first round(early_fraction * num_steps) steps, `late` afterwards."""
    if num_steps <= 0 or not 0 <= step < num_steps:
        raise ValueError(f"step {step} outside 0..{num_steps - 1}")
    if not 0.0 <= early_fraction <= 1.0:
        raise ValueError("early_fraction must lie in [0, 1]")
    n_early = int(round(early_fraction * num_steps))
    return tuple(early) if step < n_early else tuple(late)


def amortized_cube_tokens(num_steps: int, early_fraction: float = 0.3, early=EARLY_CUBE, late=LATE_CUBE) -> float:
    """The single cube size with the same total kernel-path cost over the schedule.  The
    kernel path costs in proportion to the number of cubes, 1 / (tokens per cube), so the
    amortised size is the harmonic mean of the per-step cube sizes."""
    sizes = []
    for s in range(num_steps):
        t, h, w = cube_for_step(s, num_steps, early_fraction, early, late)
        sizes.append(t * h * w)
    return len(sizes) / sum(1.0 / v for v in sizes)
