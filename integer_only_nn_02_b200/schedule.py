"""Learning-rate schedule of the paper's training runs as the integer multiply-shift that
the SGD kernels take.

"Memory-Efficient Integer-Only Training of Deep Neural Networks", Table 10: every run
uses SGD with momentum 0.9 and a cosine learning rate with linear warmup (base LR
0.1 / 0.05 / 0.001 by model, 0 or 5 warmup epochs).  The kernels apply the rate as
lr = lr_mul * 2^-lr_shift, an integer multiply and a shift of the exponent.  The host
evaluates the schedule once per step and picks the multiply-shift closest to it with a
multiplier of at most `bits` bits; nothing on the device sees a floating-point value.
"""
from __future__ import annotations

import math


def cosine_warmup(step: int, total_steps: int, base_lr: float, warmup_steps: int = 0,
                  final_lr: float = 0.0) -> float:
    """Linear warmup from base_lr / warmup_steps to base_lr over the first warmup_steps
    steps, then a half cosine from base_lr down to final_lr at total_steps."""
    if step < 0 or total_steps <= 0:
        raise ValueError("step must be >= 0 and total_steps > 0")
    if warmup_steps > 0 and step < warmup_steps:
        return base_lr * (step + 1) / warmup_steps
    span = max(1, total_steps - warmup_steps)
    t = min(1.0, (step - warmup_steps) / span)
    return final_lr + (base_lr - final_lr) * 0.5 * (1.0 + math.cos(math.pi * t))


def mul_shift(x: float, bits: int = 8, max_shift: int = 62) -> tuple[int, int]:
    """(mul, shift) with mul * 2^-shift nearest to x >= 0, 0 <= mul < 2^bits and
    0 <= shift <= max_shift; (0, 0) for x = 0 (or below the smallest representable step)."""
    if x < 0 or bits < 1:
        raise ValueError("x must be >= 0 and bits >= 1")
    if x == 0:
        return 0, 0
    # the largest shift whose multiplier still fits in `bits` bits
    shift = bits - 1 - math.floor(math.log2(x))
    shift = max(0, min(shift, max_shift))
    mul = round(x * 2.0 ** shift)
    while mul >= (1 << bits) and shift > 0:  # rounding carried into another bit
        shift -= 1
        mul = round(x * 2.0 ** shift)
    if mul >= (1 << bits):
        raise ValueError(f"{x} needs more than {bits} bits with a non-negative shift")
    return (mul, shift) if mul else (0, 0)


def lr_mul_shift(step: int, total_steps: int, base_lr: float, warmup_steps: int = 0,
                 bits: int = 8) -> tuple[int, int]:
    """The SGD kernels' (lr_mul, lr_shift) at `step` of a cosine-with-warmup run."""
    return mul_shift(cosine_warmup(step, total_steps, base_lr, warmup_steps), bits)


MOMENTUM_0_9 = (230, 8)      # 0.8984, the momentum of every run in Table 10
WEIGHT_DECAY_1E_4 = (105, 20)  # 1.0014e-4, the weight decay of every run in Table 10
