"""Seeded synthetic inputs for the integer-only (C,e) training path.

This module holds the tensor container and the random draws, nothing else: none of
the method's arithmetic lives here, so the CPU oracle and the CUDA path both draw
their inputs from it.

Every draw uses numpy's PCG64 ``default_rng(seed)``, in the order the config
builders below list.  The shapes are the layer shapes of the networks the paper
trains ("Memory-Efficient Integer-Only Training of Deep Neural Networks",
Abstract and Table 9: ResNet-18/50, ViT-Ti/B); no dataset is involved.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

E_ZERO = -128  # exponent byte of an all-zero group


def cdiv(a: int, b: int) -> int:
    return -(-a // b)


@dataclass
class CE:
    """A (C,e) matrix: int8 mantissas [rows, cols] and an int8 exponent per group.

    Groups are ``g_rows`` x ``g_cols`` blocks; the exponent grid is
    ``[cdiv(rows, g_rows), cdiv(cols, g_cols)]`` row-major.  Edge groups may be short.
    """

    mant: np.ndarray
    exp: np.ndarray
    g_rows: int
    g_cols: int
    meta: dict = field(default_factory=dict)

    @property
    def rows(self) -> int:
        return int(self.mant.shape[0])

    @property
    def cols(self) -> int:
        return int(self.mant.shape[1])

    @property
    def grid(self) -> tuple[int, int]:
        return cdiv(self.rows, self.g_rows), cdiv(self.cols, self.g_cols)

    def copy(self) -> "CE":
        return CE(self.mant.copy(), self.exp.copy(), self.g_rows, self.g_cols, dict(self.meta))


def empty_ce(rows: int, cols: int, g_rows: int, g_cols: int) -> CE:
    g_rows = max(1, min(g_rows, rows)) if rows else max(1, g_rows)
    g_cols = max(1, min(g_cols, cols)) if cols else max(1, g_cols)
    return CE(
        np.zeros((rows, cols), np.int8),
        np.full((cdiv(rows, g_rows), cdiv(cols, g_cols)), E_ZERO, np.int8),
        g_rows,
        g_cols,
    )


# --------------------------------------------------------------------------- draws


def uniform(rng, shape):
    """Mantissas uniform in [-127, 127]."""
    return rng.integers(-127, 128, size=shape).astype(np.int8)


def clipped_gaussian(rng, shape, sigma):
    return np.clip(np.rint(rng.normal(0.0, sigma, size=shape)), -127, 127).astype(np.int8)


def clipped_laplace(rng, shape, scale=16.0):
    return np.clip(np.rint(rng.laplace(0.0, scale, size=shape)), -127, 127).astype(np.int8)


def relu_like(rng, shape):
    """50 % zeros, nonzeros uniform in [1, 127] (post-ReLU activations)."""
    zero = rng.random(size=shape) < 0.5
    vals = rng.integers(1, 128, size=shape)
    return np.where(zero, 0, vals).astype(np.int8)


def exps(rng, shape, lo, hi):
    """Exponent bytes uniform in [lo, hi]."""
    return rng.integers(lo, hi + 1, size=shape).astype(np.int8)


def with_groups(mant, g_rows, g_cols, exp_draw):
    """Attach an exponent grid drawn by ``exp_draw(grid_shape)``."""
    rows, cols = mant.shape
    g_rows = max(1, min(g_rows, rows))
    g_cols = max(1, min(g_cols, cols))
    grid = (cdiv(rows, g_rows), cdiv(cols, g_cols))
    return CE(mant, np.asarray(exp_draw(grid), dtype=np.int8).reshape(grid), g_rows, g_cols)


def zero_velocity(rows, cols, g_rows, g_cols):
    """Zero-initialised velocity: C = 0, every group E_ZERO."""
    return empty_ce(rows, cols, g_rows, g_cols)


# --------------------------------------------------------------------------- configs

MOMENTUM = (230, 8)  # beta = 0.9 as the multiply-shift 230 >> 8 (Table 10: momentum 0.9)


def single_linear(seed=0, m=64, k=128, n=64):
    """Single integer linear layer fwd + bwd + SGD step (64x128 weight, 64 tokens)."""
    rng = np.random.default_rng(seed)
    X = with_groups(uniform(rng, (m, k)), m, k, lambda g: np.full(g, -7))
    W = with_groups(uniform(rng, (n, k)), 1, k, lambda g: exps(rng, g, -10, -6))
    dY = with_groups(uniform(rng, (m, n)), m, n, lambda g: np.full(g, -12))
    V = zero_velocity(n, k, 1, k)
    return dict(
        X=X, W=W, dY=dY, V=V, out_group=32, sgd=dict(mom=MOMENTUM, lr=(1, 4)),
        shapes=dict(M=m, K=k, N=n),
    )


def vit_ti_mlp(seed=0, tokens=64 * 197, d=192, hidden=768, group=32):
    """ViT-Ti MLP block step: tokens x 192 -> 768 -> 192, integer GELU in between."""
    rng = np.random.default_rng(seed)
    X = with_groups(clipped_gaussian(rng, (tokens, d), 32), 1, d, lambda g: exps(rng, g, -8, -6))
    W1 = with_groups(uniform(rng, (hidden, d)), 1, d, lambda g: exps(rng, g, -10, -6))
    W2 = with_groups(uniform(rng, (d, hidden)), 1, hidden, lambda g: exps(rng, g, -10, -6))
    dY2 = with_groups(clipped_laplace(rng, (tokens, d)), 1, d, lambda g: exps(rng, g, -14, -12))
    V1 = zero_velocity(hidden, d, 1, d)
    V2 = zero_velocity(d, hidden, 1, hidden)
    return dict(
        X=X, W1=W1, W2=W2, dY2=dY2, V1=V1, V2=V2, out_group=group,
        sgd=dict(mom=MOMENTUM, lr=(1, 4)), shapes=dict(M=tokens, D=d, H=hidden),
    )


def resnet18_conv3x3(seed=0, n=128, h=56, w=56, c=64, k=64, group=32):
    """ResNet-18 stage-1 3x3 conv, stride 1, pad 1, NHWC activations, KRSC weights."""
    rng = np.random.default_rng(seed)
    npix = n * h * w
    X = with_groups(relu_like(rng, (npix, c)), npix, group, lambda g: exps(rng, g, -8, -6))
    W = with_groups(uniform(rng, (k, 9 * c)), 1, 9 * c, lambda g: exps(rng, g, -10, -6))
    dY = with_groups(clipped_laplace(rng, (npix, k)), npix, group, lambda g: exps(rng, g, -14, -12))
    conv = dict(n=n, h=h, w=w, c=c, k=k, r=3, s=3, stride=1, pad=1)
    return dict(X=X, W=W, dY=dY, conv=conv, out_group=group)


def resnet18_block_tail(seed=0, n=128, h=56, w=56, c=64, group=32):
    """Tensors around a ResNet-18 stage-1 basic block's convolutions (NHWC, channel groups
    spanning all pixels): the second conv's output Y (signed, before the residual add),
    the block input X (post-ReLU), the upstream gradient dA and the conv branch's input
    gradient dXc (signed)."""
    rng = np.random.default_rng(seed)
    npix = n * h * w
    Y = with_groups(clipped_gaussian(rng, (npix, c), 32), npix, group, lambda g: exps(rng, g, -8, -6))
    X = with_groups(relu_like(rng, (npix, c)), npix, group, lambda g: exps(rng, g, -8, -6))
    dA = with_groups(clipped_laplace(rng, (npix, c)), npix, group, lambda g: exps(rng, g, -14, -12))
    dXc = with_groups(clipped_laplace(rng, (npix, c)), npix, group, lambda g: exps(rng, g, -15, -12))
    return dict(Y=Y, X=X, dA=dA, dXc=dXc, shape=dict(n=n, h=h, w=w, c=c), group=group)


def vit_b_linear_trio(seed=0, tokens=64 * 197, d=768, hidden=3072, group=64):
    """ViT-B MLP linears 768 -> 3072 -> 768: fwd, bwd-data, bwd-weight for both."""
    rng = np.random.default_rng(seed)
    X = with_groups(clipped_gaussian(rng, (tokens, d), 24), 1, group, lambda g: exps(rng, g, -9, -7))
    W1 = with_groups(clipped_gaussian(rng, (hidden, d), 24), 1, group, lambda g: exps(rng, g, -10, -8))
    W2 = with_groups(clipped_gaussian(rng, (d, hidden), 24), 1, group, lambda g: exps(rng, g, -10, -8))
    dY1 = with_groups(clipped_laplace(rng, (tokens, hidden)), 1, group, lambda g: exps(rng, g, -14, -12))
    dY2 = with_groups(clipped_laplace(rng, (tokens, d)), 1, group, lambda g: exps(rng, g, -14, -12))
    return dict(X=X, W1=W1, W2=W2, dY1=dY1, dY2=dY2, out_group=group,
                shapes=dict(M=tokens, D=d, H=hidden))


def resnet50_param_shapes():
    """Parameter tensor shapes of ResNet-50 (torchvision layout): 161 tensors."""
    shapes = [(64, 3, 7, 7), (64,), (64,)]
    inplanes = 64
    for width, blocks in ((64, 3), (128, 4), (256, 6), (512, 3)):
        out = width * 4
        for b in range(blocks):
            shapes += [(width, inplanes, 1, 1), (width,), (width,),
                       (width, width, 3, 3), (width,), (width,),
                       (out, width, 1, 1), (out,), (out,)]
            if b == 0:
                shapes += [(out, inplanes, 1, 1), (out,), (out,)]
            inplanes = out
    shapes += [(1000, 2048), (1000,)]
    return shapes


def resnet50_sgd_arena(seed=0, group=64, lo=-16, hi=-4):
    """ResNet-50-sized SGD state as one padded arena of rows of ``group`` elements.

    Each parameter tensor is flattened and padded with zeros to a multiple of
    ``group`` so that no group crosses a tensor boundary; the arena is a
    [n_groups, group] (C,e) matrix with one exponent per row.  W and V mantissas are
    uniform, G mantissas clipped Laplace(16); exponents per group uniform in
    [lo, hi], drawn independently for W, V and G.
    """
    rng = np.random.default_rng(seed)
    shapes = resnet50_param_shapes()
    numels = [int(np.prod(s)) for s in shapes]
    rows = [cdiv(n, group) for n in numels]
    n_rows = sum(rows)
    valid = np.zeros((n_rows, group), bool)
    r0 = 0
    for n, nr in zip(numels, rows):
        flat = np.zeros(nr * group, bool)
        flat[:n] = True
        valid[r0:r0 + nr] = flat.reshape(nr, group)
        r0 += nr

    def draw(mant_fn):
        m = mant_fn(rng, (n_rows, group))
        m = np.where(valid, m, 0).astype(np.int8)
        e = exps(rng, (n_rows, 1), lo, hi)
        return CE(m, e, 1, group)

    W = draw(uniform)
    V = draw(uniform)
    G = draw(lambda r, s: clipped_laplace(r, s))
    return dict(W=W, V=V, G=G, numel=sum(numels), n_tensors=len(shapes),
                sgd=dict(mom=MOMENTUM, lr=(205, 11)), valid=valid)


CONFIGS = {
    "single_linear": single_linear,
    "vit_ti_mlp": vit_ti_mlp,
    "resnet18_conv3x3": resnet18_conv3x3,
    "vit_b_linear_trio": vit_b_linear_trio,
    "resnet50_sgd": resnet50_sgd_arena,
}
