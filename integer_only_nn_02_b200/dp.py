"""Data-parallel training of the integer-only (C,e) layers: one process per GPU, the
batch (tokens or images) split over the ranks of a torch.distributed process group (NCCL
over NVLink / NVSwitch between GPUs; gloo for CPU tests of the collectives).

"Memory-Efficient Integer-Only Training of Deep Neural Networks" trains ResNets and
ViTs on ImageNet (Abstract; Table 10 batch sizes), i.e. with batches that a
multi-GPU run splits this way.  Forward and backward-data Products with row-local
output groups only touch the rank's own rows.  The one exchange is in the
backward-weight Product dW = dY^T X, which contracts over the batch:

  1. each rank finds the ALIGN_MAX targets of its shard (largest group exponent of
     every column of dY and X);
  2. MAX all-reduce of those targets (int8; E_ZERO = -128 sorts below every exponent);
  3. each rank aligns its shard to the whole-batch targets and contracts it exactly
     into integer sums;
  4. SUM all-reduce of the sums (int32 when the whole batch keeps them below 2^31,
     else int64);
  5. every rank rounds the same sums (FIT) into dW.

Convolutions (ConvSplit, ConvWeightGrad): activation exponents are uniform over
pixels, so nothing is aligned across the batch.  Outputs whose channel groups span all
pixels take one MAX all-reduce of the groups' needs between the Product pass and the
rounding pass; dW takes one SUM all-reduce of int64 sums.

Integer addition is exact in any order, so every rank ends with the single-device
result on the whole batch, bit for bit, and the replicated SGD step keeps the weights
identical on all ranks.  The arithmetic is in libict's kernels; this module only holds
the buffers and issues the collectives.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import ict

QMAX = 127


def world_size(group=None) -> int:
    return dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1


def merge_targets(e: torch.Tensor, group=None) -> None:
    """Element-wise MAX over the ranks, in place: the int8 alignment targets of a
    backward-weight Product, or the int32 group needs of a split convolution."""
    if world_size(group) > 1:
        dist.all_reduce(e, op=dist.ReduceOp.MAX, group=group)


def merge_sums(acc: torch.Tensor, group=None) -> None:
    """Step 4: element-wise SUM of the exact integer sums over the ranks, in place."""
    if world_size(group) > 1:
        dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)


def sum_bits(total_rows: int | None) -> int:
    """Width of the sums: 32 bits when every sum of the whole batch stays below 2^31
    (total_rows * 127^2 < 2^31), else 64; 64 when the batch size is not known."""
    return 32 if total_rows is not None and total_rows * QMAX * QMAX < (1 << 31) else 64


class LinearWeightGrad:
    """dW = dY^T X of one linear layer over a batch split across the ranks of `group`.

    Holds the target vectors, the sums and the workspace, sized for shards of up to the
    given shapes.  `total_rows` bounds the batch size summed over all ranks; it selects
    32-bit sums (half the exchanged bytes) when they cannot overflow.
    """

    def __init__(self, dY: ict.DevCE, X: ict.DevCE, group=None, total_rows: int | None = None):
        self.group = group
        self.M, self.N = dY.cols, X.cols
        dev = dY.mant.device
        self.bits = sum_bits(total_rows)
        if self.bits == 32 and dY.rows * QMAX * QMAX >= (1 << 31):
            self.bits = 64
        # e_dy and e_x side by side: one MAX all-reduce covers both
        self.e = torch.empty(self.M + self.N, dtype=torch.int8, device=dev)
        self.e_dy, self.e_x = self.e[: self.M], self.e[self.M:]
        ld = -(-self.N // 4) * 4
        dtype = torch.int32 if self.bits == 32 else torch.int64
        self.acc_buf = torch.empty((self.M, ld), dtype=dtype, device=dev)
        self.acc = self.acc_buf[:, : self.N]
        self.ws = torch.empty(max(256, ict.ict_linear_bwd_weight_partial_workspace(dY, X)), dtype=torch.uint8,
                              device=dev)

    @property
    def exchanged_bytes(self) -> int:
        """Bytes each rank contributes to the two all-reduces of one call."""
        return self.e.numel() + self.acc.numel() * self.acc.element_size()

    def __call__(self, dY: ict.DevCE, X: ict.DevCE, dW: ict.DevCE) -> None:
        if (dY.cols, X.cols) != (self.M, self.N):
            raise ValueError("operand widths differ from the ones this object was built for")
        ict.ict_linear_bwd_weight_targets(dY, X, self.e_dy, self.e_x, self.ws)
        merge_targets(self.e, self.group)
        ict.ict_linear_bwd_weight_partial(dY, X, self.e_dy, self.e_x, self.acc, self.ws)
        merge_sums(self.acc_buf, self.group)
        ict.ict_requant(self.acc, dW, 0, self.e_dy, self.e_x)


class ConvSplit:
    """Forward or backward-data convolution over a batch split across the ranks of
    `group`, with output groups spanning all pixels (the channel groups of convolution
    activations): the shard's Product writes its int32 sums and each group's largest
    need, a MAX all-reduce of the needs gives the whole batch's group exponents, and the
    shard's rows are rounded with them.  Every rank's operands must carry the whole
    batch's exponents (true of the outputs of this class)."""

    def __init__(self, direction: int, d: dict, a: ict.DevCE, b: ict.DevCE, out: ict.DevCE, group=None):
        self.direction, self.d, self.group = direction, dict(d), group
        dev = a.mant.device
        self.need = torch.empty(-(-out.cols // min(out.g_cols, out.cols)), dtype=torch.int32, device=dev)
        self.ws = torch.empty(max(256, ict.ict_conv_workspace(direction, d)), dtype=torch.uint8, device=dev)

    def __call__(self, a: ict.DevCE, b: ict.DevCE, out: ict.DevCE) -> None:
        ict.ict_conv_split_begin(self.direction, self.d, a, b, out, self.need, self.ws)
        merge_targets(self.need, self.group)
        ict.ict_conv_split_end(self.direction, self.d, a, b, out, self.need, self.ws)


class ConvWeightGrad:
    """Convolution dW over a batch split across the ranks of `group`: exact int64 sums of
    the shard, a SUM all-reduce, one FIT (pixel-uniform operand exponents need no
    alignment, and they are the same on every rank)."""

    def __init__(self, d: dict, group=None, device="cuda"):
        self.d, self.group = dict(d), group
        K, RSC = d["k"], d["r"] * d["s"] * d["c"]
        self.acc = torch.empty((K, RSC), dtype=torch.int64, device=device)
        self.e_k = torch.empty(K, dtype=torch.int8, device=device)
        self.e_rsc = torch.empty(RSC, dtype=torch.int8, device=device)
        self.ws = torch.empty(max(256, ict.ict_conv_workspace(2, d)), dtype=torch.uint8, device=device)

    @property
    def exchanged_bytes(self) -> int:
        return self.acc.numel() * 8

    def __call__(self, dY: ict.DevCE, X: ict.DevCE, dW: ict.DevCE) -> None:
        ict.ict_conv_bwd_weight_partial(self.d, dY, X, self.acc, self.e_k, self.e_rsc, self.ws)
        merge_sums(self.acc, self.group)
        ict.ict_requant(self.acc, dW, 0, self.e_k, self.e_rsc)
