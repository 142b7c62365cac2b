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


def scatter_row_sums(sums: torch.Tensor, shard: torch.Tensor, group=None) -> None:
    """SUM over the ranks of `sums` ([world * c] rows), rank r keeping rows [r c, (r+1) c)
    in `shard` ([c] rows).  With one rank the shard is the whole tensor."""
    if world_size(group) > 1:
        dist.reduce_scatter_tensor(shard, sums, op=dist.ReduceOp.SUM, group=group)
    else:
        shard.copy_(sums)


def gather_rows(t: torch.Tensor, group=None) -> None:
    """Every rank's block of rows of `t` ([world * c] rows, rank r owning [r c, (r+1) c))
    copied to every rank, in place."""
    world = world_size(group)
    if world > 1:
        c = t.shape[0] // world
        r = dist.get_rank(group)
        dist.all_gather_into_tensor(t, t[r * c:(r + 1) * c], group=group)


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


class ShardedLinearUpdate:
    """Backward weight and SGD step of one linear layer with the optimizer state sharded
    over the ranks (reduce-scatter form).  The weight has row-local groups, so rows are
    independent through the FIT of dW and the SGD step:

      1. targets and their MAX all-reduce, the shard's exact sums (as LinearWeightGrad);
      2. reduce-scatter of the sums over rows: rank r receives the summed rows
         [r c, (r + 1) c) of dW, c = ceil(M / world);
      3. FIT of those rows into its dW rows, the SGD step on its rows of W and of the
         velocity V (V is only held for those rows);
      4. all-gather of the updated W rows (mantissas and exponents) into every rank's W.

    Every rank ends with the W a single device computes on the whole batch, bit for bit;
    each rank sends about half the bytes of the all-reduce form and holds 1/world of V.
    The object owns W (rows padded to a multiple of world) and the velocity shard; use
    `self.W` as the layer's weight.
    """

    def __init__(self, dY: ict.DevCE, X: ict.DevCE, W: ict.DevCE, V: ict.DevCE, group=None,
                 total_rows: int | None = None, mom=(230, 8), lr=(1, 4)):
        if W.g_rows != 1 and W.rows > 1:
            raise ValueError("the weight's groups must be row-local")
        self.group, self.mom, self.lr = group, mom, lr
        self.world = world_size(group)
        self.rank = dist.get_rank(group) if self.world > 1 else 0
        self.grad = LinearWeightGrad(dY, X, group, total_rows)
        M, N, G = W.rows, W.cols, W.g_cols
        self.M, self.chunk = M, -(-M // self.world)
        Mp = self.chunk * self.world
        dev = W.mant.device
        ngc = W.exp.shape[1]
        # the weight, rows padded to Mp so that each rank's rows are one equal block
        self.w_mant = torch.zeros((Mp, W.mant.shape[1]), dtype=torch.int8, device=dev)
        self.w_exp = torch.full((Mp, ngc), -128, dtype=torch.int8, device=dev)
        self.w_mant[:M].copy_(W.mant)
        self.w_exp[:M].copy_(W.exp)
        self.W = ict.DevCE(self.w_mant[:M], self.w_exp[:M], 1, G, cols=N)
        r0, r1 = self.rank * self.chunk, min(M, (self.rank + 1) * self.chunk)
        self.r0, self.r1 = r0, r1
        self.W_shard = ict.DevCE(self.w_mant[r0:r1], self.w_exp[r0:r1], 1, G, cols=N) if r1 > r0 else None
        self.V_shard = None
        if r1 > r0:
            vm = V.mant[r0:r1].clone()
            ve = V.exp[r0:r1].clone()
            self.V_shard = ict.DevCE(vm, ve, 1, G, cols=N)
            self.dW_shard = ict.DevCE.empty(r1 - r0, N, 1, G)
        acc = self.grad.acc_buf
        self.sums = torch.zeros((Mp, acc.shape[1]), dtype=acc.dtype, device=dev)  # padded rows stay 0
        self.sums_shard = torch.empty((self.chunk, acc.shape[1]), dtype=acc.dtype, device=dev)

    @property
    def exchanged_bytes(self) -> int:
        """Bytes each rank contributes per call: targets, one row block of sums, W rows."""
        g = self.grad
        return (g.e.numel() + self.sums_shard.numel() * self.sums_shard.element_size()
                + self.chunk * (self.w_mant.shape[1] + self.w_exp.shape[1]))

    def __call__(self, dY: ict.DevCE, X: ict.DevCE) -> None:
        g = self.grad
        ict.ict_linear_bwd_weight_targets(dY, X, g.e_dy, g.e_x, g.ws)
        merge_targets(g.e, self.group)
        ict.ict_linear_bwd_weight_partial(dY, X, g.e_dy, g.e_x, self.sums[: self.M, : g.N], g.ws)
        mine = self.sums[: self.M]
        if self.world > 1:
            scatter_row_sums(self.sums, self.sums_shard, self.group)
            mine = self.sums_shard[: self.r1 - self.r0]
        if self.r1 > self.r0:
            ict.ict_requant(mine[:, : g.N], self.dW_shard, 0, g.e_dy[self.r0:self.r1], g.e_x)
            ict.ict_sgd_momentum_step(self.W_shard, self.V_shard, self.dW_shard, self.mom, self.lr)
        gather_rows(self.w_mant, self.group)
        gather_rows(self.w_exp, self.group)
