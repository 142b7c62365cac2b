"""The data-parallel backward weight's two collectives (integer_only_nn_02_b200.dp), run
by two gloo ranks on CPU.  Each rank computes its shard's steps with the oracle; the
ranks exchange targets and sums through dp.merge_targets / dp.merge_sums, and every rank
must end with the single-device oracle result on the whole batch, bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from integer_only_nn_02_b200 import dp
from integer_only_nn_02_b200.workloads import CE, E_ZERO, with_groups

pytestmark = pytest.mark.timeout(300)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _batch(K, M, N, seed):
    rng = np.random.default_rng(seed)

    def ce(rows, cols, elo, ehi):
        m = rng.integers(-127, 128, size=(rows, cols)).astype(np.int8)
        t = with_groups(m, 1, 8, lambda g: rng.integers(elo, ehi + 1, size=g))
        zero = rng.random(t.exp.shape) < 0.1  # some all-zero groups
        t.exp[zero] = E_ZERO
        for gi, gj in zip(*np.nonzero(zero)):
            t.mant[gi, gj * 8:(gj + 1) * 8] = 0
        return t

    return ce(K, M, -14, -3), ce(K, N, -9, -1)


def _shard(t, a, b):
    return CE(t.mant[a:b].copy(), t.exp[a:b].copy(), 1, t.g_cols)


def _rank(rank, world, port, cuts, bits, K, M, N, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dY, X = _batch(K, M, N, seed=7)
        a, b = cuts[rank]
        sdy, sx = _shard(dY, a, b), _shard(X, a, b)
        # step 1 on this shard, then the MAX exchange
        e = torch.from_numpy(np.concatenate([oracle.align(sdy, 0)[1], oracle.align(sx, 0)[1]]))
        dp.merge_targets(e)
        e_dy, e_x = e[:M].numpy(), e[M:].numpy()
        # step 3 on this shard, then the SUM exchange
        acc = oracle.align_to(sdy, 0, e_dy).astype(np.int64).T @ oracle.align_to(sx, 0, e_x).astype(np.int64)
        t = torch.from_numpy(acc.astype(np.int32 if bits == 32 else np.int64))
        dp.merge_sums(t)
        got = oracle.requant(t.numpy().astype(np.int64), 1, N, 0, row_exp=e_dy, col_exp=e_x)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), mant=got.mant, exp=got.exp)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts,bits", [([(0, 37), (37, 90)], 32), ([(0, 90), (90, 90)], 64)])
def test_two_ranks_match_single_device(tmp_path, cuts, bits):
    K, M, N = 90, 24, 40
    mp.spawn(_rank, args=(2, _free_port(), cuts, bits, K, M, N, str(tmp_path)), nprocs=2, join=True)
    dY, X = _batch(K, M, N, seed=7)
    ref = oracle.linear_bwd_weight(dY, X)
    for r in range(2):
        got = np.load(tmp_path / f"r{r}.npz")
        assert (got["mant"] == ref.mant).all() and (got["exp"] == ref.exp).all(), f"rank {r}"


def test_sum_width():
    assert dp.sum_bits(None) == 64
    assert dp.sum_bits(8 * 12608) == 32  # 100 864 * 127^2 < 2^31
    assert dp.sum_bits(133_145) == 64    # 133 145 * 127^2 >= 2^31
    assert dp.sum_bits(133_144) == 32
