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


def _conv_batch(seed=5, n=2, h=4, w=4, c=64, k=64, G=32):
    from integer_only_nn_02_b200.workloads import clipped_laplace, relu_like

    rng = np.random.default_rng(seed)
    npix = n * h * w
    X = with_groups(relu_like(rng, (npix, c)), npix, G, lambda g: rng.integers(-9, -5, size=g))
    W = with_groups(rng.integers(-127, 128, size=(k, 9 * c)).astype(np.int8), 1, 9 * c,
                    lambda g: rng.integers(-11, -6, size=g))
    dY = with_groups(clipped_laplace(rng, (npix, k)), npix, G, lambda g: rng.integers(-14, -11, size=g))
    return X, W, dY, dict(n=n, h=h, w=w, c=c, k=k, r=3, s=3, stride=1, pad=1), G


def _conv_rank(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        X, W, dY, d, G = _conv_batch()
        hw = d["h"] * d["w"]
        rows = slice(rank * hw, (rank + 1) * hw)  # one image per rank
        Xr = CE(X.mant[rows].copy(), X.exp.copy(), hw, G)
        dYr = CE(dY.mant[rows].copy(), dY.exp.copy(), hw, G)
        dr = dict(d, n=1)
        # forward: the shard's largest need per output group column, MAX over the ranks
        acc, r = oracle.conv_acc(oracle.CONV_FWD, dr, Xr, W)
        need = np.full(d["k"] // G, -(2 ** 30), np.int32)
        for i, j in zip(*np.nonzero(acc)):
            need[j // G] = max(need[j // G], oracle.need(int(acc[i, j]), int(r[i, j])))
        t = torch.from_numpy(need)
        dp.merge_targets(t)
        # backward weight: exact int64 sums of the shard, SUM over the ranks
        accw, _ = oracle.conv_acc(oracle.CONV_BWD_WEIGHT, dr, dYr, Xr)
        s = torch.from_numpy(accw.copy())
        dp.merge_sums(s)
        np.savez(os.path.join(out_dir, f"c{rank}.npz"), need=t.numpy(), accw=s.numpy())
    finally:
        dist.destroy_process_group()


def test_two_ranks_conv_exchanges(tmp_path):
    """Convolution split by images: the MAX of the ranks' group needs is the whole batch's
    group exponent, and the SUM of their int64 dW sums is the whole batch's sums."""
    mp.spawn(_conv_rank, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    X, W, dY, d, G = _conv_batch()
    Y = oracle.conv(oracle.CONV_FWD, d, X, W, X.rows, G)
    accw, _ = oracle.conv_acc(oracle.CONV_BWD_WEIGHT, d, dY, X)
    for r in range(2):
        got = np.load(tmp_path / f"c{r}.npz")
        # the exponent FIT picks from the largest need: raised to -127, E_ZERO for none
        exps = [E_ZERO if n < -(2 ** 29) else max(int(n), -127) for n in got["need"]]
        assert exps == Y.exp[0].tolist(), f"rank {r}"
        assert np.array_equal(got["accw"], accw), f"rank {r}"


def _sharded_rank(rank, world, port, out_dir):
    """Reduce-scatter form on the oracle: each rank rounds and updates only its rows of
    W and V, then the rows are gathered."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        K, M, N, G = 90, 24, 40, 40
        dY, X = _batch(K, M, N, seed=9)
        rng = np.random.default_rng(10)
        W = with_groups(rng.integers(-127, 128, size=(M, N)).astype(np.int8), 1, G, lambda s: rng.integers(-9, -6, size=s))
        V = with_groups(rng.integers(-127, 128, size=(M, N)).astype(np.int8), 1, G, lambda s: rng.integers(-14, -10, size=s))
        a, b = [(0, 40), (40, 90)][rank]
        sdy, sx = _shard(dY, a, b), _shard(X, a, b)
        e = torch.from_numpy(np.concatenate([oracle.align(sdy, 0)[1], oracle.align(sx, 0)[1]]))
        dp.merge_targets(e)
        e_dy, e_x = e[:M].numpy(), e[M:].numpy()
        acc = oracle.align_to(sdy, 0, e_dy).astype(np.int64).T @ oracle.align_to(sx, 0, e_x).astype(np.int64)
        c = -(-M // world)
        sums = torch.zeros((c * world, N), dtype=torch.int64)
        sums[:M] = torch.from_numpy(acc)
        shard = torch.empty((c, N), dtype=torch.int64)
        dp.scatter_row_sums(sums, shard)
        r0, r1 = rank * c, min(M, (rank + 1) * c)
        dW = oracle.requant(shard[: r1 - r0].numpy(), 1, G, 0, row_exp=e_dy[r0:r1], col_exp=e_x)
        rows = lambda t: CE(t.mant[r0:r1].copy(), t.exp[r0:r1].copy(), 1, G)
        Wn, _ = oracle.sgd_step(rows(W), rows(V), dW)
        wm = torch.zeros((c * world, N), dtype=torch.int8)
        we = torch.zeros((c * world, 1), dtype=torch.int8)
        wm[r0:r1] = torch.from_numpy(Wn.mant)
        we[r0:r1] = torch.from_numpy(Wn.exp)
        dp.gather_rows(wm)
        dp.gather_rows(we)
        np.savez(os.path.join(out_dir, f"s{rank}.npz"), mant=wm[:M].numpy(), exp=we[:M].numpy())
    finally:
        dist.destroy_process_group()


def test_two_ranks_sharded_update_matches_single_device(tmp_path):
    mp.spawn(_sharded_rank, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    K, M, N, G = 90, 24, 40, 40
    dY, X = _batch(K, M, N, seed=9)
    rng = np.random.default_rng(10)
    W = with_groups(rng.integers(-127, 128, size=(M, N)).astype(np.int8), 1, G, lambda s: rng.integers(-9, -6, size=s))
    V = with_groups(rng.integers(-127, 128, size=(M, N)).astype(np.int8), 1, G, lambda s: rng.integers(-14, -10, size=s))
    Wn, _ = oracle.sgd_step(W, V, oracle.linear_bwd_weight(dY, X, 1, G))
    for r in range(2):
        got = np.load(tmp_path / f"s{r}.npz")
        assert np.array_equal(got["mant"], Wn.mant) and np.array_equal(got["exp"], Wn.exp), f"rank {r}"
