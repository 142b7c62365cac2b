"""B-bit mantissas (Table 4 of "Memory-Efficient Integer-Only Training of Deep Neural
Networks" trains with INT8 down to INT4; Table 7's clip bound q_max = 2^(B-1) - 1): the
linear Products in all three directions and the SGD update against the oracle's B-bit
routines, bit for bit, for B = 2..8; INT8-only entry points refuse other widths."""
import numpy as np
import pytest

import oracle
from integer_only_nn_02_b200.workloads import CE
from tests.test_oracle_pins import rand_ce

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ict():
    from integer_only_nn_02_b200 import ict as _ict

    return _ict


def same(got: CE, ref: CE, what=""):
    assert got.mant.shape == ref.mant.shape, what
    bad = np.argwhere(got.mant != ref.mant)
    assert bad.size == 0, f"{what}: {len(bad)} mantissas differ, first {bad[:5].tolist()}"
    bad = np.argwhere(got.exp != ref.exp)
    assert bad.size == 0, f"{what}: {len(bad)} exponents differ, first {bad[:5].tolist()}"


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("M,N,K,G", [(300, 192, 160, 32), (260, 320, 768, 64), (1000, 128, 384, 128)])
def test_linear_bits(ict, bits, M, N, K, G):
    q = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(bits * 31 + M + N + K)
    X = rand_ce(rng, M, K, 1, 32, elo=-9, ehi=-6, mag=q)
    W = rand_ce(rng, N, K, 1, 64, elo=-10, ehi=-7, mag=q)
    dY = rand_ce(rng, M, N, 1, 32, elo=-14, ehi=-11, mag=q)
    d = ict.DevCE.from_host
    ict.ict_set_mantissa_bits(bits)
    try:
        Y = ict.linear_fwd(d(X), d(W), G).to_host()
        dX = ict.linear_bwd_data(d(dY), d(W), G).to_host()
        dW = ict.linear_bwd_weight(d(dY), d(X)).to_host()
    finally:
        ict.ict_set_mantissa_bits(8)
    same(Y, oracle.linear_bits(0, X, W, bits, 1, G), f"fwd B={bits}")
    same(dX, oracle.linear_bits(1, dY, W, bits, 1, G), f"bwd-data B={bits}")
    same(dW, oracle.linear_bits(2, dY, X, bits, 1, K), f"bwd-weight B={bits}")
    for t in (Y, dX, dW):
        assert np.abs(t.mant.astype(int)).max() <= q
    code, raw = ict.ict_get_device_status()
    assert code == 0, (code, raw)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("rows,cols,G", [(64, 128, 128), (100, 64, 64), (12, 768, 768), (30, 200, 64)])
def test_sgd_bits(ict, bits, rows, cols, G):
    q = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(bits * 7 + rows + cols)
    W = rand_ce(rng, rows, cols, 1, G, -16, -4, zero_groups=0.05, mag=q)
    V = rand_ce(rng, rows, cols, 1, G, -16, -4, zero_groups=0.3, mag=q)
    Gr = rand_ce(rng, rows, cols, 1, G, -16, -4, zero_groups=0.05, mag=q)
    for mom, lr in (((230, 8), (1, 4)), ((230, 8), (205, 11))):
        W2, V2 = oracle.sgd_step_bits(W, V, Gr, bits, mom, lr)
        dW, dV, dG = ict.DevCE.from_host(W), ict.DevCE.from_host(V), ict.DevCE.from_host(Gr)
        ict.ict_set_mantissa_bits(bits)
        try:
            ict.ict_sgd_momentum_step(dW, dV, dG, mom, lr)
        finally:
            ict.ict_set_mantissa_bits(8)
        same(dV.to_host(), V2, f"velocity B={bits}")
        same(dW.to_host(), W2, f"weight B={bits}")
    code, raw = ict.ict_get_device_status()
    assert code == 0, (code, raw)


def test_int8_only_entry_points_refuse_other_widths(ict):
    rng = np.random.default_rng(3)
    H = ict.DevCE.from_host(rand_ce(rng, 16, 64, 1, 32))
    dG = ict.DevCE.from_host(rand_ce(rng, 16, 64, 1, 32))
    ict.ict_set_mantissa_bits(4)
    try:
        with pytest.raises(ict.IctError) as ei:
            ict.gelu_bwd(H, dG)
        assert ei.value.code == 2
        with pytest.raises(ict.IctError):
            ict.sum_(H, dG)
        ict.gelu_fwd(H)  # never widens a mantissa: accepted
    finally:
        ict.ict_set_mantissa_bits(8)
    with pytest.raises(ict.IctError):
        ict.ict_set_mantissa_bits(9)
    assert ict.ict_get_mantissa_bits() == 8
