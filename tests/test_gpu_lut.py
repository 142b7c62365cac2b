"""GPU parity of the lookup-table nonlinearities ("Memory-Efficient Integer-Only Training
of Deep Neural Networks", Table 7: GELU through LUT_fwd / LUT_bwd; Table 8: the output
head through LUT_exp / LUT_log) against the oracle, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from integer_only_nn_02_b200.workloads import CE, E_ZERO
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


def status_ok(ict):
    code, raw = ict.ict_get_device_status()
    assert code == 0, (code, raw)


@pytest.mark.parametrize("rows,cols,G,erange", [(64, 768, 32, (-9, -5)), (130, 96, 16, (-30, 6)),
                                                (17, 64, 64, (-127, 127)), (300, 3072, 64, (-8, -4))])
def test_gelu_lut(ict, rows, cols, G, erange):
    rng = np.random.default_rng(rows + cols + G)
    H = rand_ce(rng, rows, cols, 1, G, elo=erange[0], ehi=erange[1], zero_groups=0.05)
    dY = rand_ce(rng, rows, cols, 1, G, elo=-16, ehi=-8, zero_groups=0.05)
    dH_, dY_ = ict.DevCE.from_host(H), ict.DevCE.from_host(dY)
    same(ict.gelu_lut_fwd(dH_).to_host(), oracle.gelu_lut_fwd(H), "gelu lut fwd")
    same(ict.gelu_lut_bwd(dH_, dY_).to_host(), oracle.gelu_lut_bwd(H, dY, 1, G), "gelu lut bwd")
    status_ok(ict)


@pytest.mark.parametrize("rows,classes,zg,dg,erange", [
    (256, 10, 10, 10, (-5, -2)),       # CIFAR-10 head, one group per row
    (256, 1000, 1000, 1000, (-7, -3)),  # ImageNet head
    (64, 100, 50, 25, (-9, 2)),        # two logit groups per row (aligned first), four gradient groups
    (33, 1000, 64, 200, (-30, 8)),     # exponents beyond the table rows on both sides
    (8, 3, 3, 3, (-4, -4)),
])
def test_softmax_ce(ict, rows, classes, zg, dg, erange):
    rng = np.random.default_rng(rows + classes + zg)
    Z = rand_ce(rng, rows, classes, 1, zg, elo=erange[0], ehi=erange[1], zero_groups=0.05)
    Z.mant[0] = 0                       # an all-zero row: uniform probabilities
    Z.exp[0] = E_ZERO
    hot = min(3, classes - 1)
    if rows > 2:
        Z.mant[1] = -127                # a confident row
        Z.mant[1, hot] = 127
        Z.exp[1] = max(erange[0], 0)
    tgt = rng.integers(0, classes, size=rows).astype(np.int32)
    tgt[1 % rows] = hot
    loss_ref, dZ_ref = oracle.softmax_ce(Z, tgt, 1, dg)
    loss, dZ = ict.softmax_ce(ict.DevCE.from_host(Z), torch.from_numpy(tgt), dg)
    assert np.array_equal(loss.cpu().numpy(), loss_ref), "loss"
    same(dZ.to_host(), dZ_ref, "dZ")
    status_ok(ict)
