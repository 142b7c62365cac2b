"""The allocation-free forward Product against the workspace entry point and the oracle.

ict_linear_fwd_noalloc serves callers that cannot give the library a device workspace
(host frameworks that reserve all device memory up front, statically budgeted
deployments, code that must not call cudaMalloc/cudaFree because those can block or
synchronise the device).  It keeps its scratch in one fixed array inside the library.
This file is collected last so that a run stopping at the first failure has already
run every other test; it passes alone in a fresh process and after the others.
"""
import numpy as np
import pytest

from integer_only_nn_02_b200.workloads import CE, clipped_gaussian, with_groups

pytestmark = pytest.mark.gpu


def _inputs(seed, M=1000, N=768, K=384):
    rng = np.random.default_rng(seed)
    # (1, 64) input groups: both operands need the alignment copy the scratch holds
    X = with_groups(clipped_gaussian(rng, (M, K), 24), 1, 64, lambda g: rng.integers(-9, -6, size=g))
    W = with_groups(clipped_gaussian(rng, (N, K), 24), 1, 64, lambda g: rng.integers(-10, -7, size=g))
    return X, W


def test_noalloc_matches_workspace_entry_twice():
    import oracle
    from integer_only_nn_02_b200 import ict

    for seed in (11, 12):  # two calls in a row share the scratch array
        X, W = _inputs(seed)
        dX, dW = ict.DevCE.from_host(X), ict.DevCE.from_host(W)
        ref = ict.linear_fwd(dX, dW, 64).to_host()
        Y = ict.DevCE.empty(X.rows, W.rows, 1, 64)
        assert ict.ict_linear_workspace(ict.OP_LINEAR_FWD, dX, dW, Y) > 0
        ict.ict_linear_fwd_noalloc(dX, dW, Y)
        got = Y.to_host()
        assert np.array_equal(got.mant, ref.mant) and np.array_equal(got.exp, ref.exp), seed
        # and, directly, against the CPU oracle
        want = oracle.linear_fwd(X, W, 1, 64)
        assert np.array_equal(got.mant, want.mant) and np.array_equal(got.exp, want.exp), seed
    code, raw = ict.ict_get_device_status()
    assert code == 0, (code, raw)


def test_noalloc_rejects_scratch_beyond_its_limit():
    from integer_only_nn_02_b200 import ict

    M, K = 20000, 1024  # aligned copy of X alone is 20 MB > 16 MiB
    X = CE(np.ones((M, K), np.int8), np.zeros((M, K // 64), np.int8), 1, 64)
    W = CE(np.ones((64, K), np.int8), np.zeros((64, 1), np.int8), 1, K)
    dX, dW = ict.DevCE.from_host(X), ict.DevCE.from_host(W)
    Y = ict.DevCE.empty(M, 64, 1, 64)
    assert ict.ict_linear_workspace(ict.OP_LINEAR_FWD, dX, dW, Y) > ict.NOALLOC_SCRATCH_BYTES
    with pytest.raises(ict.IctError) as ei:
        ict.ict_linear_fwd_noalloc(dX, dW, Y)
    assert ei.value.code == 4  # ICT_ERR_WORKSPACE
