"""A training step captured as one CUDA graph (ict.StepGraph) gives, replay after
replay, the same bits as the oracle running the same steps one after the other: a
ViT-Ti-shaped MLP block (fc1, integer GELU, fc2, both backward directions, SGD with
momentum on both weights) on a ragged token count, two chained steps."""
import numpy as np
import pytest

import oracle
from integer_only_nn_02_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def same(got, ref, what):
    assert np.array_equal(got.mant, ref.mant), f"{what}: mantissas differ"
    assert np.array_equal(got.exp, ref.exp), f"{what}: exponents differ"


def oracle_step(X, W1, W2, dY2, V1, V2, G, mom, lr):
    H = oracle.linear_fwd(X, W1, 1, G)
    Gl = oracle.gelu_fwd(H)
    Y = oracle.linear_fwd(Gl, W2, 1, G)
    dG = oracle.linear_bwd_data(dY2, W2, 1, G)
    dW2 = oracle.linear_bwd_weight(dY2, Gl, 1, W2.cols)
    dH = oracle.gelu_bwd(H, dG, 1, G)
    dX = oracle.linear_bwd_data(dH, W1, 1, G)
    dW1 = oracle.linear_bwd_weight(dH, X, 1, W1.cols)
    W1n, V1n = oracle.sgd_step(W1, V1, dW1, mom, lr)
    W2n, V2n = oracle.sgd_step(W2, V2, dW2, mom, lr)
    return dict(Y=Y, dX=dX, W1=W1n, V1=V1n, W2=W2n, V2=V2n)


@pytest.mark.parametrize("tokens", [300, 1000])
def test_mlp_step_graph_two_replays(tokens):
    import torch

    from integer_only_nn_02_b200 import ict

    cfg = wl.vit_ti_mlp(seed=11, tokens=tokens)
    G, mom, lr = cfg["out_group"], cfg["sgd"]["mom"], cfg["sgd"]["lr"]
    E = ict.DevCE
    X, W1, W2, dY2, V1, V2 = (E.from_host(cfg[k]) for k in ("X", "W1", "W2", "dY2", "V1", "V2"))
    D, Hd = X.cols, W1.rows
    H, Gl, dG, dH = (E.empty(tokens, Hd, 1, G) for _ in range(4))
    Y, dX = E.empty(tokens, D, 1, G), E.empty(tokens, D, 1, G)
    dW2, dW1 = E.empty(D, Hd, 1, Hd), E.empty(Hd, D, 1, D)
    w = ict.ict_linear_workspace
    ws = torch.empty(max(256, w(0, X, W1, H), w(0, Gl, W2, Y), w(1, dY2, W2, dG), w(2, dY2, Gl, dW2),
                         w(1, dH, W1, dX), w(2, dH, X, dW1)), dtype=torch.uint8, device="cuda")

    def step():
        ict.ict_linear_fwd(X, W1, H, ws)
        ict.ict_gelu_fwd(H, Gl)
        ict.ict_linear_fwd(Gl, W2, Y, ws)
        ict.ict_linear_bwd_data(dY2, W2, dG, ws)
        ict.ict_linear_bwd_weight(dY2, Gl, dW2, ws)
        ict.ict_gelu_bwd(H, dG, dH)
        ict.ict_linear_bwd_data(dH, W1, dX, ws)
        ict.ict_linear_bwd_weight(dH, X, dW1, ws)
        ict.ict_sgd_momentum_step(W1, V1, dW1, mom, lr)
        ict.ict_sgd_momentum_step(W2, V2, dW2, mom, lr)

    graph = ict.StepGraph(step, warmup=1)  # the warm-up is step 1
    assert graph.launches > 0
    graph.replay()  # step 2
    torch.cuda.synchronize()
    code, raw = ict.ict_get_device_status()
    assert code == 0, (code, raw)

    s1 = oracle_step(cfg["X"], cfg["W1"], cfg["W2"], cfg["dY2"], cfg["V1"], cfg["V2"], G, mom, lr)
    s2 = oracle_step(cfg["X"], s1["W1"], s1["W2"], cfg["dY2"], s1["V1"], s1["V2"], G, mom, lr)
    for name, got in (("Y", Y), ("dX", dX), ("W1", W1), ("V1", V1), ("W2", W2), ("V2", V2)):
        same(got.to_host(), s2[name], f"step 2 {name}")
