"""GPU parity of the training step on the page "kronecker-layer-benchmark", section "Setup".

The network is the 3-layer MLP 1024 -> 1024 -> 1024 -> 10 with ReLU: two KronLinear layers
(m = 32, r = 4) and a dense head, with cross-entropy plus lambda * sum|S|. The parameter
gradients that autograd collects through the library's kernels are compared with an fp64
chain rule on the host:
- the Kronecker layers' forward and backward come from the oracle;
- ReLU, the dense head, the softmax cross-entropy and the subgradient sign(S) of the penalty
  are written out in numpy.

Each ReLU mask is a decision that floating point makes. Both sides take it in the GPU's
precision: the host chain rule applies the masks of the GPU's own pre-activations (a TF32
pre-activation within rounding of zero may fall on the other side of it in fp64). The tolerance
is the layer's, widened for two layers in series: 1e-4 exact FP32, 1e-2 TF32.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import rel_err, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "tf32": 1e-2}


@pytest.mark.parametrize("fused", [False, True], ids=["autograd_l1", "fused_l1"])
@pytest.mark.parametrize("path", ["f32", "tf32"])
def test_mlp_gradients_match_oracle_chain_rule(path, fused):
    """fused: the penalty's gradient comes from the layers' backward (dS epilogue)."""
    from kronecker_factored_structured_b200.train_step import KronMLP
    torch.manual_seed(11)
    lam = 1e-3
    model = KronMLP(1024, 10, block=32, rank=4, path=path, fused_l1=lam if fused else None)
    with torch.no_grad():   # non-trivial S (zeros included) and biases
        for l in (model.l1, model.l2):
            l.S.copy_(torch.randn_like(l.S))
            l.S[torch.rand_like(l.S) < 0.25] = 0.0
            l.bias.copy_(0.1 * torch.randn_like(l.bias))
    N = 64
    g = torch.Generator().manual_seed(5)
    x = torch.randn(N, 1024, generator=g)
    labels = torch.randint(0, 10, (N,), generator=g)
    xd, ld = x.cuda(), labels.cuda()
    loss = torch.nn.functional.cross_entropy(model(xd).float(), ld) + lam * model.penalty()
    loss.backward()
    torch.cuda.synchronize()

    with torch.no_grad():   # the GPU's pre-activations (same deterministic kernels)
        z1g = model.l1(xd)
        z2g = model.l2(torch.relu(z1g))
    m1, m2 = to_np(z1g) > 0, to_np(z2g) > 0
    P = {n: to_np(p) for n, p in model.named_parameters()}
    xn = x.double().numpy()
    # forward, fp64, with the GPU's ReLU masks
    z1 = oracle.forward(xn, P["l1.S"], P["l1.A"], P["l1.B"], P["l1.bias"])
    h1 = z1 * m1
    z2 = oracle.forward(h1, P["l2.S"], P["l2.A"], P["l2.B"], P["l2.bias"])
    h2 = z2 * m2
    logits = h2 @ P["head.weight"].T + P["head.bias"]
    # softmax cross-entropy (mean over rows)
    e = np.exp(logits - logits.max(axis=1, keepdims=True))
    prob = e / e.sum(axis=1, keepdims=True)
    onehot = np.eye(10)[labels.numpy()]
    dlogits = (prob - onehot) / N
    ref = {"head.weight": dlogits.T @ h2, "head.bias": dlogits.sum(axis=0)}
    dz2 = (dlogits @ P["head.weight"]) * m2
    g2 = oracle.backward(h1, P["l2.S"], P["l2.A"], P["l2.B"], dz2)
    dz1 = g2["dX"] * m1
    g1 = oracle.backward(xn, P["l1.S"], P["l1.A"], P["l1.B"], dz1)
    for name, gg in (("l1", g1), ("l2", g2)):
        ref[f"{name}.S"] = gg["dS"] + lam * np.sign(P[f"{name}.S"])
        ref[f"{name}.A"] = gg["dA"]
        ref[f"{name}.B"] = gg["dB"]
        ref[f"{name}.bias"] = gg["dbias"]
    errs = {n: rel_err(to_np(p.grad), ref[n]) for n, p in model.named_parameters()}
    bad = {n: e for n, e in errs.items() if not e <= TOL[path]}
    assert not bad, f"{path}: gradient errors above {TOL[path]}: {bad} (all: {errs})"
    # the first layer's input needs no gradient: dX of layer 1 is never requested
    assert not xd.requires_grad


def test_train_step_benchmark_runs():
    from kronecker_factored_structured_b200.train_step import KronMLP, time_model
    model = KronMLP(1024, 10, block=32, rank=4, path="tf32")
    r = time_model(model, 256, 1024, 10, 1e-4, warmup=2, steps=3, dtype=torch.float32)
    assert np.isfinite(r["final_loss"]) and r["ms_per_step"] > 0 and r["peak_mem_mb"] > 0


def test_train_step_cuda_graph_replay_matches_eager():
    """The whole step captured in a CUDA graph (library kernels included: the cooperative
    parameter-gradient launch and its barrier reset are graph nodes) gives the eager step's
    parameters after the same number of steps."""
    from kronecker_factored_structured_b200.train_step import KronMLP, time_model
    out = {}
    for graph in (False, True):
        torch.manual_seed(3)
        model = KronMLP(1024, 10, block=32, rank=4, path="tf32")
        # 8 steps each: eager 6 + 2; graph 3 eager warm-up steps before the capture, 3 + 2 replays
        time_model(model, 256, 1024, 10, 1e-4, warmup=3 if graph else 6, steps=2,
                   dtype=torch.float32, graph=graph, capturable=True)
        torch.cuda.synchronize()
        out[graph] = {n: to_np(p) for n, p in model.named_parameters()}
    for n in out[False]:
        assert rel_err(out[True][n], out[False][n]) <= 1e-5, n
