"""Dry run of bench.py's 32-layer stack measurement on the CPU (2 layers, 16 tokens).

The library calls are replaced by fakes that check every operand's shape and
stamp their outputs with a code for (layer, projection); each fake then checks
that its inputs carry the codes of the producers the chain rule names:
q = Q(h), k = K(h), v = V(h), a = O(q), g = G(a), u = U(a), h' = D(g + u), and
backward dh = dX_q + dX_k + dX_v, da = dX_g + dX_u, each projection's saved U.
This checks the wiring of the timed chain; the kernels themselves are covered
by the GPU parity tests.
"""

import pytest
import torch

import bench
from bit_nf4_quantized_blk_b200 import binding, workloads

LAYERS, M = 2, 16
Q, K_, V, O, G, UP, D = range(7)


def _code(layer, t):
    return float(layer * 8 + t + 1)  # small integers: exact in bf16, and so are their sums


@pytest.fixture
def fakes(monkeypatch):
    from bit_nf4_quantized_blk_b200 import build

    build.build()
    projs = workloads.LAYER7B
    proj_of = {}
    calls = []

    def which(w):
        """(layer, t) of a weight from the order the stack creates them in."""
        return proj_of[id(w)]

    def quantize_batched(Ws, outs, ws, d_status=None, stream=None):
        assert len(Ws) == len(outs) == 7 * LAYERS
        for i, (W, o) in enumerate(zip(Ws, outs)):
            assert W.dtype == torch.float32 and tuple(W.shape) == (o.rows, o.cols)
            assert (o.rows, o.cols) == (projs[i % 7].n, projs[i % 7].k)
            proj_of[id(o)] = (i // 7, i % 7)
        calls.append("quantize")

    def fwd(w, X, A, B, r, s, Y, U_out, ws, stream=None):
        layer, t = which(w)
        assert X.shape == (M, w.cols) and Y.shape == (M, w.rows) and U_out.shape == (M, r)
        assert A.shape == (r, w.cols) and B.shape == (w.rows, r)
        want = {O: _code(layer, Q), G: _code(layer, O), UP: _code(layer, O),
                D: _code(layer, G) + _code(layer, UP)}.get(t)
        if t in (Q, K_, V) and layer > 0:
            want = _code(layer - 1, D)
        if want is not None:
            assert X[0, 0].item() == want, f"fwd layer {layer} proj {t}: input {X[0, 0].item()} != {want}"
        Y.fill_(_code(layer, t))
        U_out.fill_(_code(layer, t))
        calls.append(("fwd", layer, t))

    def bwd(w, X, dY, A, B, r, s, dX, accumulate, dA, dB, ws, U=None, stream=None):
        layer, t = which(w)
        assert X.shape == (M, w.cols) and dY.shape == (M, w.rows) and dX.shape == (M, w.cols)
        assert dA.shape == (r, w.cols) and dB.shape == (w.rows, r) and U.shape == (M, r)
        assert U[0, 0].item() == _code(layer, t), "the backward must get its projection's saved U"
        x_want = {O: _code(layer, Q), G: _code(layer, O), UP: _code(layer, O),
                  D: _code(layer, G) + _code(layer, UP)}.get(t)
        if t in (Q, K_, V) and layer > 0:
            x_want = _code(layer - 1, D)
        if x_want is not None:
            assert X[0, 0].item() == x_want, f"bwd layer {layer} proj {t}: input"
        g = -_code(layer, t)  # gradient codes are negative, forward codes positive
        dy_want = {G: -_code(layer, D), UP: -_code(layer, D), O: -_code(layer, G) - _code(layer, UP),
                   Q: -_code(layer, O)}.get(t)
        if t == D and layer < LAYERS - 1:
            dy_want = -_code(layer + 1, Q) - _code(layer + 1, K_) - _code(layer + 1, V)
        if dy_want is not None:
            assert dY[0, 0].item() == dy_want, f"bwd layer {layer} proj {t}: upstream gradient"
        expected_acc = 1 if t in (UP, K_, V) else 0
        assert accumulate == expected_acc, f"layer {layer} proj {t}: accumulate"
        if accumulate:
            dX.add_(g)
        else:
            dX.fill_(g)
        calls.append(("bwd", layer, t))

    def timed(fn, steps, warmup, world, window=None):
        fn()
        return 1.0

    monkeypatch.setattr(binding, "_check_placement", lambda t, name: None)
    monkeypatch.setattr(binding, "qlora_nf4_quantize_batched", quantize_batched)
    monkeypatch.setattr(binding, "qlora_linear_fwd", fwd)
    monkeypatch.setattr(binding, "qlora_linear_bwd", bwd)
    monkeypatch.setattr(binding, "qlora_workspace_reset", lambda ws, stream=None: None)
    monkeypatch.setattr(binding, "qlora_workspace_status", lambda ws, stream=None: 0)
    monkeypatch.setattr(bench, "timed", timed)
    return calls


def test_stack_chain_wiring(fakes):
    res = bench.bench_stack(steps=1, warmup=0, layers=LAYERS, M=M, device="cpu")
    fwd = [c for c in fakes if c[0] == "fwd"]
    bwd = [c for c in fakes if c[0] == "bwd"]
    assert fakes[0] == "quantize"
    assert fwd == [("fwd", layer, t) for layer in range(LAYERS) for t in (Q, K_, V, O, G, UP, D)]
    assert bwd == [("bwd", layer, t) for layer in reversed(range(LAYERS)) for t in (D, G, UP, O, Q, K_, V)]
    assert res["fwd_bwd"]["flops"] == bench.step_flops(M) * LAYERS
    assert res["quantize"]["weights"] == sum(p.n * p.k for p in workloads.LAYER7B) * LAYERS
