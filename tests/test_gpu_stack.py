"""GPU parity for the 32-layer chained stack of the 7B layer's projections.

Per layer (no attention or norm): q = Q(h), k = K(h), v = V(h), a = O(q),
g = G(a), u = U(a), h' = D(g + u).  k and v are leaves that receive seeded
upstream gradients, the last h' receives a seeded gradient, and the backward
is the chain rule through the same graph (dh = dX_q + dX_k + dX_v, da = dX_g +
dX_u, formed with the accumulate flag of the backward).  All 224 weights (6.98 G
fp32 values with 0.1% x10 outliers) are quantized with double quantization in
batched calls.  Parity is teacher-forced: for sampled layers, every projection
is checked against the oracle on the exact activations and upstream gradients
the GPU used (64 sampled rows of Y and dX, all of dA and dB).
"""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding, workloads
from gpu_helpers import assert_close, assert_state_equal, bf16_to_np, require_gpu
from oracle import lora, nf4

pytestmark = pytest.mark.gpu

M = 8192
R = 16
S = 32.0 / 16
LAYERS = 32
CHECK_LAYERS = (0, 31)
Q, K_, V, O, G, U, D = range(7)


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def test_stack_32_layers_chained():
    require_gpu()
    torch.cuda.synchronize()
    # ---- quantize every layer (batched per layer), keep the check layers' fp32 weights
    qweights, adapters, w_cpu = [], [], {}
    for layer in range(LAYERS):
        Ws, As, Bs = [], [], []
        for t in range(7):
            W, A, B = workloads.stack_projection(layer, t, device="cuda")
            Ws.append(W)
            As.append(A)
            Bs.append(B)
        outs = [binding.NF4Weight.empty(p.n, p.k) for p in workloads.LAYER7B]
        qws = torch.empty(binding.qlora_nf4_quantize_batched_ws_bytes(outs), dtype=torch.uint8, device="cuda")
        binding.qlora_nf4_quantize_batched(Ws, outs, qws)
        if layer in CHECK_LAYERS:
            w_cpu[layer] = [w.cpu() for w in Ws]
        del Ws, qws
        qweights.append(outs)
        adapters.append((As, Bs))
    torch.cuda.synchronize()

    ws = torch.empty(max(binding.qlora_linear_ws_bytes(M, p.n, p.k, R) for p in workloads.LAYER7B),
                     dtype=torch.uint8, device="cuda")
    binding.qlora_workspace_reset(ws)

    def fwd(layer, t, x):
        p = workloads.LAYER7B[t]
        y = torch.empty((M, p.n), dtype=torch.bfloat16, device="cuda")
        u = torch.empty((M, R), dtype=torch.float32, device="cuda")
        A, B = adapters[layer][0][t], adapters[layer][1][t]
        binding.qlora_linear_fwd(qweights[layer][t], x, A, B, R, S, y, u, ws)
        return y, u

    # ---- forward through the stack, saving what the backward needs
    h = workloads.stack_input(M, device="cuda")
    saved = []
    for layer in range(LAYERS):
        q, uq = fwd(layer, Q, h)
        k, uk = fwd(layer, K_, h)
        v, uv = fwd(layer, V, h)
        a, ua = fwd(layer, O, q)
        g, ug = fwd(layer, G, a)
        u, uu = fwd(layer, U, a)
        gu = g + u  # model plumbing between projections, outside the method
        h_next, ud = fwd(layer, D, gu)
        saved.append(dict(h=h, q=q, a=a, gu=gu, uq=uq, uk=uk, uv=uv, ua=ua, ug=ug, uu=uu, ud=ud, out=h_next))
        h = h_next
    assert torch.isfinite(h.float()).all(), "stack output overflowed"

    # ---- backward
    checks = {}

    def bwd(layer, t, x, dy, u, dx, accumulate):
        p = workloads.LAYER7B[t]
        A, B = adapters[layer][0][t], adapters[layer][1][t]
        dA = torch.empty((R, p.k), dtype=torch.float32, device="cuda")
        dB = torch.empty((p.n, R), dtype=torch.float32, device="cuda")
        dx_before = dx.clone() if (accumulate and layer in CHECK_LAYERS) else None
        binding.qlora_linear_bwd(qweights[layer][t], x, dy, A, B, R, S, dx, accumulate, dA, dB, ws, U=u)
        if layer in CHECK_LAYERS:
            checks[(layer, t)] = dict(x=x, dy=dy, dA=dA, dB=dB, dx=dx.clone(), dx_before=dx_before)

    dh = workloads.stack_leaf_grad(LAYERS - 1, "top", M, device="cuda")
    for layer in reversed(range(LAYERS)):
        sv = saved[layer]
        dgu = torch.empty((M, 14336), dtype=torch.bfloat16, device="cuda")
        bwd(layer, D, sv["gu"], dh, sv["ud"], dgu, 0)
        da = torch.empty((M, 4096), dtype=torch.bfloat16, device="cuda")
        bwd(layer, G, sv["a"], dgu, sv["ug"], da, 0)
        bwd(layer, U, sv["a"], dgu, sv["uu"], da, 1)
        dq = torch.empty((M, 4096), dtype=torch.bfloat16, device="cuda")
        bwd(layer, O, sv["q"], da, sv["ua"], dq, 0)
        dh_prev = torch.empty((M, 4096), dtype=torch.bfloat16, device="cuda")
        bwd(layer, Q, sv["h"], dq, sv["uq"], dh_prev, 0)
        bwd(layer, K_, sv["h"], workloads.stack_leaf_grad(layer, "k", M, device="cuda"), sv["uk"], dh_prev, 1)
        bwd(layer, V, sv["h"], workloads.stack_leaf_grad(layer, "v", M, device="cuda"), sv["uv"], dh_prev, 1)
        dh = dh_prev
    assert binding.qlora_workspace_status(ws) == 0
    assert torch.isfinite(dh.float()).all(), "stack gradient overflowed"

    # ---- teacher-forced parity on the check layers
    rng = np.random.default_rng(5)
    for layer in CHECK_LAYERS:
        for t in range(7):
            c = checks[(layer, t)]
            st = nf4.quantize_weight(w_cpu[layer][t].numpy())
            assert_state_equal(qweights[layer][t], st, f"layer {layer} proj {t}")
            Wh = nf4.bf16_bits_to_f32(nf4.dequantize_weight(st, "bf16")).astype(np.float64)
            A, B = _np(adapters[layer][0][t]), _np(adapters[layer][1][t])
            rows = rng.choice(M, 64, replace=False)
            X, dY = _np(c["x"]), _np(c["dy"])
            y_gpu = {Q: "q", O: "a", D: "out"}.get(t)
            if y_gpu is not None:
                assert_close(bf16_to_np(saved[layer][y_gpu])[rows], lora.lora_forward_rows(rows, X, Wh, A, B, S),
                             f"Y layer {layer} proj {t}")
            dx_ref = lora.lora_backward_rows(rows, dY, Wh, A, B, S)
            if c["dx_before"] is not None:
                dx_ref = dx_ref + _np(c["dx_before"])[rows]
            assert_close(bf16_to_np(c["dx"])[rows], dx_ref, f"dX layer {layer} proj {t}")
            dA_ref, dB_ref = lora.lora_adapter_grads(X, dY, A, B, S)
            assert_close(_np(c["dA"]), dA_ref, f"dA layer {layer} proj {t}")
            assert_close(_np(c["dB"]), dB_ref, f"dB layer {layer} proj {t}")
