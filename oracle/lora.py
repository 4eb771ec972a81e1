"""LoRA linear forward and backward in fp64 (oracle).

Test infrastructure: only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may use this module.

The layer is ``Y = X W_hat^T + s (X A^T) B^T`` with ``W_hat`` the dequantized
frozen weight ``[d_out, d_in]``, ``A`` ``[r, d_in]``, ``B`` ``[d_out, r]`` and
``s = alpha / r`` ("FT-02: QLoRA -- Fine-Tuning with Quantization", section
"4. The LoRA mechanics the API wraps", the ``LoRALinear`` class; "QLoRA: NF4
storage, gradients and local integration", ``FrozenNF4LoRA.forward``).

For an upstream gradient ``G = dY`` the page "QLoRA: NF4 storage, gradients
and local integration" (the paragraph after the teaching program, section
"Exact CPU teaching quantizer and adapter gradient path") gives::

    dB = s G^T X A^T      dA = s B^T G^T X      dX = G W_hat + s G B A

and no gradient for the frozen ``W_hat``.  Below, ``U = X A^T`` and
``V = G B``, so ``dB = s G^T U`` and ``dA = s V^T X``.

Inputs are decoded to fp64 exactly (bf16 and fp32 values are fp64 values);
every product and sum is fp64 through numpy's matmul.  ``U`` and ``V`` are
used unrounded.
"""

from __future__ import annotations

import numpy as np

F64 = np.float64


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=F64)


def lora_forward(X, W_hat, A, B, s: float):
    """``(Y, U)`` with ``U = X A^T`` and ``Y = X W_hat^T + s U B^T``.

    "FT-02: QLoRA -- Fine-Tuning with Quantization", section "4. The LoRA
    mechanics the API wraps" (``LoRALinear.forward``); "QLoRA: NF4 storage,
    gradients and local integration", ``FrozenNF4LoRA.forward``.
    """
    X, W_hat, A, B = _f64(X), _f64(W_hat), _f64(A), _f64(B)
    U = X @ A.T
    Y = X @ W_hat.T + F64(s) * (U @ B.T)
    return Y, U


def lora_backward(X, dY, W_hat, A, B, s: float):
    """``(dX, dA, dB, V)`` for the upstream gradient ``dY`` of ``Y``.

    The gradient formulas of "QLoRA: NF4 storage, gradients and local
    integration", the paragraph after the teaching program (section "Exact
    CPU teaching quantizer and adapter gradient path"), with ``V = dY B``.
    """
    X, dY, W_hat, A, B = _f64(X), _f64(dY), _f64(W_hat), _f64(A), _f64(B)
    s = F64(s)
    U = X @ A.T
    V = dY @ B
    dX = dY @ W_hat + s * (V @ A)
    dA = s * (V.T @ X)
    dB = s * (dY.T @ U)
    return dX, dA, dB, V


def lora_forward_rows(rows, X, W_hat, A, B, s: float) -> np.ndarray:
    """Rows ``rows`` of ``Y`` only (each output row depends on its own input
    row): :func:`lora_forward` on those rows, the same passage."""
    Y, _ = lora_forward(_f64(X)[rows], W_hat, A, B, s)
    return Y


def lora_backward_rows(rows, dY, W_hat, A, B, s: float) -> np.ndarray:
    """Rows ``rows`` of ``dX`` only: ``dX[m] = dY[m] W_hat + s (dY[m] B) A``
    (the ``dX`` formula of :func:`lora_backward`, row by row)."""
    dYr, W_hat, A, B = _f64(dY)[rows], _f64(W_hat), _f64(A), _f64(B)
    return dYr @ W_hat + F64(s) * ((dYr @ B) @ A)


def lora_adapter_grads(X, dY, A, B, s: float):
    """``(dA, dB)`` alone: they need no ``W_hat`` (the ``dA`` and ``dB``
    formulas of :func:`lora_backward`, the same passage)."""
    X, dY, A, B = _f64(X), _f64(dY), _f64(A), _f64(B)
    s = F64(s)
    dA = s * ((dY @ B).T @ X)
    dB = s * (dY.T @ (X @ A.T))
    return dA, dB


def merge(W_hat, A, B, s: float) -> np.ndarray:
    """The merged weight ``W_hat + s B A`` in fp64.

    "FT-02: QLoRA -- Fine-Tuning with Quantization", section "4. The LoRA
    mechanics the API wraps" (the merge proof: one dense layer with weight
    ``W0 + (alpha/r) B A`` computes the two-branch output); "QLoRA: NF4
    storage, gradients and local integration", section "Merge changes the
    operator: test it explicitly" (merging into the dequantized ``Qhat(W)``
    matches the unmerged quantized layer in exact arithmetic; requantizing
    the result adds ``Qhat(M) - M``).  ``W_hat`` here is the fp32 dequantized
    weight (before any bf16 rounding).
    """
    W_hat, A, B = _f64(W_hat), _f64(A), _f64(B)
    return W_hat + F64(s) * (B @ A)
