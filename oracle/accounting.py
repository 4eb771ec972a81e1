"""Storage and parameter accounting (oracle).

Test infrastructure: only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may use this module.

* Bits per quantized weight: 4 bits of code plus the amortised scales.
  Without double quantization one fp32 scale per 64 weights (4.5 bits); with
  it one 8-bit code per 64 weights and one fp32 second-level scale per 256
  codes (4.126953125 bits).  "QLoRA: NF4 storage, gradients and local
  integration", section "Double quantization: correct the scale arithmetic",
  and ``bits_per_weight`` in the teaching program; "QLoRA Deep Dive: 4-bit
  NormalFloat & Double Quantization Internals", section "Memory Savings
  Analysis".
* Stored bytes of one tensor in this library's layout: packed codes, int8
  scale codes, fp32 second-level scales and the fp32 mean offset (the stored
  "scale offset" of the same section).
* LoRA parameter counts: ``r (d_in + d_out)`` per adapted projection ("QLoRA:
  NF4 storage ...", section "Memory accounting before optimization";
  "FT-02: QLoRA -- Fine-Tuning with Quantization", section "4. The LoRA
  mechanics the API wraps", rank x alpha grid).
"""

from __future__ import annotations


def bits_per_weight(double_quant: bool, block: int = 64, dq_block: int = 256) -> float:
    """Amortised bits per quantized weight, ignoring tails and the mean offset."""
    if double_quant:
        return 4 + 8 / block + 32 / (block * dq_block)
    return 4 + 32 / block


def stored_bytes(n: int, block: int = 64, dq_block: int = 256) -> int:
    """Bytes of the packed state of one n-weight tensor (n a multiple of 2*block)."""
    n_blocks = -(-n // block)
    n_chunks = -(-n_blocks // dq_block)
    return n // 2 + n_blocks + 4 * n_chunks + 4


def lora_params(r: int, shapes) -> int:
    """Adapter parameters for projections of shapes ``(d_out, d_in)``."""
    return sum(r * (d_out + d_in) for d_out, d_in in shapes)
