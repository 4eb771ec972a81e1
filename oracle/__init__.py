"""Plain CPU oracle for the QLoRA NF4 linear path (test infrastructure).

This package is test infrastructure, not product code.  Only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it.  It shares no code, table or helper with the CUDA library in
``bit_nf4_quantized_blk_b200``; the two only meet through the seeded input
generators, which hold none of the method's arithmetic.

What it computes, and where each step comes from (page titles, sections):

* ``oracle.nf4``   -- the 16-level NF4 codebook, blockwise absmax quantization
  to 4-bit codes packed two per byte, double quantization of the block scales
  to 8 bits with a per-chunk fp32 second-level scale and a per-tensor mean
  offset, and the dequantizer.  Sources: "QLoRA: NF4 storage, gradients and
  local integration" (sections "NF4: nonuniform reconstruction levels",
  "Double quantization: correct the scale arithmetic", "Exact CPU teaching
  quantizer and adapter gradient path"); "QLoRA Deep Dive: 4-bit NormalFloat &
  Double Quantization Internals" (sections "The Quantization Process in
  QLoRA", "2. Squeezing More Memory: Double Quantization (DQ)").
* ``oracle.lora``  -- the LoRA linear forward and its gradients in fp64.
  Sources: "QLoRA: NF4 storage, gradients and local integration" (the
  gradient paragraph closing "Exact CPU teaching quantizer and adapter
  gradient path"); "FT-02: QLoRA -- Fine-Tuning with Quantization"
  (section "4. The LoRA mechanics the API wraps").
* ``oracle.accounting`` -- bits per weight and storage bytes of the packed
  state, adapter parameter counts.

Every function is written for a reader to check against the pages by eye:
no blocking, fusion or reordering beyond what the definition states.
Readings of points the pages leave open are stated in the docstrings.
"""
