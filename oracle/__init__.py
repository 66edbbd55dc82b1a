"""CPU oracle for layer-streamed NF4 QLoRA training.  TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import anything from this
package.  The product path (the C-ABI library and its Python binding) never
does, and it shares no code with this package: the oracle rebuilds every
table, quantiser and layer step from the pages and the published mathematics.

Precision: quantisation and dequantisation follow the fp32 arithmetic that
the pages fix (fp32 NF4 and nested code tables, fp32 absmax, nested absmax
and offset), so bytes and dequantised weights are exact results.  Everything
else (linear, LoRA, RMSNorm, RoPE, attention, SiLU MLP, cross-entropy, AdamW)
is computed in float64; where the path stores a tensor in bf16 ("bf16
compute" in the workloads), the oracle rounds the float64 value to bf16 at the
same point.  ``rnd=False`` turns those roundings off, giving a pure float64
function that finite differences can check.

Modules
  codebooks  NF4 (16 fp32) and nested 8-bit (256 fp32) code tables
  quant      blockwise NF4 + double quantisation, dequantisation, byte counts
  bf16       round-to-nearest-even bf16 helpers on numpy arrays
  layer      decoder-layer forward and hand-derived backward
  model      embedding, stack, cross-entropy, AdamW, one training step
  account    FLOP and byte accounting used by the throughput metric

Parity unpinned: which exact NF4 constants and which 8-bit nested table the
pages' system used.  The pages print neither; the tables here follow the
published constructions named in ``codebooks`` and are pinned to those
definitions only.
"""
