"""CPU oracle for hybrid-precision attention — TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously-correct NumPy restatement of what the hybrid-precision
attention hot path computes (HyQuant: Hybrid-Precision Quantization for LLM
Attention).  It exists to check the CUDA library, never to stand in for it:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import it.  It shares no code
with the CUDA path; both take their inputs from
``hybrid_precision_attention_b200.synth``.

Precision: the K4V4 pack is evaluated in float32 exactly as its definition
states (bit-exact target); everything else (dequantised values, softmax,
column mass, attention outputs) is float64.

Modules
  formats    K4V4 pack / dequant, OCP FP8 e4m3 rounding, per-block FP8 scaling
  select     column-mass vertical-line scores and the stable top-k
  attention  decode attention over a hybrid cache, hybrid causal prefill
  hybrid     the hybrid KV-cache state machine (prefix init, decode steps,
             reselection every 64 tokens, staging -> hybrid merge)
"""
from . import formats, select, attention, hybrid  # noqa: F401
