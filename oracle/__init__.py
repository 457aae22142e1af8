"""Plain CPU oracle for the QLoRA NF4 frozen linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, table or constant generator with the CUDA library; the two meet only
through the seeded input generators in ``bit_nf4_quantized_28_b200.workloads``
(which hold none of the method's arithmetic).

Every function follows one passage of the source pages, cited in its
docstring by page title and section:

* [QLoRA glossary] -- Ultralytics glossary page "QLoRA" (Italian):
  "Come funziona QLoRA" (NF4 levels, blocks of 64, double quantization in
  blocks of 256, forward/backward through the dequantized weights), the NF4
  snippet that builds the levels and prints the NF4/INT4 errors, and
  "Compromessi" (dequantization on every pass).
* [LoRA y QLoRA en Profundidad] -- skyvanguard lesson 5: "Cómo Funciona LoRA"
  (delta_W = B @ A, A is r x d_in, B is d_out x r), "Alpha (lora_alpha)"
  (update scaled by alpha/r), "Inicialización" (B starts at zero),
  "Doble Cuantización", "Dropout (lora_dropout)" (zeroes random elements of
  the LoRA layers' input; 0.05 in the lesson's config), "Optimizadores
  Paginados" (paged_adamw_8bit: Adam with 8-bit states), and the QLoRA config
  (compute dtype bfloat16).
* [Módulo 4: QLoRA] -- course module 4: 4.2 (4 bits = 0.5 byte per weight),
  4.3 b) (the scale constants are quantized again, to 8 bits), 4.4 (only the
  LoRA matrices train; weights are dequantized to BF16 for the passes).

Modules: ``nf4`` (levels, encode, double quantization, dequantization,
packing, bf16 rounding, the worked-example errors), ``linear`` (the forward
and backward of the frozen linear with its LoRA path, in fp64), ``merge``
(the adapter folded into the dequantized weight), ``dropout`` (LoRA
dropout: the Philox4x32-10 keep mask and the layer with it, in fp64) and
``adamw8`` (the AdamW step on A and B with 8-bit states: the textbook
AdamW in fp64, the states stored as E4M3 codes with block scales).
"""

from . import nf4, linear, merge, dropout, adamw8  # noqa: F401
