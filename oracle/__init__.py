"""CPU oracle for the layer-streamed NF4 + LoRA training step.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg may import, call or execute anything in this package.
The CUDA library never calls it, and it never calls the CUDA library: the two share no
code, tables or constants.  Inputs come from the `synth` generator module.

Precision: float64 for all floating-point arithmetic, except where the quantised format
itself fixes a narrower type (NF4 codebook stored as float32, double-quantised absmax in
float32, dequantised weights rounded to bfloat16), which is part of what the format
defines.

Sources.  The method comes from five web pages about the open-source "Soup" trainer:
  * rug.gal radar "Soup ... layer streaming" (Spanish, Italian and French copies), lead and
    "En detalle" / "Nel dettaglio" / "En détail";
  * "Soup: afinar un modelo de 8.000 millones de parámetros en un portátil con 4 GB de
    gráfica" (guillermodelpino.com), sections "El streaming de capas, que es el truco de la
    casa", the soup.yaml example, "Preguntas frecuentes";
  * "Soup promete fine-tuning de modelo 8B em GPU de notebook com 4 GB" (imasters.com.br),
    sections "Como cabe um 8B em 4 GB", "Do SFT para os métodos de preferência" and "O que
    muda para quem constrói no Brasil".
The pages name NF4, LoRA, the Llama-3.1-8B decoder layer, SFT, DPO, KTO, ORPO, SimPO and a
merge command but print no formula; where they are silent each function states the textbook
definition it follows (QLoRA, LoRA, Llama, DPO, KTO, ORPO, SimPO and AdamW papers).

Modules: nf4 (codebook, quantise / dequantise, blob sizes), model (decoder layer, LoRA, SFT
and DPO losses, backward passes, AdamW, LoRA merge), pref (KTO, ORPO, SimPO).

Parity status per function: every function here is pinned by tests/test_oracle_*.py
(closed forms, library routines, finite differences, a published table).  The composed
training step's absolute loss on random weights has no printed value to compare with:
"parity unpinned" beyond the pins of its parts.
"""
from . import nf4, model, pref  # noqa: F401
