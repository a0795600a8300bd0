"""CPU oracle for the QLoRA linear layer — TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct numpy (float64 unless a step is fixed to
float32 for bit-exactness).  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it.  It shares no code with the
CUDA library and never imports it.

Sources (cited by page title and section throughout):
  [P1] "LoRA and QLoRA fine-tuning: mechanics, and when not to fine-tune"
  [P2] "Fine-Tuning on a Budget: LoRA and QLoRA"
  [P3] "LoRA vs QLoRA: Fine-Tuning LLMs Guide"
  [P4] "LoRA and QLoRA Explained: Efficient Techniques for Fine-Tuning AI Models"
  [P5] "LoRA vs QLoRA: Parameter-Efficient Fine-Tuning Explained"

Parity status of each function is stated in its docstring.  The single
function whose numbers the pages do not fix is the absolute value of the NF4
levels (the outermost quantile probability is not printed): its structure is
pinned, its digits are "parity unpinned" beyond that structure.
"""
from . import nf4, lora, adam  # noqa: F401
