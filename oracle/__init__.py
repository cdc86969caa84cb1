"""CPU oracle for the NF4-LoRA hot path -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct numpy code that states what the method computes,
step by step, in the notation of the source pages. It exists so that the CUDA
path can be checked against something written independently of it:

* it shares no code, header, table or constant generator with
  ``quantized_lora_fine_b200`` (the NF4 table here is built with mpmath at 50
  digits; the CUDA side carries its own table);
* only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
  ``bench.py`` may import it; the product path never does.

Source pages cited in the docstrings (by title and section):

* [QLoRA-blog]  "QLoRA: How to fine-tune large language models with less memory"
  (sections "The algebra", "1. NormalFloat", "2. Double quantization",
  "One training step", "A worked memory budget for 65 billion weights").
* [LoRA-blog]   "LoRA: Fine-tuning a model by learning a small update"
  (scaled eq. (3), "How much smaller is the trainable part?",
  "Serving models and switching tasks").
* [AQLoRA]      "AQLoRA: A Zero-Search Recipe for Fast Quantized LoRA
  Fine-Tuning" summary page (sections 3.1-3.3, 7).
* [Lesson-17]   "Lesson 17. What QLoRA Actually Costs" (warm-up questions).
* [QLoRA-notes] "QLoRA: Quantized LoRA - Complete Comparison with LoRA"
  (BitsAndBytesConfig / LoraConfig listings).

Functions whose results have no external pin are marked "parity unpinned" in
their docstrings. Today that is only the exact bit values of the NF4 code
table against third-party NF4 tables (the pages do not print the 16 values);
the table itself is pinned by its defining quantile property.
"""
from . import nf4, lora, layer_error, storage  # noqa: F401
