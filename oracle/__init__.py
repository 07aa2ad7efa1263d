"""CPU oracle for layer-streamed LoRA fine-tuning: test infrastructure, not a product path.

Plain, slow and meant to be checked by eye: numpy in fp64 (weights and activations enter as the
fp32/bf16 values the GPU sees). Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import it. It shares no code with the CUDA library.

Sources, cited by the short names below (section or paragraph of each page):

* [5ID]   "Layer streaming fine-tuning for 8B model on 4GB GPU" (5id.vn news post).
* [TKN]   "Soup: Fine-Tuning an 8B Model on a 4 GB Laptop GPU, One Layer at a Time" (toknow.ai).
* [LACH]  Tutorial "Fine-tune Llama 3.1 8B on a 4GB GPU with Soup" (lachieslifestyle.com).
* [CODE]  "Fine-Tuning an 8B Parameter Model on a 4 GB Laptop GPU" (codeinktechnologies.com).
* [TESS]  "Soup CLI fine-tunes Llama-3.1-8B on a 4 GB laptop GPU, and that changes who owns AI"
          (thetesserapress.com).
* [QLORA] Dettmers et al., "QLoRA: Efficient Finetuning of Quantized LLMs" (2023), which [CODE]
          names as the origin of NF4 and double quantisation.

The pages print no formulas; where a step is the plainest reading rather than the pages' text,
the docstring says "reading".
"""
from . import nf4, model  # noqa: F401
