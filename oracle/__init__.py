"""Plain, slow, fp64 CPU oracle for the QLoRA NF4 projection and gated MLP.

TEST INFRASTRUCTURE ONLY.  (``oracle/c/`` restates the tiny configuration in
plain C loops; ``oracle/c_oracle.py`` binds it.)  Nothing in the product path (the ``libqlora``
shared library and its Python binding) may import, call or link this package.
Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` use it.  It shares no code with the CUDA path: its bf16
rounding, NF4 codebook, quantiser, dequantiser, LoRA algebra and activation
derivatives are written here from the pages, independently.

Sources (web pages on Unsloth's QLoRA kernels; cited by title and section):

* [Mistral blog]  "用 Unsloth 微调 Mistral，速度提升 14 倍" (chapter heading
  "Unsloth 更新：支持 Mistral 及多项性能提升"): the benchmark configuration
  block (QLoRA nf4 layers, rank 16, alpha 16, dropout 0), the per-optimisation
  table "逐项性能拆解", its items "1. 减少数据类型提升", "2. Bitsandbytes
  bfloat16" and "10、11. 手动 Autograd" (the chained-matmul bracket order).
* [Gemma blog]  "使用 Unsloth 微调 Gemma：速度提升 2.4 倍，显存占用降低 58%",
  section "GeGLU 与 Swiglu 激活函数".
* [Show HN]  "Show HN: 80% faster, 50% less memory, 0% loss of accuracy Llama
  finetuning": highlights 1 (hand-derived backprop) and 4 (exact, no
  approximation); the thread links the QLoRA paper (arXiv 2305.14314) for the
  NormalFloat format.
* [Reddit talk]  "探索让 LLM 训练加速的神奇技巧" (r/LocalLLaMA talk summary):
  kernel list items 链式矩阵乘法, 融合LoRA, SwiGLU, RMS Layernorm.
* [Gemma blog] "+1 to RMS LayerNorm" (the (1 + w) gain of Gemma).

The pages do not print the NF4 codebook, the block size or the absmax type;
the oracle takes the QLoRA NormalFloat construction (block 64, fp32 absmax,
16 levels from N(0,1) quantiles) in its plainest reading.  Every reading the
pages leave open is stated in the docstring of the function that makes it.

Parity status: every function here is pinned by a CPU test under ``tests/``
(closed forms, invariants, brute force, finite differences, or an independent
library routine used as a textbook).  The one exception is agreement of the
codebook with the table printed in the QLoRA paper itself: that paper is not
available here, so that single comparison is "parity unpinned"; the
construction is pinned by its defining property instead.
"""

from .bf16 import bf16_bits_to_f64, f32_to_bf16_bits, f64_to_f32
from .nf4 import (NF4_BLOCK, nf4_codebook, nf4_dequantize, nf4_midpoints,
                  nf4_quantize, nf4_quantize_bruteforce)
from .lora import (ACTIVATIONS, act_fwd, act_grad, linear_bwd, linear_fwd,
                   mlp_bwd, mlp_fwd)
from .cost import bracket_costs, bracket_speedup_limit
from .norm import rmsnorm_bwd, rmsnorm_fwd

__all__ = [
    "bf16_bits_to_f64", "f32_to_bf16_bits", "f64_to_f32",
    "NF4_BLOCK", "nf4_codebook", "nf4_midpoints", "nf4_quantize",
    "nf4_quantize_bruteforce", "nf4_dequantize",
    "ACTIVATIONS", "act_fwd", "act_grad", "linear_fwd", "linear_bwd",
    "mlp_fwd", "mlp_bwd", "bracket_costs", "bracket_speedup_limit", "rmsnorm_fwd", "rmsnorm_bwd",
]
