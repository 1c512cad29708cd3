"""CPU oracle for the QLoRA NF4 linear layer: TEST INFRASTRUCTURE ONLY.

This package is the slow, plain reference the CUDA library is checked against.
Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
arm of ``bench.py`` may import it. The GPU library never calls it, shares no code,
table or constant generator with it, and fails loudly when its CUDA extension is
missing instead of falling back here.

Everything is NumPy (float64 for real-valued results, explicit float32 where the
method fixes fp32 rounding) plus ``statistics.NormalDist`` for the inverse normal
CDF. Sources, cited by page title and section:

  * "QLoRA: Efficient Finetuning of Quantized LLMs" (Heng's Blog), 贡献一 4-bit
    NormalFloat (codebook, blockwise absmax, nearest level, stored 4-bit index),
    贡献二 Double Quantization (8-bit float codes in blocks of 256 after subtracting
    the mean; overhead 0.5 -> 0.127 bit/param), and the opening formula
    h = dequant(W0^NF4) x + (alpha/r) B A x with only A and B trained.
  * "AQLoRA: a zero-search scheme for fast quantized LoRA fine-tuning", §3.1
    (profiling pass): per-layer blockwise NF4 reconstruction error over 64-element
    blocks of the flattened weight.
  * "LowRA" article (cloud.tencent.com.cn), §4.1 (per-output-channel quantization,
    64-element absmax group normalisation, thresholds = bin edges, mappings =
    representative values, Fig. 3), 第五部分 (weighted Lloyd-Max learner of the
    mappings and thresholds).

Parity status of each function is listed in its docstring. Conventions the pages
leave open (tail probability of the NF4 grid, nibble order, tie rules, the 8-bit
float format for double quantization) are self-consistent readings and marked
"parity unpinned" where no page fixes them.
"""
from . import numerics, nf4, linear, chanq, rank, lloyd, loftq  # noqa: F401
