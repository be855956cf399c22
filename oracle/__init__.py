"""Oracle for the TurboQuant hot path: a plain, slow, fp64 CPU restatement of the method.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this package: only the
tests, the smoke check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` use it.
It shares no code with the CUDA library (``kv_cache_vector_06_b200``); the only thing the two
sides share is the seeded input generator module ``synth``, which holds none of the method's
arithmetic.

Sources (web pages, cited by title and section):
  [LP]  "TurboQuant 学习路径：论文 → 技术 → 数学" (zzszmyf.github.io)
  [JJ]  "谷歌 TurboQuant 深度拆解：LLM 内存压缩 6 倍、推理加速 8 倍、零精度损失" (juejin.cn)
  [VC]  vocus.cc article on TurboQuant (PolarQuant stage / QJL 1-bit stage)
  [ZC]  "TurboQuant+ 深度解析" (zhichai.net)

Modules:
  codebook   Lloyd-Max codebook for the post-rotation coordinate density
  rotation   randomized Walsh-Hadamard rotation (FWHT and dense Sylvester form)
  encode     norm -> rotate -> codes -> residual -> QJL signs; packing / unpacking
  estimate   query preparation and the unbiased inner-product estimator
  attention  decode attention over the compressed cache (contiguous and paged)
  search     inner-product top-k and recall against exact brute force

Parity status: every function is pinned by a ``-m "not gpu"`` test against something other
than itself (closed forms, library routines, brute force, invariants, Monte Carlo); see the
header of each module.
"""
from . import codebook, rotation, encode, estimate, attention, search  # noqa: F401
