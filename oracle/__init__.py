"""CPU oracle for the Psi-Spec decode iteration (test infrastructure only).

This package is the plain, slow, obviously-correct restatement of what the
CUDA path computes.  It exists to check that path and nothing else: only the
test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
leg of ``bench.py`` may import it.  The product (the ``libuno`` shared library
and its Python binding) never imports, links or calls anything in here, and
this package never imports the product.

All floating-point arithmetic is numpy float64.  Inputs given in bfloat16 or
float32 are upcast exactly before use.

Sources.  The method is described only on web pages about the paper
"Unlocking Lossless Speedups in LLMs via Discrete Diffusion" (the "Uno"
models).  Citations in this package name the page and its section:

* Summary  = the daily-paper summary page titled
  "通过离散扩散实现 LLM 无损加速：扩散增强自回归模型" (section 方法关键点).
* Walkthrough = the blog page titled
  "不砸掉重来，给自回归 LLM 装一对“扩散翅膀”：Uno 的无损加速之路"
  (sections 一句话直觉, Diffusion Distillation：一步蒸馏 + 块级扩散,
  Ψ-Spec 采样器：起草、验证、两种模式).
* Abstract = the paper's English abstract as reprinted on the abstract pages.
* Philox  = Salmon, Moraes, Dror & Shaw, "Parallel random numbers: as easy
  as 1, 2, 3", SC'11, section on the Philox family.

Modules:

* :mod:`oracle.philox`  - Philox4x32-10 and the uniform draws of the sampler.
* :mod:`oracle.model`   - transformer forward with gated LoRA and an explicit
  block-causal mask matrix.
* :mod:`oracle.psispec` - the Psi-Spec linear sampler (draft, verify,
  residual resample, commit), AR-only decode and prefill.

Parity status of each function is stated in its docstring.  Functions with no
independent pin say "parity unpinned".
"""
