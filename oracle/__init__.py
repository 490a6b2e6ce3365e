"""CPU oracle for the batch-invariant, error-compensated decode step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product (the CUDA library and its
Python binding) imports, links or calls this package; only the test-suite,
the benchmark's CPU-baseline leg and the smoke check do.  It shares no code,
table or constant generator with the CUDA path.

Two kinds of functions live here:

* encodings (`oracle.encodings`): results that are by definition bit patterns
  -- the binary16 hi/lo split of the error-compensated GEMM, the packed weight
  image, the INT16 KV-cache codes and scales.  They are written step by step
  from their definitions (IEEE-754 binary16, round-half-to-even; strict fp32
  division for the quantiser) so the GPU must match them bit for bit.
* references (`oracle.reference`): the plain mathematical definitions of what
  the path approximates -- matrix product, RMSNorm, rotary embedding, softmax
  attention over the dequantised cache, the decode layer and the layer stack --
  evaluated in float64.

Sources (cited per function):
  [HEAL]  "Demystifying Numerical Instability in LLM Inference: Achieving
          Reproducible Inference for Mission-Critical Tasks with HEAL"
          (gist.science explainer of arXiv 2606.21023).
  [BI]    Blog summary of Thinking Machines Lab, "Defeating Nondeterminism in
          LLM Inference" (mobiles-han.blogspot.com, 2025/09), section
          "解決へのアプローチ：3種の主要演算の再設計" (table of RMSNorm /
          MatMul / Attention).
Every function here is pinned by a `-m "not gpu"` test against closed forms,
an independent library routine or brute force; none is "parity unpinned".
"""
