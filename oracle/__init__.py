"""CPU oracle for the Elastic Attention prefill path — TEST INFRASTRUCTURE ONLY.

Plain, slow, fp64 numpy statement of what the path computes, written from the
paper summary "Elastic Attention: Test-time Adaptive Sparsity Ratios for
Efficient Transformers" (paperlayer.ai, arXiv 2601.17367v2).  Only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may use
it; the product path (the CUDA library and its Python binding) never imports
it and shares no code with it.

Modules:
  router    — boundary pooling, key projection, task MLP, router MLP, hard
              threshold (section 3 "Attention Router"; appendix H.4 "Router
              Input Length"; section 5 "Attention Router" for the x4 width;
              section 1 for the 0.27M-parameter budget).
  attention — the hybrid-head mechanism: each KV-head group runs full causal
              attention or a sparse pattern, outputs concatenated per head
              (section 2 "Hybrid Head Mechanism"; section 3 "Attention
              Router"; appendix D.1 "Sparse Inference").
  sparsity  — model sparsity ratio and effective sparsity ratio (section 2
              "Sparsity Ratio Computation"; appendix C.1 "Sparsity Assignment").
  assignment — retrieval scores, static retrieval-head assignment
              k = floor((1 - Omega_MSR) L H) and whole-stack sparsity
              (appendix C.1 "Retrieval Score Calculation", "Sparsity
              Assignment").
  xattention — XAttention block selection feeding the block-sparse heads'
              layout (section 4 "Evaluation Setting": tau = 0.9; the method
              restated from Xu et al. 2025, whose agreement with XAttention's
              own implementation is "parity unpinned").

Inputs are taken as given (bf16 inputs arrive already widened to float) and
every product and sum runs in float64.  Where the pages leave a step open the
reading taken is stated in the function's docstring; every one of them is
pinned by tests in ``tests/test_oracle_*.py`` except the agreement of the
router's wiring with the paper's trained router, which no page fixes: that
part is "parity unpinned" (the written form is pinned, its identity with the
paper's network is not).
"""
from . import assignment, attention, router, sparsity, xattention  # noqa: F401
from .attention import FULL, STREAMING, BLOCK_SPARSE, STREAMING_BLOCKS  # noqa: F401
