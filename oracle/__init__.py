"""Plain float64 CPU oracle for FlashPrefill V2 block-sparse prefill attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code, header, table or helper with the CUDA library under
``block_sparse_long_fp2_b200/``; the only code both sides use is the seeded
input generator ``block_sparse_long_fp2_b200.synth``, which holds none of
the method's arithmetic.

Every function restates, in float64 NumPy and in the pages' order, one step
of the method described in "FlashPrefill V2: Block-Sparse Prefill Attention
for Long-Context LLM Serving" (metallab.ai summary of arXiv 2608.19758):

* Figure 3 -- stage 1 pools block means and selects blocks per KV head
  under PackGQA; stage 2 attends over the selected blocks and merges the
  correction path inside the online softmax.
* Figure 4 -- each pruned block J adds the surrogate |B_J| e^{s_J} (v_J, 1)
  to the softmax numerator and denominator.
* Abstract -- "max-based dynamic thresholding" (Table 9 calls the threshold
  alpha; here it is tau).
* Table 1 footnote / Table 7 -- FP8 via direct online quantisation.
* Table 6 -- chunked prefill (a chunk of new queries over a KV cache holding
  the earlier tokens): ``oracle.fp2_chunked``, under the reading stated in
  its module docstring.

Pinned by ``tests/test_oracle.py`` and ``tests/test_oracle_chunked.py`` (see
the module docstrings of ``oracle.fp2_oracle`` and ``oracle.fp2_chunked`` for
which pin covers which function).  No function here is "parity unpinned".
"""

from .fp2_oracle import (  # noqa: F401
    block_layout,
    block_means,
    block_scores,
    select_blocks,
    plan,
    attend,
    attend_rows,
    dense_attention,
    gather_paged,
    e4m3_round,
    quantize_e4m3,
    dequantize_e4m3,
)
from .fp2_chunked import (  # noqa: F401
    chunk_layout,
    query_block_means,
    plan_chunk,
    attend_chunk,
)
