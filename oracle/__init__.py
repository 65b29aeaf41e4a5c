"""Plain float64 CPU oracle for the exact attention forward and its FP8 pre-processing.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` leg and its
``--impl reference`` arm) may import or run it.  It shares no code with the CUDA path.

Sources (the three pages this project restates; cited by page title and section):

* "FlashAttention-3" (lyirs.cc), intro formula and section "数学对象没变" (the
  mathematical object is unchanged): ``Attention(Q,K,V) = softmax(Q K^T / sqrt(d)) V``.
* same page, section "先回顾 FlashAttention 家族保留下来的部分": per-row running statistics
  ``m_i = max_j s_ij`` and ``l_i = sum_j exp(s_ij - m_i)``.
* "FlashAttention-2/3" (compassingai.com), section "技术原理": the standard three-step
  computation and the tiled outer-Q / inner-K,V loop with the m/l correction.
* "Flash Attention V3 ... 解析" (jsqmd.com), section 2.2: only the logsumexp is kept per row.
* "FlashAttention-3", section "FP8 路径与低精度误差": ``x~ = H D x`` with ``D`` a random
  sign diagonal and ``H`` a Hadamard transform; "FlashAttention-2/3", section
  "FA-3：拥抱 Hopper", feature 3: per-block (not global) FP8 scales.

Modules
-------
``oracle.attention``  two-pass attention (the definition), the pages' blockwise m/l
                      recurrence, a lazy-rescale blockwise variant in base 2, a packed
                      batch of sequences of different lengths built on the definition, and
                      the merge of two partial results over disjoint key sets.
``oracle.fp8``        Sylvester Hadamard matrix, fast Walsh-Hadamard transform in float32,
                      E4M3 (OCP E4M3FN) rounding/encoding, per-block quantisation.
``oracle.rope``       rotary position embedding (rotate-half pairing, caller's cos/sin
                      tables) in float32, ahead of the Hadamard/E4M3 pre-processing.
``oracle.attention_bwd``  the backward pass (dQ, dK, dV) from the chain rule on whole score
                      matrices, the same evaluated a block of query rows at a time (for long
                      sequences), also per sequence of a packed batch; the pages only state that
                      it exists and recomputes the softmax ("FlashAttention-3", "适用范围和工程限制";
                      "Flash Attention V3 解析" 2.1).

Every function is pinned by ``tests/test_oracle_*.py`` against closed forms, invariants,
library routines (torch SDPA in float64, scipy's Hadamard, ml_dtypes/torch float8), central
finite differences of the forward oracle (for the backward) and hand-derived fixtures in
``tests/golden/``.
"""

from .attention import (  # noqa: F401
    attention_ref,
    attention_blockwise_ref,
    attention_blockwise_lazy_ref,
    attention_varlen_ref,
    merge_partials_ref,
    visible_mask,
)
from .attention_bwd import (  # noqa: F401
    attention_bwd_ref,
    attention_bwd_chunked_ref,
    attention_varlen_bwd_ref,
    softmax_bwd_delta,
    softmax_probs,
)
from .fp8 import (  # noqa: F401
    E4M3_MAX,
    sylvester_hadamard,
    hadamard_rotate_ref,
    fwht_f32,
    e4m3_round,
    e4m3_encode,
    e4m3_decode,
    hadamard_quant_ref,
    dequant_ref,
)
from .rope import rope_ref  # noqa: F401
