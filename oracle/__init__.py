"""fp64 CPU oracle for dynamic sparse attention -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct NumPy implementation of what the CUDA
library computes, written from the pages' description of the method:

* MInference 1.0 ("MInference 1.0: Accelerating Pre-filling for Long-Context
  LLMs via Dynamic Sparse Attention"), section "方法介紹" (method): the
  block-sparse index from mean-pooled Q and K (pooling commutes with MatMul),
  the vertical-slash index from the attention of the last queries against all
  keys, and block-sparse FlashAttention over the chosen 64x64 blocks; Fig. 4:
  slash lines run as 64x64 blocks, vertical lines as 1x64 column tiles.
* Squeezed Attention ("Squeezed Attention：基于语义聚类的长上下文LLM推理加速"),
  section "技术方案" (online stage): score the query against every cluster
  centroid, keep the top clusters, attend only over their keys and values;
  (offline stage, ``clusters.py``): Lloyd's K-means over the fixed context's
  keys, the centroids and the cluster -> key map.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The CUDA product path never calls it, and it
shares no code with the CUDA path: the only thing both see is the seeded
synthetic input from ``synth``.

Every function works in fp64 on bf16 values widened exactly to fp64.

Parity pins (tests that tie this oracle to something other than itself) live
in ``tests/test_oracle_pins.py``.  The planted-structure recall is reported as
a diagnostic only ("parity unpinned": the pages fix no expected recall).
"""

from .blocksel import (  # noqa: F401
    pool_blocks,
    ratio_ppm,
    extra_budget,
    max_blocks_per_row,
    select_top,
    block_scores,
    block_index,
)
from .vslash import vs_scores, vs_topk, vs_plan, vs_index  # noqa: F401
from .attention import sparse_attention_rows, sparse_attention, dense_lists  # noqa: F401
from .decode import decode_centroids, decode_select, decode_attention, sparse_decode  # noqa: F401
from .ties import compare_index_sets  # noqa: F401
from .ashape import a_shape_lists  # noqa: F401
from .clusters import (  # noqa: F401
    segment_means,
    kmeans_assign,
    kmeans_update,
    kmeans,
    kmeans_objective,
    cluster_csr,
    cluster_select,
    cluster_tokens,
    cluster_decode_attention,
)
