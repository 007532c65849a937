"""CPU oracle for block-sparse attention with in-softmax block approximation.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.  Only the test suite,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
or run anything in this package.  The library ``libsparseattn`` never calls it
and shares no code, constant or helper with it.

Everything here is plain numpy in float64, written step by step from the
definitions on the pages it cites:

* [SLA2]  "SLA2: Sparse-Linear Attention with Learnable Routing and QAT"
* [SALAD] "SALAD: Achieve High-Sparsity Attention via Efficient Linear
          Attention Tuning for Video Diffusion Transformer"
* [PISA]  "PISA - Atenção Esparsa por Partes para Transformers de Difusão
          Eficientes"
* [SPLA]  "SPLA - Block Sparse Plus Linear Attention para Modelagem de
          Contexto Longo"
* [SFA]   "Scaling Attention via Feature Sparsity" (feature_sparse.py)

Pinning status of each public function (what fixes it other than itself) is
listed in ``oracle.sparse_attention.__doc__``.
"""

from .sparse_attention import (  # noqa: F401
    block_pool,
    route_scores,
    decode_route_scores,
    topk_from_scores,
    k_from_percent,
    sparse_attention,
    decode_attention,
    e4m3_round,
    quantise_blocks_e4m3,
    fp8_attention,
)
from .feature_sparse import sfa_codes, sfa_densify, sfa_attention  # noqa: F401
from .backward import sparse_attention_backward, sparse_attention_lse  # noqa: F401
