"""CPU oracle for the DSA hot path -- test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It shares no code with the CUDA library.
"""
from .dsa_ref import (attention_probs, bf16_decode, bf16_encode_rne, dense_mla,  # noqa: F401
                      e4m3_decode, e4m3_encode_rne, forward, indexer_scores, sparse_mla,
                      topk_select)
from . import projection  # noqa: F401,E402
from . import backward  # noqa: F401,E402
