"""The five synthetic DSA workloads, by name.

Shapes follow the DeepSeek-V3.2 sparse-attention description: a 128-dim FP8
lightning-indexer key per token, top-2048 fine-grained selection, and MQA-form
MLA over a 512-dim latent plus a 64-dim decoupled-RoPE key (page "一文讀懂
DeepSeek-V3.2核心技術DSA", section "DSA 的兩大核心組件" and "四步工作流程";
page "DeepSeek-V3.2加速技术详解", section 3.2).  Head counts, the value
distributions and the softmax scale are the workload's own choices.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

D_INDEX = 128      # lightning-indexer key/query width
D_LATENT = 512     # MLA latent (also the value) width
D_ROPE = 64        # decoupled RoPE key width
D_QK = D_LATENT + D_ROPE   # 576: width of one MLA key row
D_V = D_LATENT             # 512


@dataclass(frozen=True)
class Workload:
    name: str
    cfg_id: int            # sub-stream id used by the input generator
    kind: str              # "prefill" | "decode" | "chunked_prefill"
    k: int                 # top-k
    h_index: int           # indexer heads H_I
    heads: int             # MLA query heads H
    # prefill / chunked prefill
    seq_len: int = 0
    chunk: int = 0
    # decode
    batch: int = 0
    ctx_min: int = 0
    ctx_max: int = 0
    q_per_seq: int = 0
    sm_scale: float = field(default=1.0 / math.sqrt(D_QK))


WORKLOADS: dict[str, Workload] = {
    "tiny_prefill": Workload("tiny_prefill", 1, "prefill", k=256, h_index=4, heads=8,
                             seq_len=1024),
    "prefill_8k": Workload("prefill_8k", 2, "prefill", k=2048, h_index=64, heads=128,
                           seq_len=8192),
    "decode_b64": Workload("decode_b64", 3, "decode", k=2048, h_index=64, heads=128,
                           batch=64, ctx_min=4096, ctx_max=32768, q_per_seq=1),
    "chunked_64k": Workload("chunked_64k", 4, "chunked_prefill", k=2048, h_index=64,
                            heads=128, seq_len=65536, chunk=4096),
    "decode_128k_mtp2": Workload("decode_128k_mtp2", 5, "decode", k=2048, h_index=64,
                                 heads=128, batch=16, ctx_min=131072, ctx_max=131072,
                                 q_per_seq=2),
    # batch-1 long-context decode (one sequence at 131072, one new token), run
    # with a paged cache: the second decode workload of the paged-serving setting
    "decode_b1_128k": Workload("decode_b1_128k", 6, "decode", k=2048, h_index=64,
                               heads=128, batch=1, ctx_min=131072, ctx_max=131072,
                               q_per_seq=1),
}
