"""fp64 CPU oracle for exact softmax attention and the e4m3 Q/K quantiser.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
its Python binding) imports, links or runs anything in this package.  Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline leg
and its ``--impl reference`` arm) may use it.

The oracle shares no code with the GPU path: no kernels, headers, helpers,
tables or constant generators.  The one module both sides use is the seeded
input generator ``tiled_attention_12_b200.synth``, which holds none of the
method's arithmetic.

Sources (web pages on FlashAttention, cited by title and section):
  * "Flash Attention" tag page (guijiagi.com), excerpts "Flash Attention
    解决了什么问题" (the plain definition S = QK^T/sqrt(d), P = softmax(S),
    O = PV) and "Flash Attention 系列回顾" (the (batch, heads, seq, dim) layout).
  * "从理论到实现：基于Triton剖析FlashAttention三代的演进与优化",
    §2.1 (online softmax), §3.1 (block causal mask), §4.1 (FP8 dynamic scales).
  * "FlashAttention速度提升的核心原理", §1.3 (online softmax renormalisation).
  * "深度解析注意力机制的变体与演进", sections "Block Sparse Attention" and
    "Ring Attention".

Every function below says which passage it follows.
"""

from .attention import attention_ref, attention_rows, attention_flops
from .online import online_attention
from .brute import brute_attention
from .e4m3 import e4m3_decode, e4m3_encode_rne_satfinite, E4M3_MAX
from .quantize import quantize_e4m3_tiles, dequantize_e4m3_tiles
from .backward import attention_bwd_ref, attention_bwd_d
from .block_sparse import attention_block_sparse_ref, attention_block_sparse_rows, block_sparse_flops
from .merge import merge_partials_ref, ring_schedule

__all__ = [
    "attention_ref", "attention_rows", "attention_flops", "online_attention",
    "brute_attention", "e4m3_decode", "e4m3_encode_rne_satfinite", "E4M3_MAX",
    "quantize_e4m3_tiles", "dequantize_e4m3_tiles", "attention_bwd_ref", "attention_bwd_d",
    "attention_block_sparse_ref", "attention_block_sparse_rows", "block_sparse_flops",
    "merge_partials_ref", "ring_schedule",
]
