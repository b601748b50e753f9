"""Closed-form KV-cache size.

TEST INFRASTRUCTURE (see ``oracle/__init__``).

Page "5.KV Cache 管理 & PagedAttention", Q1 (1.1 核心公式推导, 1.2 代码实现) and
the "KV Cache 显存占用计算" listing on page "paged-attention-and-vllm-inference":
every layer stores a K and a V of num_kv_heads * head_dim elements per token,
so

    bytes = 2 * num_layers * num_kv_heads * head_dim * seq_len * batch * dtype_bytes

with num_kv_heads = num_heads for MHA and the smaller KV head count for
GQA/MQA, and dtype_bytes = 2 for FP16, 1 for an FP8/INT8 cache (Q1, 1.3).
"""


def kv_cache_bytes(num_layers: int, num_kv_heads: int, head_dim: int, seq_len: int,
                   batch_size: int, dtype_bytes: int) -> int:
    per_token_per_layer = 2 * num_kv_heads * head_dim * dtype_bytes  # K + V
    return num_layers * per_token_per_layer * seq_len * batch_size


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, dtype_bytes: int) -> int:
    """K + V bytes one token adds across all layers."""
    return kv_cache_bytes(num_layers, num_kv_heads, head_dim, 1, 1, dtype_bytes)
