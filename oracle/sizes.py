"""Closed forms for KV-cache sizes and block counts (oracle; test infrastructure only).

Page "LLM 推理引擎 Continuous Batching 与 PagedAttention":
* §1.2 (KV Cache 的本质): bytes per token = 2 (K and V) x layers x heads x
  head_dim x bytes per element.
* §3.2 (核心数据结构, ``BlockManager.allocate``): a request of n tokens takes
  ceil(n / block_size) blocks.
* §3.4 (Block Size 的选择): the last block of a request wastes at most
  block_size - 1 token slots; the expected waste fraction is about
  (block_size / 2) / average length.
"""
from __future__ import annotations


def kv_bytes_per_token(layers: int, heads: int, head_dim: int, bytes_per_elem: int) -> int:
    """K and V bytes one token occupies across all layers (§1.2)."""
    return 2 * layers * heads * head_dim * bytes_per_elem


def blocks_needed(num_tokens: int, block_size: int) -> int:
    """ceil(num_tokens / block_size), in integers (§3.2)."""
    if num_tokens < 0 or block_size <= 0:
        raise ValueError("num_tokens must be >= 0 and block_size > 0")
    return (num_tokens + block_size - 1) // block_size


def internal_waste(num_tokens: int, block_size: int) -> int:
    """Unused token slots in a request's last block (§3.4)."""
    return blocks_needed(num_tokens, block_size) * block_size - num_tokens


def expected_waste_fraction(block_size: int, avg_len: float) -> float:
    """The page's estimate of the wasted fraction, (block_size / 2) / avg_len (§3.4)."""
    return (block_size / 2) / avg_len
