"""Seeded synthetic inputs for the paged-KV attention workloads.

This module holds random draws and workload constants only: sequence
lengths, free-list permutations, churn-op draws and N(0, 1) fp16 tensors.
It holds none of the attention or block-allocation arithmetic (no block
counts, no slot numbers, no softmax).  Both the CPU oracle and the CUDA path
consume these draws and do their own bookkeeping from them.

Every draw comes from its own child generator
``numpy.random.default_rng([seed, purpose, *index])`` so that the order in
which a consumer asks for draws never changes their values.

The five workloads follow the paged-attention decode shapes of the page
"LLM 推理引擎 Continuous Batching 与 PagedAttention" (Llama-2-7B: 32 heads of
dimension 128, fp16, §1.2; default block size 16 and 32 for long sequences,
§3.4; chunked prefill, §4.3; shared system-prompt prefix, §4.1) and of the
chapter "动态批处理算法" (§4.5: 7B model, batch 32, requests of 64-1024
tokens).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

# Child-generator purposes.  Changing a number changes every workload.
_PURPOSE = {
    "lens": 1,
    "free_order": 2,
    "churn": 3,
    "churn_final": 4,
    "q": 5,
    "k_new": 6,
    "v_new": 7,
    "k_ctx": 8,
    "v_ctx": 9,
    "q_chunk": 10,
    "k_chunk": 11,
    "v_chunk": 12,
    "k_prefix": 13,
    "v_prefix": 14,
    "garbage": 15,
}

_CHUNK = 1 << 22


def rng(seed: int, purpose: str, *index: int) -> np.random.Generator:
    """Independent generator for one purpose (and optional index)."""
    return np.random.default_rng([int(seed), _PURPOSE[purpose], *[int(i) for i in index]])


def normal_fp16(gen: np.random.Generator, shape) -> np.ndarray:
    """N(0, 1) samples rounded to fp16, drawn in fixed-size float32 chunks."""
    out = np.empty(shape, dtype=np.float16)
    flat = out.reshape(-1)
    for i in range(0, flat.size, _CHUNK):
        n = min(_CHUNK, flat.size - i)
        flat[i:i + n] = gen.standard_normal(n, dtype=np.float32)
    return out


@dataclasses.dataclass(frozen=True)
class ChurnSpec:
    """Seeded allocate/append/free churn run on the pool before the step."""
    n_ops: int = 10_000
    max_tokens: int = 512


@dataclasses.dataclass(frozen=True)
class PrefillSpec:
    """One chunked-prefill request appended after an already cached prefix."""
    ctx_before: int = 1536
    chunk: int = 512


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic paged-attention step.

    ``decode_lens[s]`` is sequence s's length *including* the token decoded
    in this step (its K/V is written by the step before attention reads it).
    ``pool_factor`` sizes the pool as that multiple of the demanded blocks
    (rounded up); ``pool_blocks`` fixes the pool size instead.
    """
    name: str
    seed: int
    num_heads: int
    head_dim: int
    block_size: int
    decode_lens: tuple
    pool_factor: Optional[float] = None
    pool_blocks: Optional[int] = None
    shuffle_free_list: bool = True
    churn: Optional[ChurnSpec] = None
    prefill: Optional[PrefillSpec] = None
    shared_prefix: int = 0

    @property
    def num_seqs(self) -> int:
        return len(self.decode_lens)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    # ---- draws -----------------------------------------------------------
    def free_order(self, num_blocks: int) -> np.ndarray:
        """Initial free-list order of the pool (int32)."""
        if not self.shuffle_free_list:
            return np.arange(num_blocks, dtype=np.int32)
        return rng(self.seed, "free_order").permutation(num_blocks).astype(np.int32)

    def q(self) -> np.ndarray:
        return normal_fp16(rng(self.seed, "q"), (self.num_seqs, self.num_heads, self.head_dim))

    def k_new(self) -> np.ndarray:
        return normal_fp16(rng(self.seed, "k_new"), (self.num_seqs, self.num_heads, self.head_dim))

    def v_new(self) -> np.ndarray:
        return normal_fp16(rng(self.seed, "v_new"), (self.num_seqs, self.num_heads, self.head_dim))

    def context_kv(self, seq: int, n_tokens: int):
        """Logical K/V of sequence ``seq``'s private cached context (fp16 [n, H, D])."""
        shape = (n_tokens, self.num_heads, self.head_dim)
        return (normal_fp16(rng(self.seed, "k_ctx", seq), shape),
                normal_fp16(rng(self.seed, "v_ctx", seq), shape))

    def prefix_kv(self):
        """Logical K/V of the shared prefix (fp16 [shared_prefix, H, D])."""
        shape = (self.shared_prefix, self.num_heads, self.head_dim)
        return (normal_fp16(rng(self.seed, "k_prefix"), shape),
                normal_fp16(rng(self.seed, "v_prefix"), shape))

    def prefill_qkv(self):
        """q, k, v of the prefill chunk (fp16 [chunk, H, D] each)."""
        shape = (self.prefill.chunk, self.num_heads, self.head_dim)
        return (normal_fp16(rng(self.seed, "q_chunk"), shape),
                normal_fp16(rng(self.seed, "k_chunk"), shape),
                normal_fp16(rng(self.seed, "v_chunk"), shape))

    def prefill_context_kv(self):
        """Logical K/V of the prefill request's cached prefix."""
        shape = (self.prefill.ctx_before, self.num_heads, self.head_dim)
        return (normal_fp16(rng(self.seed, "k_ctx", 1 << 20), shape),
                normal_fp16(rng(self.seed, "v_ctx", 1 << 20), shape))

    def churn_ops(self):
        """Churn draws: (kind in {0: allocate, 1: append, 2: free}, u in [0,1), tokens)."""
        g = rng(self.seed, "churn")
        n = self.churn.n_ops
        kind = g.integers(0, 3, size=n)
        u = g.random(n)
        tokens = g.integers(1, self.churn.max_tokens + 1, size=n)
        return kind, u, tokens

    def churn_final_order(self, n_live: int) -> np.ndarray:
        """Order in which the churn requests still live at the end are freed."""
        return rng(self.seed, "churn_final").permutation(n_live)


# Request-id namespaces used by both workload builders.
CHURN_REQ_BASE = 1_000_000
PREFILL_REQ = 900_000
PREFIX_REQ = 800_000


def _uniform_lens(seed, n, lo, hi):
    return tuple(int(x) for x in rng(seed, "lens").integers(lo, hi + 1, size=n))


def _log_uniform_lens(seed, n, lo, hi):
    g = rng(seed, "lens")
    return tuple(int(round(math.exp(x))) for x in g.uniform(math.log(lo), math.log(hi), size=n))


def tiny() -> Workload:
    """4 sequences {5,16,17,33}, 4 heads x 64, bs 16, a 16-block permuted pool."""
    return Workload(name="tiny_b4_h4_d64_bs16", seed=1, num_heads=4, head_dim=64, block_size=16,
                    decode_lens=(5, 16, 17, 33), pool_blocks=16)


def llama7b_b32() -> Workload:
    """Llama-2-7B layer shape, batch 32, lengths uniform in [64, 1024], pool 1.1x demand."""
    return Workload(name="llama2_7b_decode_b32_len64_1024_bs16", seed=2, num_heads=32, head_dim=128,
                    block_size=16, decode_lens=_uniform_lens(2, 32, 64, 1024), pool_factor=1.1)


def llama7b_b256_ragged() -> Workload:
    """Batch 256, lengths log-uniform in [16, 4096], pool 1.5x demand fragmented by 10k churn ops."""
    return Workload(name="llama2_7b_decode_b256_loguniform16_4096_bs16_churn10k", seed=3,
                    num_heads=32, head_dim=128, block_size=16,
                    decode_lens=_log_uniform_lens(3, 256, 16, 4096), pool_factor=1.5,
                    shuffle_free_list=False, churn=ChurnSpec())


def mixed_prefill_decode() -> Workload:
    """512-token causal prefill chunk after 1536 cached tokens + 64 decodes in [128, 2048]."""
    return Workload(name="mixed_prefill512_ctx1536_plus_decode64_len128_2048_bs16", seed=4,
                    num_heads=32, head_dim=128, block_size=16,
                    decode_lens=_uniform_lens(4, 64, 128, 2048), pool_factor=1.1,
                    prefill=PrefillSpec())


def long_shared_prefix() -> Workload:
    """8 sequences of 32768 at bs 32 sharing a 1024-token refcounted prefix."""
    return Workload(name="longctx_b8_len32768_bs32_shared_prefix1024", seed=5, num_heads=32,
                    head_dim=128, block_size=32, decode_lens=(32768,) * 8, pool_factor=1.1,
                    shared_prefix=1024)


def causal_prefill_8k() -> Workload:
    """One 8192-token prompt prefilled as a single causal chunk (nothing cached before it)."""
    return Workload(name="llama2_7b_prefill8192_causal_bs16", seed=6, num_heads=32, head_dim=128,
                    block_size=16, decode_lens=(), pool_factor=1.1,
                    prefill=PrefillSpec(ctx_before=0, chunk=8192))


WORKLOADS = {
    "tiny": tiny,
    "b32": llama7b_b32,
    "b256": llama7b_b256_ragged,
    "mixed": mixed_prefill_decode,
    "longctx": long_shared_prefix,
    "prefill8k": causal_prefill_8k,
}


def get(name: str) -> Workload:
    return WORKLOADS[name]()


def with_block_size(w: Workload, block_size: int) -> Workload:
    """The same requests and draws with another block size (for block-size sweeps)."""
    if block_size == w.block_size:
        return w
    return dataclasses.replace(w, block_size=int(block_size), name=f"{w.name}__bs{block_size}")


def garbage_block_ids(seed: int, shape, num_blocks: int) -> np.ndarray:
    """In-range but wrong block ids used to fill the padding of packed block tables in tests."""
    return rng(seed, "garbage").integers(0, num_blocks, size=shape).astype(np.int32)
