"""Oracle swapping between a GPU pool and a CPU pool (test infrastructure only).

Page "LLM 推理引擎 Continuous Batching 与 PagedAttention", §4.4 (Swap：CPU
offload): ``SwappingManager`` owns one block manager per pool; swapping a
request out allocates it in the CPU pool with its length, copies its blocks
and frees it in the GPU pool (§5.4 uses this instead of recomputation when a
request is preempted); swapping in is the reverse.  The page's sketch frees
before it allocates, allocates whole blocks' worth of tokens, and leaves the
copy as a comment; the reading taken here allocates the destination first,
with the request's own length (so a full destination refuses the move with
nothing changed, and the moved request keeps its length), copies block i of
the source table to block i of the destination table, then frees the source.
"""
from __future__ import annotations

from .block_manager import EXISTS, NOT_FOUND, OK, BlockManager


def _move(src: BlockManager, dst: BlockManager, req, src_k, src_v, dst_k, dst_v):
    if req not in src.block_tables:
        return NOT_FOUND
    if req in dst.block_tables:
        return EXISTS
    st = dst.allocate(req, src.seq_lens[req])
    if st != OK:
        return st
    if src_k is not None:
        for s, d in zip(src.block_tables[req], dst.block_tables[req]):
            dst_k[d] = src_k[s]
            dst_v[d] = src_v[s]
    return src.free(req)


class SwappingManager:
    def __init__(self, gpu: BlockManager, cpu: BlockManager):
        if gpu.block_size != cpu.block_size:
            raise ValueError("pools differ in block size")
        self.gpu, self.cpu = gpu, cpu

    def swap_out(self, req, gpu_k=None, gpu_v=None, cpu_k=None, cpu_v=None):
        return _move(self.gpu, self.cpu, req, gpu_k, gpu_v, cpu_k, cpu_v)

    def swap_in(self, req, gpu_k=None, gpu_v=None, cpu_k=None, cpu_v=None):
        return _move(self.cpu, self.gpu, req, cpu_k, cpu_v, gpu_k, gpu_v)
