"""Double-buffered block pipeline on the device: the decode of block b+1
overlaps the consumer (the block's matrix multiplications) of block b.

Source: "DFloat11 : compression sans perte pour l'inference GPU qui reduit les
LLM a 70 % de leur taille" (fr.news.hada.io), << Decompression par bloc
transformer >> (each transformer block's matrices are decompressed together,
in one kernel launch, right before the block runs) and << Decompression
adaptee a l'inference GPU >> (the decompressed matrices are used by the
matrix multiplications and then discarded).

`BlockPipeline` keeps two BF16 scratch buffers.  Block b+1 is decoded into
one of them on a side stream while the caller's consumer runs on the compute
stream over the other; CUDA events order the two streams (a scratch is
decoded into only after the consumer of its previous block has finished, and a
block is consumed only after its decode has finished).  Every step runs in
the library's kernels; this module only schedules launches.
"""
from __future__ import annotations

from typing import Callable, Sequence

from . import DF11Tensor, decode_block, read_error

__all__ = ["BlockPipeline"]


class BlockPipeline:
    """Device-resident compressed blocks (`DF11Tensor`s on one CUDA device),
    decoded one ahead of their consumer into two alternating scratch buffers."""

    def __init__(self, blocks: Sequence[DF11Tensor], device="cuda"):
        import torch
        if not blocks:
            raise ValueError("no blocks")
        self.device = torch.device(device)
        for b in blocks:
            if b.device == "cpu":
                raise ValueError("blocks must be on the device (DF11Tensor.to('cuda'))")
        self.blocks = list(blocks)
        n_max = max(max(b.n_elems for b in self.blocks), 8)
        self.scratch = [torch.empty(n_max, dtype=torch.bfloat16, device=self.device) for _ in range(2)]
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.decode_stream = torch.cuda.Stream(device=self.device)

    def run(self, order: Sequence[int], consumer: Callable[[int, list], None], stream=None) -> None:
        """Runs `consumer(block_index, matrix_views)` on the compute stream
        (`stream`, the current stream by default) for the blocks in `order`
        (indices into `blocks`, repeats allowed), each decoded beforehand on
        the side stream.  Returns after enqueueing; kernel error bits
        accumulate in `self.err` (see `check`)."""
        import torch
        compute = stream or torch.cuda.current_stream(self.device)
        order = list(order)
        if not order:
            return
        decoded = [torch.cuda.Event(), torch.cuda.Event()]
        consumed = [torch.cuda.Event(), torch.cuda.Event()]
        used = [False, False]
        # the side stream starts after the work already queued on the compute
        # stream (the scratch buffers may still be read by an earlier run)
        self.decode_stream.wait_stream(compute)

        def decode(i: int):
            slot = i % 2
            if used[slot]:
                self.decode_stream.wait_event(consumed[slot])
            decode_block(self.blocks[order[i]], self.scratch[slot], self.err, self.decode_stream)
            decoded[slot].record(self.decode_stream)
            used[slot] = True

        decode(0)
        for i, bi in enumerate(order):
            if i + 1 < len(order):
                decode(i + 1)
            slot = i % 2
            compute.wait_event(decoded[slot])
            with torch.cuda.stream(compute):
                consumer(bi, self.blocks[bi].views(self.scratch[slot]))
            consumed[slot].record(compute)
        compute.wait_stream(self.decode_stream)

    def check(self, stream=None) -> None:
        """Synchronises and raises if any decode reported corrupt data."""
        read_error(self.err, stream)
