"""Streaming compressed blocks from host memory (the CPU-offload setting).

Source: "DFloat11 : compression sans perte pour l'inference GPU qui reduit les
LLM a 70 % de leur taille" (fr.news.hada.io) -- the method keeps the model
compressed and decompresses each transformer block on the GPU right before
its matrix multiplications; when the model does not fit on the GPU, the
compressed weights can live in host memory and cross PCIe compressed, which
moves about 70 % of the BF16 bytes.

`BlockStreamer` keeps every block's compressed arrays in pinned host memory
and, per block, copies them into one of two device slots on a copy stream
while the compute stream decodes the previous block into a reusable BF16
scratch and runs the caller's consumer on the decoded matrices.  CUDA
events order the two streams: a slot is refilled only after the compute
stream has finished decoding from it, and a block is decoded only after its
copy has landed.  Every step runs in the library's kernels; this module only
schedules copies and launches.
"""
from __future__ import annotations

from typing import Callable, Sequence

from . import _ARRAYS, DF11Tensor, _Tensor, decode_block, read_error

__all__ = ["BlockStreamer", "RawStreamer"]


def _torch():
    import torch
    return torch


def _common_arrays(blocks: Sequence[DF11Tensor]) -> list[str]:
    """The arrays every block carries (the per-thread counts are optional)."""
    return [k for k in _ARRAYS if all(k in b.arrays for b in blocks)]


def _slot_arrays(blocks: Sequence[DF11Tensor], keys, device):
    """Two device slots, each large enough for any block's arrays."""
    torch = _torch()
    size = {k: max(int(b.arrays[k].numel()) * b.arrays[k].element_size() for b in blocks) for k in keys}
    return [{k: torch.empty(max(size[k], 16), dtype=torch.uint8, device=device) for k in keys} for _ in range(2)]


class BlockStreamer:
    """Double-buffered host-to-device streaming and decoding of compressed
    blocks.  `blocks` are host tensors from `encode_multi(..., pinned=True)`
    (pinned memory makes the copies asynchronous)."""

    def __init__(self, blocks: Sequence[DF11Tensor], device="cuda"):
        torch = _torch()
        if not blocks:
            raise ValueError("no blocks")
        for b in blocks:
            if b.device != "cpu":
                raise ValueError("blocks must be host tensors (encode_multi(..., pinned=True))")
            if not all(hasattr(a, "is_pinned") and a.is_pinned() for a in b.arrays.values()):
                raise ValueError("blocks must be in pinned host memory (encode_multi(..., pinned=True))")
        self.blocks = list(blocks)
        self.keys = _common_arrays(self.blocks)
        self.device = torch.device(device)
        self.slots = _slot_arrays(self.blocks, self.keys, self.device)
        n_max = max(b.n_elems for b in self.blocks)
        self.scratch = torch.empty(max(n_max, 8), dtype=torch.bfloat16, device=self.device)
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.copy_stream = torch.cuda.Stream(device=self.device)
        self.h2d_bytes = [sum(int(b.arrays[k].numel()) * b.arrays[k].element_size() for k in self.keys)
                          for b in self.blocks]

    def _device_view(self, b: DF11Tensor, slot: int) -> DF11Tensor:
        arrays = {k: self.slots[slot][k][: int(b.arrays[k].numel()) * b.arrays[k].element_size()]
                  for k in self.keys}
        desc = _Tensor.from_buffer_copy(b.desc)
        if "counts" not in self.keys:
            desc.counts_bytes = 0
        return DF11Tensor(desc, arrays, str(self.device), b.shapes, b.offsets, b.tiled)

    def _copy(self, b: DF11Tensor, slot: int):
        for k in self.keys:
            src = b.arrays[k].view(_torch().uint8).reshape(-1)
            self.slots[slot][k][: src.numel()].copy_(src, non_blocking=True)

    def run(self, order: Sequence[int], consumer: Callable[[int, list], None] | None = None, stream=None) -> None:
        """Streams blocks in `order` (indices into `blocks`, repeats allowed):
        each is copied, decoded into the scratch, and handed to
        `consumer(block_index, views)` on the compute stream (`stream`, the
        current stream by default).  Returns after enqueueing; kernel error
        bits accumulate in `self.err` (see `check`)."""
        torch = _torch()
        compute = stream or torch.cuda.current_stream(self.device)
        order = list(order)
        if not order:
            return
        h2d_done = [torch.cuda.Event(), torch.cuda.Event()]
        slot_free = [torch.cuda.Event(), torch.cuda.Event()]
        used = [False, False]

        def prefetch(i: int):
            slot = i % 2
            with torch.cuda.stream(self.copy_stream):
                if used[slot]:
                    self.copy_stream.wait_event(slot_free[slot])
                self._copy(self.blocks[order[i]], slot)
                h2d_done[slot].record(self.copy_stream)
            used[slot] = True

        prefetch(0)
        for i, bi in enumerate(order):
            if i + 1 < len(order):
                prefetch(i + 1)
            slot = i % 2
            compute.wait_event(h2d_done[slot])
            d = self._device_view(self.blocks[bi], slot)
            decode_block(d, self.scratch, self.err, compute)
            slot_free[slot].record(compute)
            if consumer is not None:
                with torch.cuda.stream(compute):
                    consumer(bi, d.views(self.scratch))
        # the source buffers (pinned host arrays) must outlive the copies
        compute.wait_stream(self.copy_stream)

    def check(self, stream=None) -> None:
        """Synchronises and raises if any decode reported corrupt data."""
        read_error(self.err, stream)


class RawStreamer:
    """The same pipeline for uncompressed BF16 blocks (the baseline the
    compressed stream is compared with): pinned host BF16 arrays are copied
    into two device slots and handed to the consumer as matrix views."""

    def __init__(self, mats_per_block: Sequence[Sequence], device="cuda"):
        torch = _torch()
        self.device = torch.device(device)
        self.blocks = []
        for mats in mats_per_block:
            shapes = [tuple(m.shape) for m in mats]
            flat = torch.empty(sum(int(m.size) for m in mats), dtype=torch.int16, pin_memory=True)
            off = 0
            for m in mats:
                flat[off: off + m.size].copy_(torch.from_numpy(m.reshape(-1).view("int16")))
                off += m.size
            self.blocks.append((flat, shapes))
        n_max = max(int(f.numel()) for f, _ in self.blocks)
        self.slots = [torch.empty(n_max, dtype=torch.int16, device=self.device) for _ in range(2)]
        self.copy_stream = torch.cuda.Stream(device=self.device)
        self.h2d_bytes = [2 * int(f.numel()) for f, _ in self.blocks]

    def run(self, order: Sequence[int], consumer: Callable[[int, list], None], stream=None) -> None:
        torch = _torch()
        compute = stream or torch.cuda.current_stream(self.device)
        order = list(order)
        h2d_done = [torch.cuda.Event(), torch.cuda.Event()]
        slot_free = [torch.cuda.Event(), torch.cuda.Event()]
        used = [False, False]

        def prefetch(i: int):
            slot = i % 2
            flat, _ = self.blocks[order[i]]
            with torch.cuda.stream(self.copy_stream):
                if used[slot]:
                    self.copy_stream.wait_event(slot_free[slot])
                self.slots[slot][: flat.numel()].copy_(flat, non_blocking=True)
                h2d_done[slot].record(self.copy_stream)
            used[slot] = True

        if order:
            prefetch(0)
        for i, bi in enumerate(order):
            if i + 1 < len(order):
                prefetch(i + 1)
            slot = i % 2
            compute.wait_event(h2d_done[slot])
            flat, shapes = self.blocks[bi]
            views, off = [], 0
            for s in shapes:
                n = 1
                for x in s:
                    n *= x
                views.append(self.slots[slot][off: off + n].view(torch.bfloat16).view(*s))
                off += n
            with torch.cuda.stream(compute):
                consumer(bi, views)
            slot_free[slot].record(compute)
        compute.wait_stream(self.copy_stream)
