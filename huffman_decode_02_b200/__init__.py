"""huffman_decode_02_b200 -- DFloat11 (DF11) lossless BF16 weight codec for
B200 (sm_100a): host encoder + GPU decoder behind the C ABI of libdf11.so.

This module is a thin binding: it marshals arguments (numpy / torch buffers,
CUDA streams) into the C calls declared in ``include/df11.h`` and does no
part of the codec itself.  PyTorch is used for device memory and streams
only.  There is no fallback: if ``libdf11.so`` is missing or fails to load,
importing this package raises.

Typical use::

    import huffman_decode_02_b200 as df11
    t = df11.encode(w_bf16_bits)          # host: numpy uint16 / torch bf16 (CPU)
    d = t.to("cuda")                      # device copy of the compressed arrays
    w = df11.decode(d)                    # torch.bfloat16 on the GPU, bit-exact

    blk = df11.encode_multi([q, k, v, o, gate, up, down, n1, n2])
    dblk = blk.to("cuda")
    scratch = df11.decode_block(dblk)     # one launch; dblk.views(scratch) -> matrices
"""
from __future__ import annotations

import ctypes
import os
from typing import Iterable, Sequence

import numpy as np

from . import build as _build

__all__ = [
    "DF11Error", "CorruptStreamError", "Params", "DF11Tensor", "encode", "encode_multi",
    "encode_device", "encode_device_noalloc", "save", "load", "decode", "decode_block", "decode_rows", "decode_gemv",
    "decode_gemm", "gemm", "gemm_multi", "read_error", "exponent_histogram", "lib_path", "sm_count", "to_tile_order",
    "from_tile_order",
    "KERR_COUNT_MISMATCH", "KERR_BAD_CODE", "KERR_BAD_BLOCK", "KERR_OVERRUN", "KERR_TIMEOUT", "KERR_BAD_ROW",
]

KERR_COUNT_MISMATCH = 0x1
KERR_BAD_CODE = 0x2
KERR_BAD_BLOCK = 0x4
KERR_OVERRUN = 0x8
KERR_TIMEOUT = 0x10
KERR_BAD_ROW = 0x40

_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported parameter", 3: "tensor too large",
           4: "corrupt compressed data", 5: "CUDA error", 6: "out of host memory"}


class DF11Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_STATUS.get(status, status)} (status {status})")
        self.status = status


class CorruptStreamError(DF11Error):
    pass


# --------------------------------------------------------------- ctypes ABI
class _Params(ctypes.Structure):
    _fields_ = [("max_code_len", ctypes.c_uint32), ("bytes_per_thread", ctypes.c_uint32),
                ("threads_per_block", ctypes.c_uint32), ("reserved", ctypes.c_uint32)]


class _Tensor(ctypes.Structure):
    _fields_ = [("n_elems", ctypes.c_uint64), ("total_bits", ctypes.c_uint64),
                ("n_threads", ctypes.c_uint64), ("n_blocks", ctypes.c_uint64),
                ("params", _Params), ("max_block_codes", ctypes.c_uint32),
                ("reserved2", ctypes.c_uint32), ("code_len", ctypes.c_uint8 * 256),
                ("enc_bytes", ctypes.c_uint64), ("sm_bytes", ctypes.c_uint64),
                ("gaps_bytes", ctypes.c_uint64), ("block_start_bytes", ctypes.c_uint64),
                ("lut_bytes", ctypes.c_uint64), ("counts_bytes", ctypes.c_uint64),
                ("enc", ctypes.c_void_p), ("sm", ctypes.c_void_p), ("gaps", ctypes.c_void_p),
                ("block_start", ctypes.c_void_p), ("lut", ctypes.c_void_p), ("counts", ctypes.c_void_p)]


class _GemmMat(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("w", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("out", ctypes.c_uint32), ("in_", ctypes.c_uint32)]


class _GemvMat(ctypes.Structure):
    _fields_ = [("elem_offset", ctypes.c_uint64), ("rows", ctypes.c_uint32), ("cols", ctypes.c_uint32),
                ("x", ctypes.c_void_p), ("y", ctypes.c_void_p)]


# The compressed arrays; "counts" (per-thread code counts) is optional: a
# tensor without it decodes with the count pass.
_ARRAYS = ("enc", "sm", "gaps", "block_start", "lut", "counts")
_LIB = None


def lib_path() -> str:
    return _build.LIB_PATH


def _lib():
    global _LIB
    if _LIB is not None:
        return _LIB
    path = _build.LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"libdf11.so is not built ({path}); run python -m huffman_decode_02_b200.build")
    lib = ctypes.CDLL(path)
    P, T, u64, u32, vp = ctypes.POINTER, _Tensor, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_void_p
    u16pp = P(P(ctypes.c_uint16))
    lib.df11_abi_version.restype = u32
    lib.df11_sizeof_tensor.restype = ctypes.c_size_t
    lib.df11_default_params.argtypes = [P(_Params)]
    lib.df11_default_params.restype = None
    lib.df11_status_str.restype = ctypes.c_char_p
    lib.df11_exponent_histogram.argtypes = [u16pp, P(u64), u32, P(u64)]
    lib.df11_encode_size.argtypes = [P(ctypes.c_uint16), u64, P(_Params), P(T)]
    lib.df11_encode.argtypes = [P(ctypes.c_uint16), u64, P(T)]
    lib.df11_encode_multi_size.argtypes = [u16pp, P(u64), u32, P(_Params), P(T)]
    lib.df11_encode_multi.argtypes = [u16pp, P(u64), u32, P(T)]
    lib.df11_validate.argtypes = [P(T)]
    lib.df11_decode.argtypes = [P(T), vp, vp, vp]
    lib.df11_decode_block.argtypes = [P(T), P(u64), u32, vp, vp, vp]
    lib.df11_read_error.argtypes = [vp, vp, P(u32)]
    lib.df11_device_sm_count.argtypes = [P(ctypes.c_int)]
    lib.df11_gemm_bf16.argtypes = [vp, vp, vp, u32, u32, u32, vp, vp]
    lib.df11_gemm_bf16_multi.argtypes = [P(_GemmMat), u32, u32, vp, vp]
    lib.df11_decode_rows.argtypes = [P(_Tensor), ctypes.c_uint64, vp, u32, vp, vp, vp]
    lib.df11_decode_gemv.argtypes = [P(_Tensor), P(_GemvMat), u32, u32, vp, vp]
    lib.df11_decode_gemm.argtypes = [P(_Tensor), P(_GemvMat), u32, u32, vp, vp]
    lib.df11_to_tile_order.argtypes = [vp, u32, u32, vp]
    lib.df11_from_tile_order.argtypes = [vp, u32, u32, vp]
    lib.df11_encode_device_scratch_bytes.argtypes = [u64]
    lib.df11_encode_device_scratch_bytes.restype = u64
    lib.df11_encode_device_size.argtypes = [vp, u64, P(_Params), P(T), vp, u64, vp]
    lib.df11_encode_device.argtypes = [vp, u64, P(T), vp, u64, vp]
    lib.df11_encode_device_noalloc_max_elems.restype = u64
    lib.df11_encode_device_size_noalloc.argtypes = [vp, u64, P(_Params), P(T), vp]
    lib.df11_encode_device_noalloc.argtypes = [vp, u64, P(T), vp]
    if lib.df11_abi_version() != 3 or lib.df11_sizeof_tensor() != ctypes.sizeof(_Tensor):
        raise ImportError("libdf11.so ABI does not match this binding")
    _LIB = lib
    return lib


def _check(status: int, what: str) -> None:
    if status != 0:
        cls = CorruptStreamError if status == 4 else DF11Error
        raise cls(status, what)


class Params:
    """Encoder parameters (see df11_params in include/df11.h)."""

    def __init__(self, max_code_len: int = 12, bytes_per_thread: int = 8, threads_per_block: int = 256):
        self.max_code_len = max_code_len
        self.bytes_per_thread = bytes_per_thread
        self.threads_per_block = threads_per_block

    def _c(self) -> _Params:
        return _Params(self.max_code_len, self.bytes_per_thread, self.threads_per_block, 0)


# ---------------------------------------------------------------- helpers
def _as_u16(w) -> np.ndarray:
    """BF16 bits as a contiguous numpy uint16 view (no copy when possible)."""
    try:
        import torch
        if isinstance(w, torch.Tensor):
            if w.device.type != "cpu":
                raise ValueError("encode() runs on the host: pass a CPU tensor")
            if w.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
                raise TypeError(f"expected BF16 bits, got {w.dtype}")
            w = w.contiguous().view(torch.int16).numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.asarray(w)
    if a.dtype.itemsize != 2:
        raise TypeError(f"expected 16-bit BF16 bit patterns, got {a.dtype}")
    return np.ascontiguousarray(a).reshape(-1).view(np.uint16)


def _u16_ptr(a: np.ndarray):
    if a.size == 0:
        return ctypes.cast(ctypes.c_void_p(0), ctypes.POINTER(ctypes.c_uint16))
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16))


def _stream_handle(stream, device=None) -> ctypes.c_void_p:
    """The CUDA stream to launch on: `stream` if given, else the current
    stream of `device` (of the current device when None)."""
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _on(device):
    """Makes `device` the current CUDA device for the duration of a library
    call: the C entry points launch on the current device, so the data's own
    device must be current (another device's memory would be read without
    peer access).  No switch when it already is (the common case; the switch
    costs two driver calls per library call)."""
    import contextlib

    import torch
    dev = torch.device(device)
    if dev.type == "cuda" and (dev.index is None or dev.index == torch.cuda.current_device()):
        return contextlib.nullcontext()
    return torch.cuda.device(dev)


class DF11Tensor:
    """A compressed tensor: the df11_tensor descriptor plus its five arrays,
    either on the host (numpy uint8 / uint32 arrays, or pinned torch tensors)
    or on a CUDA device (torch tensors).  ``shapes`` records the original
    matrix shapes for block tensors (element offsets in ``offsets``)."""

    def __init__(self, desc: _Tensor, arrays: dict, device: str, shapes, offsets, tiled=None):
        self.desc = desc
        self.arrays = arrays
        self.device = device
        self.shapes = list(shapes)
        self.offsets = list(offsets)
        # per matrix: stored in tile order (128 x 64 tiles, for decode_gemm)
        self.tiled = list(tiled) if tiled is not None else [False] * len(self.shapes)

    # scalar fields
    n_elems = property(lambda self: int(self.desc.n_elems))
    total_bits = property(lambda self: int(self.desc.total_bits))
    n_threads = property(lambda self: int(self.desc.n_threads))
    n_blocks = property(lambda self: int(self.desc.n_blocks))

    @property
    def code_len(self) -> np.ndarray:
        return np.frombuffer(bytes(self.desc.code_len), dtype=np.uint8).copy()

    def nbytes(self, which: str) -> int:
        return int(getattr(self.desc, which + "_bytes"))

    @property
    def has_counts(self) -> bool:
        return "counts" in self.arrays

    def compressed_bytes(self) -> int:
        """Bytes the stored format needs: exponent stream, sign/mantissa,
        gaps, block starts and the 256-byte code-length table (the pages'
        arrays; the optional per-thread counts are `counts_bytes()`)."""
        return ((self.total_bits + 7) // 8 + self.n_elems + (5 * self.n_threads + 7) // 8
                + 4 * (self.n_blocks + 1) + 256)

    def counts_bytes(self) -> int:
        """Bytes of the per-thread code counts (one per thread), 0 without them."""
        return self.n_threads if self.has_counts else 0

    def bits_per_weight(self) -> float:
        return 8.0 * self.compressed_bytes() / max(1, self.n_elems)

    def without_counts(self) -> "DF11Tensor":
        """The same tensor without its per-thread counts (shares the arrays):
        decoding it runs the count pass of the two-step kernel."""
        arrays = {k: v for k, v in self.arrays.items() if k != "counts"}
        desc = _Tensor.from_buffer_copy(self.desc)
        desc.counts_bytes = 0
        return DF11Tensor(desc, arrays, self.device, self.shapes, self.offsets, self.tiled)

    def host_array(self, which: str) -> np.ndarray:
        a = self.arrays[which]
        if self.device != "cpu":
            a = a.cpu()
        if not isinstance(a, np.ndarray):
            a = a.numpy()
        return a.view(np.uint32) if which == "block_start" else a.view(np.uint8)

    def _bind(self) -> _Tensor:
        """A new descriptor with the arrays' current addresses."""
        d = _Tensor.from_buffer_copy(self.desc)
        for name in _ARRAYS:
            a = self.arrays.get(name)
            ptr = None if a is None else (a.ctypes.data if isinstance(a, np.ndarray) else a.data_ptr())
            setattr(d, name, ptr)
        return d

    def _desc_for_call(self) -> _Tensor:
        """The descriptor for a library call (the entry points only read it):
        rebuilt only when an array's address or the descriptor changed since
        the last call, so repeated calls on small tensors skip the marshalling."""
        ptrs = tuple(None if a is None else (a.ctypes.data if isinstance(a, np.ndarray) else a.data_ptr())
                     for a in (self.arrays.get(name) for name in _ARRAYS))
        key = (ptrs, bytes(self.desc))
        cached = getattr(self, "_bound", None)
        if cached is None or cached[0] != key:
            d = _Tensor.from_buffer_copy(self.desc)
            for name, ptr in zip(_ARRAYS, ptrs):
                setattr(d, name, ptr)
            cached = (key, d)
            self._bound = cached
        return cached[1]

    def _offsets_c(self):
        """The matrix offsets as a ctypes uint64 array (built once)."""
        key = tuple(self.offsets)
        cached = getattr(self, "_offs_c", None)
        if cached is None or cached[0] != key:
            cached = (key, (ctypes.c_uint64 * len(key))(*key))
            self._offs_c = cached
        return cached[1]

    def to(self, device, non_blocking: bool = False) -> "DF11Tensor":
        """Copies the five arrays to a device (torch tensors, 16-byte aligned)."""
        import torch
        dev = torch.device(device)
        arrays = {}
        for name in self.arrays:
            a = self.arrays[name]
            if isinstance(a, np.ndarray):
                a = torch.from_numpy(a.view(np.uint8))
            b = torch.empty(a.numel() * a.element_size(), dtype=torch.uint8, device=dev)
            b.copy_(a.view(torch.uint8).reshape(-1), non_blocking=non_blocking)
            arrays[name] = b
        return DF11Tensor(_Tensor.from_buffer_copy(self.desc), arrays, str(dev), self.shapes, self.offsets,
                          self.tiled)

    def views(self, decoded):
        """Splits a decoded block buffer into the original matrices (a matrix
        stored in tile order comes back in tile order: see from_tile_order)."""
        out = []
        for shape, lo, hi in zip(self.shapes, self.offsets[:-1], self.offsets[1:]):
            out.append(decoded[lo:hi].view(*shape) if shape else decoded[lo:hi])
        return out


def _alloc_host(nbytes: int, pinned: bool):
    if pinned:
        import torch
        return torch.empty(max(nbytes, 16), dtype=torch.uint8, pin_memory=True)
    # 64-byte aligned numpy buffer
    raw = np.empty(max(nbytes, 16) + 64, dtype=np.uint8)
    off = (-raw.ctypes.data) % 64
    return raw[off: off + max(nbytes, 16)]


def to_tile_order(w) -> np.ndarray:
    """A [rows, cols] BF16 matrix (numpy uint16 bits or a CPU torch tensor;
    rows a multiple of 128, cols of 64) in tile order: its 128 x 64 tiles, row
    tiles in order, the 64-column tiles of a row tile in order, each tile
    row-major (the element order df11_decode_gemm reads).  Flat uint16."""
    a = _as_u16(w)
    shape = tuple(getattr(w, "shape", ()))
    if len(shape) != 2:
        raise ValueError("to_tile_order expects a 2-D matrix")
    out = np.empty(a.size, dtype=np.uint16)
    _check(_lib().df11_to_tile_order(ctypes.c_void_p(a.ctypes.data), int(shape[0]), int(shape[1]),
                                     ctypes.c_void_p(out.ctypes.data)), "to_tile_order")
    return out


def from_tile_order(tiled, rows: int, cols: int) -> np.ndarray:
    """Inverse of to_tile_order: the [rows, cols] row-major matrix (uint16)."""
    a = _as_u16(tiled)
    if a.size != rows * cols:
        raise ValueError("size does not match rows x cols")
    out = np.empty((rows, cols), dtype=np.uint16)
    _check(_lib().df11_from_tile_order(ctypes.c_void_p(a.ctypes.data), int(rows), int(cols),
                                       ctypes.c_void_p(out.ctypes.data)), "from_tile_order")
    return out


def _encode_impl(mats: list[np.ndarray], shapes, params: Params | None, pinned: bool,
                 counts: bool = True, tiled=None) -> DF11Tensor:
    lib = _lib()
    k = len(mats)
    ptrs = (ctypes.POINTER(ctypes.c_uint16) * max(1, k))(*[_u16_ptr(m) for m in mats])
    sizes = (ctypes.c_uint64 * max(1, k))(*[m.size for m in mats])
    desc = _Tensor()
    pc = (params or Params())._c()
    _check(lib.df11_encode_multi_size(ptrs, sizes, k, ctypes.byref(pc), ctypes.byref(desc)), "encode (size)")
    names = _ARRAYS if counts else _ARRAYS[:-1]
    arrays = {name: _alloc_host(int(getattr(desc, name + "_bytes")), pinned) for name in names}
    for name in names:
        a = arrays[name]
        setattr(desc, name, a.ctypes.data if isinstance(a, np.ndarray) else a.data_ptr())
    _check(lib.df11_encode_multi(ptrs, sizes, k, ctypes.byref(desc)), "encode")
    for name in _ARRAYS:
        setattr(desc, name, None)
    if not counts:
        desc.counts_bytes = 0
    offsets = [0]
    for m in mats:
        offsets.append(offsets[-1] + m.size)
    return DF11Tensor(desc, arrays, "cpu", shapes, offsets, tiled)


def encode(w, params: Params | None = None, pinned: bool = False, counts: bool = True) -> DF11Tensor:
    """Host encoder for one BF16 matrix (numpy uint16 bits or a CPU torch
    tensor): histogram, length-limited canonical Huffman code, packing, aux
    (with the optional per-thread code counts unless ``counts`` is False)."""
    shape = tuple(getattr(w, "shape", ()))
    return _encode_impl([_as_u16(w)], [shape], params, pinned, counts)


def encode_multi(mats: Sequence, params: Params | None = None, pinned: bool = False,
                 counts: bool = True, tile_order: bool = False) -> DF11Tensor:
    """Encodes several matrices (a transformer block) as one stream with one
    shared table; ``DF11Tensor.offsets`` gives each matrix's element offset.
    ``tile_order``: every 2-D matrix whose rows are a multiple of 128 and
    columns of 64 is stored in tile order (to_tile_order), as decode_gemm
    needs; ``DF11Tensor.tiled`` records which ones."""
    shapes = [tuple(getattr(m, "shape", ())) for m in mats]
    tiled = [bool(tile_order and len(sh) == 2 and sh[0] % 128 == 0 and sh[1] % 64 == 0) for sh in shapes]
    arrs = [to_tile_order(m) if t else _as_u16(m) for m, t in zip(mats, tiled)]
    return _encode_impl(arrs, shapes, params, pinned, counts, tiled)


def encode_device(mats, params: Params | None = None, stream=None) -> DF11Tensor:
    """Encodes weights already on the GPU (a CUDA BF16 tensor, or a list of
    them encoded as one block with one shared table) with the device encoder;
    returns a device-resident DF11Tensor, byte-identical to what `encode` /
    `encode_multi` produce for the same weights."""
    import torch
    single = isinstance(mats, torch.Tensor)
    mats = [mats] if single else list(mats)
    if not mats:
        raise ValueError("no matrices")
    dev = mats[0].device
    for m in mats:
        if m.device != dev or m.device.type != "cuda" or m.dtype not in (torch.bfloat16, torch.int16):
            raise TypeError("encode_device expects CUDA BF16 tensors on one device")
    shapes = [tuple(m.shape) for m in mats]
    offsets = [0]
    for m in mats:
        offsets.append(offsets[-1] + m.numel())
    n = offsets[-1]
    if single and mats[0].is_contiguous() and mats[0].data_ptr() % 16 == 0:
        flat = mats[0].reshape(-1).view(torch.int16)
    else:  # one buffer for the whole block (device-to-device copies)
        flat = torch.empty(max(n, 8), dtype=torch.int16, device=dev)
        for m, o in zip(mats, offsets):
            flat[o: o + m.numel()].copy_(m.reshape(-1).view(torch.int16))
    lib = _lib()
    sb = int(lib.df11_encode_device_scratch_bytes(n))
    scratch = torch.empty(max(sb, 16), dtype=torch.uint8, device=dev)
    desc = _Tensor()
    pc = (params or Params())._c()
    with _on(dev):
        h = _stream_handle(stream, dev)
        _check(lib.df11_encode_device_size(ctypes.c_void_p(flat.data_ptr()), n, ctypes.byref(pc),
                                           ctypes.byref(desc), ctypes.c_void_p(scratch.data_ptr()), sb, h),
               "encode_device (size)")
        arrays = {name: torch.empty(max(int(getattr(desc, name + "_bytes")), 16), dtype=torch.uint8, device=dev)
                  for name in _ARRAYS}
        for name in _ARRAYS:
            setattr(desc, name, arrays[name].data_ptr())
        _check(lib.df11_encode_device(ctypes.c_void_p(flat.data_ptr()), n, ctypes.byref(desc),
                                      ctypes.c_void_p(scratch.data_ptr()), sb, h), "encode_device")
    for name in _ARRAYS:
        setattr(desc, name, None)
    return DF11Tensor(desc, arrays, str(dev), shapes if not single else [shapes[0]], offsets)


def encode_device_noalloc(w, params: Params | None = None, stream=None) -> DF11Tensor:
    """`encode_device` for one contiguous 16-byte-aligned CUDA BF16 tensor
    through the library's no-allocation entry points: the encoder's scratch
    is a fixed array inside libdf11 (inputs up to
    df11_encode_device_noalloc_max_elems() weights; calls must not overlap on
    a device).  The compressed arrays themselves are still allocated here."""
    import torch
    if not (isinstance(w, torch.Tensor) and w.device.type == "cuda" and w.is_contiguous()
            and w.dtype in (torch.bfloat16, torch.int16)):
        raise TypeError("encode_device_noalloc expects one contiguous CUDA BF16 tensor")
    lib = _lib()
    n = int(w.numel())
    desc = _Tensor()
    pc = (params or Params())._c()
    with _on(w.device):
        h = _stream_handle(stream, w.device)
        _check(lib.df11_encode_device_size_noalloc(ctypes.c_void_p(w.data_ptr()), n, ctypes.byref(pc),
                                                   ctypes.byref(desc), h), "encode_device_noalloc (size)")
        arrays = {name: torch.empty(max(int(getattr(desc, name + "_bytes")), 16), dtype=torch.uint8,
                                    device=w.device) for name in _ARRAYS}
        for name in _ARRAYS:
            setattr(desc, name, arrays[name].data_ptr())
        _check(lib.df11_encode_device_noalloc(ctypes.c_void_p(w.data_ptr()), n, ctypes.byref(desc), h),
               "encode_device_noalloc")
    for name in _ARRAYS:
        setattr(desc, name, None)
    return DF11Tensor(desc, arrays, str(w.device), [tuple(w.shape)], [0, n])


_FILE_MAGIC = b"DF11T002"


def save(t: DF11Tensor, path: str) -> None:
    """Writes a compressed tensor (host or device) to `path` as an .npz
    archive: the descriptor bytes (array pointers cleared), the arrays (the
    per-thread counts when the tensor has them) and the matrix shapes and
    offsets.  Nothing is decoded."""
    desc = _Tensor.from_buffer_copy(t.desc)
    for name in _ARRAYS:
        setattr(desc, name, None)
    arrays = {name: t.host_array(name).view(np.uint8).reshape(-1)[: t.nbytes(name)] for name in t.arrays}
    shapes = np.array([len(s) for s in t.shapes] + [d for s in t.shapes for d in s], dtype=np.int64)
    np.savez(path, magic=np.frombuffer(_FILE_MAGIC, dtype=np.uint8), desc=np.frombuffer(bytes(desc), dtype=np.uint8),
             offsets=np.asarray(t.offsets, dtype=np.int64), shapes=shapes,
             tiled=np.asarray(t.tiled, dtype=np.uint8), **arrays)


def load(path: str, pinned: bool = False) -> DF11Tensor:
    """Reads a tensor written by `save` into host memory (pinned torch
    buffers if `pinned`); the descriptor is checked by df11_validate."""
    with np.load(path) as z:
        if bytes(z["magic"]) != _FILE_MAGIC:
            raise ValueError("not a DF11 tensor file")
        raw = bytes(z["desc"])
        if len(raw) != ctypes.sizeof(_Tensor):
            raise ValueError("descriptor size does not match this library")
        desc = _Tensor.from_buffer_copy(raw)
        arrays = {}
        for name in _ARRAYS:
            if name == "counts" and "counts" not in z.files:
                desc.counts_bytes = 0
                continue
            a = z[name]
            if a.size != int(getattr(desc, name + "_bytes")):
                raise ValueError(f"array {name} has the wrong size")
            buf = _alloc_host(a.size, pinned)
            if pinned:
                import torch
                buf[: a.size].copy_(torch.from_numpy(np.ascontiguousarray(a)))
            else:
                buf[: a.size] = a
            arrays[name] = buf
        offsets = [int(v) for v in z["offsets"]]
        sh = [int(v) for v in z["shapes"]]
        tiled = [bool(v) for v in z["tiled"]] if "tiled" in z.files else None
    k = len(offsets) - 1
    ndims, dims = sh[:k], sh[k:]
    shapes, pos = [], 0
    for nd in ndims:
        shapes.append(tuple(dims[pos: pos + nd]))
        pos += nd
    _check(_lib().df11_validate(ctypes.byref(desc)), "load")
    return DF11Tensor(desc, arrays, "cpu", shapes, offsets, tiled)


def exponent_histogram(mats: Iterable) -> np.ndarray:
    arrs = [_as_u16(m) for m in mats]
    k = len(arrs)
    ptrs = (ctypes.POINTER(ctypes.c_uint16) * max(1, k))(*[_u16_ptr(m) for m in arrs])
    sizes = (ctypes.c_uint64 * max(1, k))(*[m.size for m in arrs])
    out = np.zeros(256, dtype=np.uint64)
    _check(_lib().df11_exponent_histogram(ptrs, sizes, k, out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64))),
           "exponent_histogram")
    return out


def _check_device(t: DF11Tensor):
    if t.device == "cpu":
        raise ValueError("decode needs the compressed arrays on a CUDA device: call .to('cuda') first")


def _new_err(device):
    import torch
    return torch.zeros(1, dtype=torch.int32, device=device)


def decode(t: DF11Tensor, out=None, err=None, stream=None):
    """Decodes a device-resident DF11Tensor into a BF16 tensor (one launch).
    ``err`` (int32[1] device tensor) collects kernel error bits; when it is
    not given, a fresh one is allocated and checked after the launch (which
    synchronises the stream)."""
    import torch
    _check_device(t)
    if out is None:
        out = torch.empty(t.n_elems, dtype=torch.bfloat16, device=t.device)
    own_err = err is None
    if own_err:
        err = _new_err(t.device)
    d = t._desc_for_call()
    with _on(t.device):
        _check(_lib().df11_decode(ctypes.byref(d), ctypes.c_void_p(out.data_ptr()),
                                  ctypes.c_void_p(err.data_ptr()), _stream_handle(stream, t.device)), "decode")
    if own_err:
        read_error(err, stream)
    return out


def decode_block(t: DF11Tensor, scratch=None, err=None, stream=None):
    """Decodes every matrix of a block tensor (from encode_multi) in one
    launch into ``scratch`` (BF16, >= n_elems); ``t.views(scratch)`` returns
    the matrices."""
    import torch
    _check_device(t)
    if scratch is None:
        scratch = torch.empty(t.n_elems, dtype=torch.bfloat16, device=t.device)
    if scratch.numel() < t.n_elems:
        raise ValueError("scratch buffer smaller than the block")
    own_err = err is None
    if own_err:
        err = _new_err(t.device)
    offs = t._offsets_c()
    d = t._desc_for_call()
    with _on(t.device):
        _check(_lib().df11_decode_block(ctypes.byref(d), offs, len(t.offsets) - 1,
                                        ctypes.c_void_p(scratch.data_ptr()),
                                        ctypes.c_void_p(err.data_ptr()), _stream_handle(stream, t.device)),
               "decode_block")
    if own_err:
        read_error(err, stream)
    return scratch


def decode_rows(t: DF11Tensor, row_len: int, rows, out=None, err=None, stream=None):
    """Decodes only the requested rows of a device-resident compressed
    [R, row_len] matrix (an embedding table): out[i] = row rows[i], as a
    [len(rows), row_len] BF16 tensor.  `rows` is an int32 CUDA tensor."""
    import torch
    _check_device(t)
    if rows.dtype not in (torch.int32,) or rows.device.type != "cuda" or rows.dim() != 1:
        raise TypeError("rows must be a 1-D int32 CUDA tensor")
    rows = rows.contiguous()
    n = int(rows.numel())
    if out is None:
        out = torch.empty(n, int(row_len), dtype=torch.bfloat16, device=t.device)
    own_err = err is None
    if own_err:
        err = _new_err(t.device)
    with _on(t.device):
        _check(_lib().df11_decode_rows(ctypes.byref(t._desc_for_call()), int(row_len), ctypes.c_void_p(rows.data_ptr()), n,
                                       ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(err.data_ptr()),
                                       _stream_handle(stream, t.device)), "decode_rows")
    if own_err:
        read_error(err, stream)
    return out


def decode_gemv(t: DF11Tensor, xs: dict, ys: dict | None = None, err=None, stream=None) -> dict:
    """Fused decode and matrix-vector products for batches T <= 4 (one
    launch): for each matrix index j in ``xs`` (indices into ``t.shapes``; a
    2-D [out, in] matrix), y_j = x_j @ W_j^T with W_j decoded on the fly and
    never written to memory.  ``xs[j]``: [T, in] bfloat16 CUDA tensors, one
    T for all.  ``ys[j]`` ([T, out] float32), when given, are added into;
    otherwise zero-filled outputs are allocated.  Returns {j: y_j}."""
    import torch
    _check_device(t)
    if not xs:
        return {}
    order = sorted(xs)
    T = None
    if ys is None:
        ys = {}
    mats = (_GemvMat * len(order))()
    for i, j in enumerate(order):
        shape = t.shapes[j]
        if len(shape) != 2:
            raise ValueError(f"matrix {j} is not 2-D")
        rows, cols = int(shape[0]), int(shape[1])
        x = xs[j]
        if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != cols or not x.is_contiguous():
            raise TypeError(f"x for matrix {j} must be a contiguous [T, {cols}] bfloat16 tensor")
        if T is None:
            T = int(x.shape[0])
        elif int(x.shape[0]) != T:
            raise ValueError("every x must have the same batch T")
        if j not in ys:
            ys[j] = torch.zeros(T, rows, dtype=torch.float32, device=t.device)
        y = ys[j]
        if y.dtype != torch.float32 or tuple(y.shape) != (T, rows) or not y.is_contiguous():
            raise TypeError(f"y for matrix {j} must be a contiguous [{T}, {rows}] float32 tensor")
        mats[i] = _GemvMat(int(t.offsets[j]), rows, cols, x.data_ptr(), y.data_ptr())
    own_err = err is None
    if own_err:
        err = _new_err(t.device)
    with _on(t.device):
        _check(_lib().df11_decode_gemv(ctypes.byref(t._desc_for_call()), mats, len(order), T,
                                       ctypes.c_void_p(err.data_ptr()), _stream_handle(stream, t.device)),
               "decode_gemv")
    if own_err:
        read_error(err, stream)
    return {j: ys[j] for j in order}


def decode_gemm(t: DF11Tensor, xs: dict, ys: dict | None = None, err=None, stream=None) -> dict:
    """Fused decode and tensor-core matrix products for any batch 1..256 (one
    launch): for each matrix index j in ``xs`` (a 2-D [out, in] matrix stored
    in tile order: ``encode_multi(..., tile_order=True)``), y_j = x_j @ W_j^T
    with W_j decoded into shared-memory operand tiles and never written to
    memory.  ``xs[j]``: [T, in] bfloat16 CUDA tensors, one T for all;
    ``ys[j]`` ([T, out] float32), when given, are added into, otherwise
    zero-filled outputs are allocated.  Returns {j: y_j}."""
    import torch
    _check_device(t)
    if not xs:
        return {}
    order = sorted(xs)
    T = None
    if ys is None:
        ys = {}
    mats = (_GemvMat * len(order))()
    for i, j in enumerate(order):
        shape = t.shapes[j]
        if len(shape) != 2 or not t.tiled[j]:
            raise ValueError(f"matrix {j} is not a 2-D matrix stored in tile order")
        rows, cols = int(shape[0]), int(shape[1])
        x = xs[j]
        if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != cols or not x.is_contiguous():
            raise TypeError(f"x for matrix {j} must be a contiguous [T, {cols}] bfloat16 tensor")
        if T is None:
            T = int(x.shape[0])
        elif int(x.shape[0]) != T:
            raise ValueError("every x must have the same batch T")
        if j not in ys:
            ys[j] = torch.zeros(T, rows, dtype=torch.float32, device=t.device)
        y = ys[j]
        if y.dtype != torch.float32 or tuple(y.shape) != (T, rows) or not y.is_contiguous():
            raise TypeError(f"y for matrix {j} must be a contiguous [{T}, {rows}] float32 tensor")
        mats[i] = _GemvMat(int(t.offsets[j]), rows, cols, x.data_ptr(), y.data_ptr())
    own_err = err is None
    if own_err:
        err = _new_err(t.device)
    with _on(t.device):
        _check(_lib().df11_decode_gemm(ctypes.byref(t._desc_for_call()), mats, len(order), T,
                                       ctypes.c_void_p(err.data_ptr()), _stream_handle(stream, t.device)),
               "decode_gemm")
    if own_err:
        read_error(err, stream)
    return {j: ys[j] for j in order}


def gemm(x, w, out=None, err=None, stream=None):
    """Y = X @ W^T on the tensor cores: x [T, in] and w [out, in] BF16 CUDA
    tensors (w may be a view of a decoded block), FP32 result [T, out]."""
    import torch
    if x.dtype != torch.bfloat16 or w.dtype != torch.bfloat16 or x.dim() != 2 or w.dim() != 2:
        raise TypeError("gemm expects 2-D bfloat16 tensors")
    if not x.is_contiguous() or not w.is_contiguous():
        raise ValueError("gemm expects contiguous tensors")
    T, k = x.shape
    n, k2 = w.shape
    if k != k2:
        raise ValueError("inner dimensions differ")
    if out is None:
        out = torch.empty(T, n, dtype=torch.float32, device=x.device)
    own_err = err is None
    if own_err:
        err = _new_err(x.device)
    if x.device != w.device or out.device != x.device:
        raise ValueError("gemm expects x, w and out on one device")
    with _on(x.device):
        _check(_lib().df11_gemm_bf16(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                     ctypes.c_void_p(out.data_ptr()), T, n, k, ctypes.c_void_p(err.data_ptr()),
                                     _stream_handle(stream, x.device)), "gemm")
    if own_err:
        read_error(err, stream)
    return out


def gemm_multi(pairs, outs=None, err=None, stream=None):
    """Several products Y_j = X_j @ W_j^T in one call (one persistent
    tensor-core launch for T > 4): ``pairs`` is a list of (x [T, in_j],
    w [out_j, in_j]) BF16 CUDA tensors with one T; returns the FP32 results
    [T, out_j] (written into ``outs`` when given)."""
    import torch
    if not pairs:
        return []
    dev = pairs[0][0].device
    T = int(pairs[0][0].shape[0])
    if outs is None:
        outs = [torch.empty(T, w.shape[0], dtype=torch.float32, device=dev) for _, w in pairs]
    if len(outs) != len(pairs):
        raise ValueError("one output per product")
    mats = (_GemmMat * len(pairs))()
    for k, ((x, w), y) in enumerate(zip(pairs, outs)):
        if x.dtype != torch.bfloat16 or w.dtype != torch.bfloat16 or x.dim() != 2 or w.dim() != 2:
            raise TypeError("gemm_multi expects 2-D bfloat16 tensors")
        if not x.is_contiguous() or not w.is_contiguous() or not y.is_contiguous():
            raise ValueError("gemm_multi expects contiguous tensors")
        if x.shape[0] != T or x.shape[1] != w.shape[1] or tuple(y.shape) != (T, w.shape[0]):
            raise ValueError("shapes do not match")
        if y.dtype != torch.float32 or x.device != dev or w.device != dev or y.device != dev:
            raise ValueError("gemm_multi expects FP32 outputs and one device")
        mats[k] = _GemmMat(x.data_ptr(), w.data_ptr(), y.data_ptr(), int(w.shape[0]), int(w.shape[1]))
    own_err = err is None
    if own_err:
        err = _new_err(dev)
    with _on(dev):
        _check(_lib().df11_gemm_bf16_multi(mats, len(pairs), T, ctypes.c_void_p(err.data_ptr()),
                                           _stream_handle(stream, dev)), "gemm_multi")
    if own_err:
        read_error(err, stream)
    return outs


def read_error(err, stream=None) -> int:
    """Reads the kernel error word (synchronises the stream); raises
    CorruptStreamError if any bit is set."""
    v = ctypes.c_uint32(0)
    with _on(err.device):
        st = _lib().df11_read_error(ctypes.c_void_p(err.data_ptr()), _stream_handle(stream, err.device),
                                    ctypes.byref(v))
    if st == 4:
        raise CorruptStreamError(4, f"decode kernel reported error bits 0x{v.value:x}")
    _check(st, "read_error")
    return int(v.value)


def sm_count() -> int:
    v = ctypes.c_int(0)
    _check(_lib().df11_device_sm_count(ctypes.byref(v)), "sm_count")
    return int(v.value)
