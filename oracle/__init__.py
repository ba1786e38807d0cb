"""The oracle: a plain, slow, obviously correct CPU implementation of the
DFloat11 exponent codec, used to check the GPU library.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg may import this package.  The
product library never imports it, and it never imports the product library:
the two share no code.  The arithmetic lives in ``df11_oracle.c`` (plain C,
one bit at a time); this module only builds it with gcc and marshals numpy
arrays in and out.

Functions (each cites its passage in ``df11_oracle.c``):

* ``histogram(w)`` -- exponent counts.
* ``huffman_lengths(count)`` -- plain Huffman code lengths (no cap).
* ``package_merge_lengths(count, cap)`` -- optimal lengths with every
  length <= cap.
* ``canonical_codes(lengths)`` -- canonical code values.
* ``encode(w, lengths)`` -- (enc bytes, sign/mantissa bytes, total bits).
* ``decode(enc, total_bits, sm, n, lengths)`` -- bit-serial tree walk;
  ``decode_range(enc, first_bit, end_bit, sm, n, lengths)`` -- the same on
  one piece of a stream (a run of whole thread blocks).
* ``aux(enc, total_bits, n, lengths, bytes_per_thread, threads_per_block)``
  -- gaps, per-thread counts and block starts recomputed from a stream.
* ``pack_gaps(gaps)`` -- 5-bit packing of gaps.
* ``exponent_stats(count, lengths)`` -- entropy, distinct values, mean length.
* ``kraft_sum_2p32(lengths)``, ``is_prefix_free(lengths)`` (the canonical
  code of the lengths), ``codes_prefix_free(codes, lengths)`` (an explicit
  code set).

Parity: pinned by the ``-m "not gpu"`` tests in ``tests/test_oracle.py``
(identity on every input, brute-force optimality, closed forms, textbook
examples under ``tests/golden/``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "df11_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")

ORC_OK = 0
ORC_ERR_ARG = -1
ORC_ERR_CAP = -2
ORC_ERR_CORRUPT = -3
ORC_ERR_NOMEM = -4
ORC_ERR_NOT_PREFIX_FREE = -5


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no vectorisation flags)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-Wall", "-Wextra", "-shared", "-fPIC",
                           "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_u64p = ctypes.POINTER(ctypes.c_uint64)


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    u64, i32 = ctypes.c_uint64, ctypes.c_int
    lib.orc_histogram.argtypes = [_u16p, u64, _u64p]
    lib.orc_exponent_stats.argtypes = [_u64p, _u8p, ctypes.POINTER(ctypes.c_double),
                                       ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double)]
    lib.orc_exponent_stats.restype = None
    lib.orc_huffman_lengths.argtypes = [_u64p, _u8p]
    lib.orc_package_merge_lengths.argtypes = [_u64p, i32, _u8p]
    lib.orc_canonical_codes.argtypes = [_u8p, _u32p]
    lib.orc_kraft_sum_2p32.argtypes = [_u8p]
    lib.orc_kraft_sum_2p32.restype = u64
    lib.orc_total_bits.argtypes = [_u16p, u64, _u8p]
    lib.orc_total_bits.restype = u64
    lib.orc_encode.argtypes = [_u16p, u64, _u8p, _u8p, u64, _u8p, _u64p]
    lib.orc_is_prefix_free.argtypes = [_u8p]
    lib.orc_codes_prefix_free.argtypes = [_u32p, _u8p]
    lib.orc_decode.argtypes = [_u8p, u64, _u8p, u64, _u8p, _u16p]
    lib.orc_decode_range.argtypes = [_u8p, u64, u64, _u8p, u64, _u8p, _u16p]
    lib.orc_aux.argtypes = [_u8p, u64, u64, _u8p, ctypes.c_uint32, ctypes.c_uint32,
                            _u8p, _u32p, _u32p, _u64p, _u64p]
    lib.orc_pack_gaps.argtypes = [_u8p, u64, _u8p, u64]
    lib.orc_pack_gaps.restype = None
    lib.orc_read_gap.argtypes = [_u8p, u64]
    lib.orc_read_gap.restype = ctypes.c_uint
    _lib = lib
    return lib


def _ptr(a: np.ndarray, ty):
    return a.ctypes.data_as(ty)


def _u16(w) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(w)).reshape(-1)
    if a.dtype != np.uint16:
        a = a.view(np.uint16) if a.dtype.itemsize == 2 else a.astype(np.uint16)
    return a


def _check(rc: int, what: str) -> None:
    if rc != ORC_OK:
        raise OracleError(f"{what} failed with status {rc}")


def histogram(w) -> np.ndarray:
    a = _u16(w)
    count = np.zeros(256, dtype=np.uint64)
    _check(_load().orc_histogram(_ptr(a, _u16p), a.size, _ptr(count, _u64p)), "histogram")
    return count


def exponent_stats(count: np.ndarray, lengths: np.ndarray | None = None):
    """(entropy bits, distinct exponent values, mean code length)."""
    c = np.ascontiguousarray(count, dtype=np.uint64)
    h = ctypes.c_double()
    k = ctypes.c_int()
    m = ctypes.c_double()
    lp = _ptr(np.ascontiguousarray(lengths, dtype=np.uint8), _u8p) if lengths is not None else None
    _load().orc_exponent_stats(_ptr(c, _u64p), lp, ctypes.byref(h), ctypes.byref(k), ctypes.byref(m))
    return h.value, k.value, m.value


def huffman_lengths(count) -> np.ndarray:
    c = np.ascontiguousarray(count, dtype=np.uint64)
    out = np.zeros(256, dtype=np.uint8)
    _check(_load().orc_huffman_lengths(_ptr(c, _u64p), _ptr(out, _u8p)), "huffman_lengths")
    return out


def package_merge_lengths(count, cap: int = 32) -> np.ndarray:
    c = np.ascontiguousarray(count, dtype=np.uint64)
    out = np.zeros(256, dtype=np.uint8)
    _check(_load().orc_package_merge_lengths(_ptr(c, _u64p), int(cap), _ptr(out, _u8p)),
           "package_merge_lengths")
    return out


def canonical_codes(lengths) -> np.ndarray:
    l8 = np.ascontiguousarray(lengths, dtype=np.uint8)
    out = np.zeros(256, dtype=np.uint32)
    _check(_load().orc_canonical_codes(_ptr(l8, _u8p), _ptr(out, _u32p)), "canonical_codes")
    return out


def kraft_sum_2p32(lengths) -> int:
    l8 = np.ascontiguousarray(lengths, dtype=np.uint8)
    return int(_load().orc_kraft_sum_2p32(_ptr(l8, _u8p)))


def is_prefix_free(lengths) -> bool:
    l8 = np.ascontiguousarray(lengths, dtype=np.uint8)
    return bool(_load().orc_is_prefix_free(_ptr(l8, _u8p)))


def codes_prefix_free(codes, lengths) -> bool:
    """Tree-insertion check of an explicit code set: codes[s] holds
    lengths[s] bits (most significant first); lengths[s] == 0 means no code."""
    c32 = np.zeros(256, dtype=np.uint32)
    l8 = np.zeros(256, dtype=np.uint8)
    c = np.asarray(codes, dtype=np.uint64).reshape(-1)
    ln = np.asarray(lengths, dtype=np.int64).reshape(-1)
    c32[: c.size] = c.astype(np.uint32)
    l8[: ln.size] = ln.astype(np.uint8)
    return bool(_load().orc_codes_prefix_free(_ptr(c32, _u32p), _ptr(l8, _u8p)))


def total_bits(w, lengths) -> int:
    a = _u16(w)
    l8 = np.ascontiguousarray(lengths, dtype=np.uint8)
    return int(_load().orc_total_bits(_ptr(a, _u16p), a.size, _ptr(l8, _u8p)))


def encode(w, lengths):
    """Returns (enc: uint8[ceil(bits/8)], sm: uint8[n], total_bits)."""
    a = _u16(w)
    l8 = np.ascontiguousarray(lengths, dtype=np.uint8)
    bits = total_bits(a, l8)
    enc = np.zeros(max(1, (bits + 7) // 8), dtype=np.uint8)
    sm = np.zeros(max(1, a.size), dtype=np.uint8)
    tb = ctypes.c_uint64()
    _check(_load().orc_encode(_ptr(a, _u16p), a.size, _ptr(l8, _u8p), _ptr(enc, _u8p), enc.size,
                              _ptr(sm, _u8p), ctypes.byref(tb)), "encode")
    return enc[: (bits + 7) // 8], sm[: a.size], int(tb.value)


def decode(enc, total_bits_: int, sm, n: int, lengths) -> np.ndarray:
    e = np.ascontiguousarray(enc, dtype=np.uint8)
    s = np.ascontiguousarray(sm, dtype=np.uint8)
    l8 = np.ascontiguousarray(lengths, dtype=np.uint8)
    if e.size == 0:
        e = np.zeros(1, dtype=np.uint8)
    if s.size == 0:
        s = np.zeros(1, dtype=np.uint8)
    out = np.zeros(max(1, n), dtype=np.uint16)
    _check(_load().orc_decode(_ptr(e, _u8p), int(total_bits_), _ptr(s, _u8p), int(n),
                              _ptr(l8, _u8p), _ptr(out, _u16p)), "decode")
    return out[:n]


def decode_range(enc, first_bit: int, end_bit: int, sm, n: int, lengths, out=None) -> np.ndarray:
    """Decodes the n weights whose codes fill bits [first_bit, end_bit) of
    ``enc``; ``sm`` holds those n weights' sign/mantissa bytes.  Writes into
    ``out`` (uint16[n]) when given.  Releases the GIL while it runs (ctypes),
    so pieces of one stream can be decoded on several host threads."""
    e = np.ascontiguousarray(enc, dtype=np.uint8)
    s = np.ascontiguousarray(sm, dtype=np.uint8)
    l8 = np.ascontiguousarray(lengths, dtype=np.uint8)
    if e.size == 0:
        e = np.zeros(1, dtype=np.uint8)
    if s.size == 0:
        s = np.zeros(1, dtype=np.uint8)
    if out is None:
        out = np.zeros(max(1, n), dtype=np.uint16)
    _check(_load().orc_decode_range(_ptr(e, _u8p), int(first_bit), int(end_bit), _ptr(s, _u8p), int(n),
                                    _ptr(l8, _u8p), _ptr(out, _u16p)), "decode_range")
    return out[:n]


def aux(enc, total_bits_: int, n: int, lengths, bytes_per_thread: int = 8,
        threads_per_block: int = 256):
    """Returns dict(gaps=uint8[n_blocks*T], counts=uint32[n_blocks*T],
    block_start=uint32[n_blocks+1], n_threads, n_blocks)."""
    lib = _load()
    e = np.ascontiguousarray(enc, dtype=np.uint8)
    if e.size == 0:
        e = np.zeros(1, dtype=np.uint8)
    l8 = np.ascontiguousarray(lengths, dtype=np.uint8)
    nt = ctypes.c_uint64()
    nb = ctypes.c_uint64()
    lib.orc_aux(_ptr(e, _u8p), int(total_bits_), int(n), _ptr(l8, _u8p), bytes_per_thread,
                threads_per_block, None, None, None, ctypes.byref(nt), ctypes.byref(nb))
    padded = nb.value * threads_per_block
    gaps = np.zeros(max(1, padded), dtype=np.uint8)
    counts = np.zeros(max(1, padded), dtype=np.uint32)
    bstart = np.zeros(nb.value + 1, dtype=np.uint32)
    _check(lib.orc_aux(_ptr(e, _u8p), int(total_bits_), int(n), _ptr(l8, _u8p), bytes_per_thread,
                       threads_per_block, _ptr(gaps, _u8p), _ptr(counts, _u32p), _ptr(bstart, _u32p),
                       ctypes.byref(nt), ctypes.byref(nb)), "aux")
    return dict(gaps=gaps[:padded], counts=counts[:padded], block_start=bstart,
                n_threads=int(nt.value), n_blocks=int(nb.value))


def pack_gaps(gaps) -> np.ndarray:
    g = np.ascontiguousarray(gaps, dtype=np.uint8)
    nbytes = (5 * g.size + 7) // 8
    out = np.zeros(max(1, nbytes), dtype=np.uint8)
    gp = g if g.size else np.zeros(1, dtype=np.uint8)
    _load().orc_pack_gaps(_ptr(gp, _u8p), g.size, _ptr(out, _u8p), out.size)
    return out[:nbytes]


def read_gap(packed, t: int) -> int:
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    return int(_load().orc_read_gap(_ptr(p, _u8p), int(t)))


def compress(w, cap: int = 32):
    """Convenience: histogram -> package-merge lengths -> encode -> aux.
    Returns a dict with every array the oracle computes for ``w``."""
    a = _u16(w)
    count = histogram(a)
    lengths = package_merge_lengths(count, cap)
    enc, sm, bits = encode(a, lengths)
    return dict(count=count, lengths=lengths, enc=enc, sm=sm, total_bits=bits, n=a.size)
