"""Host-side checks of libdf11 (no GPU): the C ABI loads and exports every
declared call; the product encoder's output is checked against the oracle
(optimal cost, byte-exact stream for the product's own code, aux recomputed
from the stream); the decode tables are exercised by a CPU walk that mirrors
the kernel's lookup rule."""
import ctypes
import os
import re
import struct

import numpy as np
import pytest

import huffman_decode_02_b200 as df11
import oracle
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "df11.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(df11_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(df11.lib_path())
    names = _header_functions()
    assert len(names) >= 14
    for name in names:
        assert hasattr(lib, name), name
    assert df11._lib().df11_abi_version() == 3


def test_status_strings():
    lib = df11._lib()
    assert lib.df11_status_str(0) == b"ok"
    assert b"corrupt" in lib.df11_status_str(4)


def _cost(count, lengths):
    return int(np.dot(np.asarray(count, dtype=np.int64), np.asarray(lengths, dtype=np.int64)))


def _unpack_gaps(packed: np.ndarray, n: int) -> np.ndarray:
    bits = np.unpackbits(packed)[: 5 * n].reshape(n, 5)
    return (bits * np.array([16, 8, 4, 2, 1], dtype=np.uint8)).sum(axis=1).astype(np.uint8)


CASES = ["all_bf16_patterns", "all_zero", "all_equal", "two_values", "random_u16",
         "neg_zero_and_nan", "single", "empty", "subnormals", "ragged_normal",
         "uniform_exponents", "fibonacci_exponents"]


def check_against_oracle(w, t, cap=12):
    w = np.ascontiguousarray(w).reshape(-1).view(np.uint16)
    count = oracle.histogram(w)
    assert np.array_equal(df11.exponent_histogram([w]), count)
    lengths = t.code_len
    k = int(np.count_nonzero(count))
    # only exponents that occur get a code; cost is optimal under the cap
    assert np.array_equal(lengths > 0, count > 0)
    assert lengths.max(initial=0) <= cap
    if k:
        assert _cost(count, lengths) == _cost(count, oracle.package_merge_lengths(count, cap))
        assert oracle.is_prefix_free(lengths)
        assert oracle.kraft_sum_2p32(lengths) == (1 << 32 if k >= 2 else 1 << 31)
    assert t.total_bits == _cost(count, lengths)
    # the stream is exactly the oracle's encoding with the product's lengths
    enc_o, sm_o, bits_o = oracle.encode(w, lengths)
    enc = t.host_array("enc")
    assert bits_o == t.total_bits
    assert np.array_equal(enc[: enc_o.size], enc_o)
    assert not enc[enc_o.size:].any()
    sm = t.host_array("sm")
    assert np.array_equal(sm[: w.size], sm_o[: w.size])
    assert not sm[w.size:].any()
    # aux recomputed from the stream by the oracle's bit-serial walk
    a = oracle.aux(enc_o, bits_o, w.size, lengths, 8, 256)
    assert a["n_threads"] == t.n_threads and a["n_blocks"] == t.n_blocks
    assert np.array_equal(t.host_array("block_start")[: t.n_blocks + 1], a["block_start"])
    assert t.desc.max_block_codes == (int(np.diff(a["block_start"]).max()) if t.n_blocks else 0)
    packed = t.host_array("gaps")
    n_fields = t.n_blocks * 256
    assert np.array_equal(_unpack_gaps(packed, n_fields), a["gaps"])
    assert np.array_equal(packed[: (5 * n_fields + 7) // 8], oracle.pack_gaps(a["gaps"]))
    # the optional per-thread code counts: the oracle's counts of code starts
    if t.has_counts:
        cnt = t.host_array("counts")
        assert t.nbytes("counts") == n_fields + 16
        assert np.array_equal(cnt[:n_fields], a["counts"].astype(np.uint8))
        assert a["counts"].max(initial=0) <= 64
        assert not cnt[n_fields:].any()
    # and the oracle decodes the product's stream back to the input
    out = oracle.decode(enc_o, bits_o, sm_o, w.size, lengths)
    assert np.array_equal(out, w)


@pytest.mark.parametrize("name", CASES)
def test_encoder_matches_oracle_adversarial(name):
    w = workloads.adversarial(name)
    t = df11.encode(w)
    check_against_oracle(w, t)


@pytest.mark.parametrize("cap", [8, 12, 20])
def test_encoder_length_cap(cap):
    w = workloads.adversarial("fibonacci_exponents")
    t = df11.encode(w, df11.Params(max_code_len=cap))
    check_against_oracle(w, t, cap)
    assert t.code_len.max() == cap


def test_encoder_normal_matrix_small():
    w = workloads.normal_matrix(512, 384, 0.02, seed=0)
    t = df11.encode(w)
    check_against_oracle(w, t)
    assert 9.5 < t.bits_per_weight() < 11.5
    t32 = df11.encode(w, df11.Params(max_code_len=32))
    check_against_oracle(w, t32, cap=32)
    # the default 12-bit cap costs almost nothing on weight-like data
    assert t.total_bits - t32.total_bits < 0.002 * t32.total_bits


def test_encoder_multichunk_boundaries():
    """Longer than the host chunk (2^20 elements), so chunk seams are hit."""
    w = workloads.adversarial("ragged_normal")
    w = np.concatenate([w, w[:1_000_001]])
    t = df11.encode(w)
    check_against_oracle(w, t)


def test_encode_multi_equals_concatenation():
    mats = [workloads.normal_matrix(r, c, s, seed=i) for i, (r, c, s) in
            enumerate([(64, 96, 0.02), (3, 5, 0.05), (128, 64, 0.01), (1, 1, 1.0)])]
    blk = df11.encode_multi(mats)
    cat = df11.encode(np.concatenate([m.reshape(-1) for m in mats]))
    for name in ("enc", "sm", "gaps", "block_start", "lut", "counts"):
        assert np.array_equal(blk.host_array(name), cat.host_array(name)), name
    assert blk.offsets == [0, 64 * 96, 64 * 96 + 15, 64 * 96 + 15 + 128 * 64, 64 * 96 + 15 + 128 * 64 + 1]


def test_invalid_params_rejected():
    w = workloads.normal_matrix(8, 8, 0.02, seed=0)
    with pytest.raises(df11.DF11Error):
        df11.encode(w, df11.Params(bytes_per_thread=4))
    with pytest.raises(df11.DF11Error):
        df11.encode(w, df11.Params(max_code_len=0))
    full = workloads.adversarial("uniform_exponents")  # 256 symbols need >= 8 bits
    with pytest.raises(df11.DF11Error):
        df11.encode(full, df11.Params(max_code_len=7))


# ------------------------------------------------ decode-table walk on CPU

def _lut_fields(lut: np.ndarray):
    b = lut.tobytes()
    magic, w1, w2, max_len, min_len, n_syms, w1_max, w2_max = struct.unpack_from("<8I", b, 0)
    lim = np.frombuffer(b, dtype=np.uint64, count=33, offset=64)
    offs = np.frombuffer(b, dtype=np.uint32, count=33, offset=336)
    symrot = lut[480:736]
    assert len(b) == 768 + 4 * (1 << w1_max) + 8 * (1 << w2_max)
    clut = np.frombuffer(b, dtype=np.uint32, count=1 << w1_max, offset=768)
    slut = np.frombuffer(b, dtype=np.uint32, count=2 << w2_max, offset=768 + 4 * (1 << w1_max)).reshape(-1, 2)
    return dict(magic=magic, w1=w1, w2=w2, max_len=max_len, lim=lim, offs=offs, symrot=symrot,
                clut=clut, slut=slut)


def _unrotate(r):
    return ((r << 1) | (r >> 7)) & 0xFF


ESC = 0x80000000


def _walk(t):
    """Decodes every thread's range with the product's tables, using the
    kernel's rules: bits at/after the thread's end are ones; the count pass
    adds whole entries into one accumulator (bits taken in the top byte,
    codes in bits 8..23) and leaves its loop on the escape flag or once the
    bits reach the thread's span; the decode pass stops on the code count.
    Returns (exponents in element order, per-thread counts)."""
    f = _lut_fields(t.host_array("lut"))
    assert f["magic"] == 0x33314644
    enc = t.host_array("enc")
    bits_all = np.unpackbits(enc)
    gaps = _unpack_gaps(t.host_array("gaps"), t.n_blocks * 256 + 1) if t.n_blocks else np.zeros(1, np.uint8)

    def win(window, pos, n):
        return int("".join(map(str, window[pos:pos + n])), 2)

    def long_len(x, lo):
        return next(l for l in range(lo, f["max_len"] + 1) if x < int(f["lim"][l]))

    out, counts = [], []
    for th in range(t.n_threads):
        gap = int(gaps[th])
        end = t.total_bits - 64 * th if th == t.n_threads - 1 else 64 + int(gaps[th + 1])
        window = np.ones(96 + 64, dtype=np.uint8)
        seg = bits_all[64 * th: 64 * th + 96]
        window[: min(96, seg.size)] = seg
        window[end:] = 1
        rem0 = end - gap
        # pass 1 (count table)
        pos, acc, lim = gap, 0, rem0 << 24
        while True:
            while acc < lim:
                e = int(f["clut"][win(window, pos, f["w1"])])
                acc += e
                pos += e & 31
            if acc < ESC:
                break
            acc -= ESC
            l = long_len(win(window, pos, 32), f["w1"] + 1)
            acc += (l << 24) | (1 << 8)
            pos += l
        n1 = (acc >> 8) & 0xFFFF
        assert pos == end and (acc >> 24) == rem0
        # pass 2 (symbol table), stops after n1 codes
        pos, syms = gap, []
        while len(syms) < n1:
            s_, m = (int(x) for x in f["slut"][win(window, pos, f["w2"])])
            if m == ESC:
                x = win(window, pos, 32)
                l = long_len(x, f["w2"] + 1)
                syms.append(int(f["symrot"][((x >> (32 - l)) + int(f["offs"][l])) & 0xFFFFFFFF & 255]))
                pos += l
            else:
                nc = (m >> 8) & 0xFF
                assert 1 <= nc <= 4
                syms.extend([(s_ >> (8 * j)) & 0xFF for j in range(nc)])
                pos += m & 31
        assert pos == end and len(syms) == n1
        out.extend(_unrotate(np.array(syms, dtype=np.uint32)).tolist())
        counts.append(n1)
    return np.array(out, dtype=np.uint32), np.array(counts)


@pytest.mark.parametrize("name", ["neg_zero_and_nan", "two_values", "all_equal", "fibonacci_small",
                                  "normal_small", "uniform_small", "long_codes"])
def test_table_walk_reproduces_exponents(name):
    rng = np.random.default_rng(9)
    if name == "fibonacci_small":
        w = workloads.adversarial("fibonacci_exponents")[:30_000]
    elif name == "normal_small":
        w = workloads.normal_matrix(100, 211, 0.02, seed=4).reshape(-1)
    elif name == "uniform_small":
        w = workloads.adversarial("uniform_exponents")[:6000]
    elif name == "long_codes":
        # exponents with geometric frequencies: long codes (> 14 bits) occur
        e = np.minimum(rng.geometric(0.45, size=40_000), 30) + 90
        w = ((e << 7) | rng.integers(0, 128, e.size)).astype(np.uint16)
    else:
        w = workloads.adversarial(name)[:20_000]
    t = df11.encode(w, df11.Params(max_code_len=32))
    expo, counts = _walk(t)
    assert np.array_equal(expo, (w.reshape(-1) >> 7) & 0xFF)
    bs = t.host_array("block_start")
    per_block = np.add.reduceat(np.concatenate([counts, np.zeros(t.n_blocks * 256 - counts.size, int)]),
                                np.arange(0, t.n_blocks * 256, 256)) if t.n_blocks else []
    assert np.array_equal(np.diff(bs[: t.n_blocks + 1]), per_block)
    if name == "long_codes":
        assert t.code_len.max() > 14


def test_save_load_round_trip(tmp_path):
    """A compressed block written and read back: identical descriptor and
    arrays, same matrix shapes and offsets, and the oracle decodes the loaded
    stream to the original weights."""
    mats = [workloads.normal_matrix(64, 48, 0.02, seed=3), workloads.normal_matrix(5, 7, 0.5, seed=4)]
    t = df11.encode_multi(mats)
    path = str(tmp_path / "blk.npz")
    df11.save(t, path)
    u = df11.load(path)
    assert bytes(u.desc)[:8] == bytes(t.desc)[:8] and u.n_elems == t.n_elems and u.total_bits == t.total_bits
    assert u.shapes == [(64, 48), (5, 7)] and u.offsets == t.offsets
    assert u.has_counts
    for k in ("enc", "sm", "gaps", "block_start", "lut", "counts"):
        np.testing.assert_array_equal(u.host_array(k).view(np.uint8)[: u.nbytes(k)],
                                      t.host_array(k).view(np.uint8)[: t.nbytes(k)])
    out = oracle.decode(u.host_array("enc"), u.total_bits, u.host_array("sm"), u.n_elems, u.code_len)
    np.testing.assert_array_equal(out, np.concatenate([m.reshape(-1) for m in mats]))
    with open(path, "r+b") as f:  # a damaged file is refused
        f.seek(0)
        f.write(b"\0" * 16)
    with pytest.raises(Exception):
        df11.load(path)


def test_concurrent_host_encodes_match_sequential():
    """Encodes from several host threads at once (the library keeps no shared
    mutable state) give the same arrays as one after another."""
    import threading
    mats = [workloads.normal_matrix(300 + 37 * i, 211, 0.02 + 0.005 * i, seed=50 + i) for i in range(4)]
    seq = [df11.encode(m) for m in mats]
    got = [None] * len(mats)

    def run(i):
        got[i] = df11.encode(mats[i])

    threads = [threading.Thread(target=run, args=(i,)) for i in range(len(mats))]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    for a, b in zip(seq, got):
        assert a.total_bits == b.total_bits and a.n_blocks == b.n_blocks
        for k in ("enc", "sm", "gaps", "block_start", "lut", "counts"):
            np.testing.assert_array_equal(a.host_array(k)[: a.nbytes(k)], b.host_array(k)[: b.nbytes(k)])


def _aligned_copy(a: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """A 16-byte aligned copy of a's bytes (returns the view and its owner)."""
    raw = a.view(np.uint8).reshape(-1)
    buf = np.zeros(raw.size + 32, dtype=np.uint8)
    k = (-buf.ctypes.data) % 16
    view = buf[k: k + raw.size]
    view[:] = raw
    return view, buf


def test_decode_gemv_argument_checks():
    """df11_decode_gemv rejects bad calls before any GPU work (so these run
    without a GPU): batch outside 1..4 and more than 16 matrices are
    unsupported; misaligned, overlapping, out-of-order or out-of-range
    matrices and NULL vectors are invalid arguments; no matrices is a no-op."""
    lib = df11._lib()
    mats = [workloads.normal_matrix(64, 32, 0.02, seed=1), workloads.normal_matrix(32, 64, 0.02, seed=2)]
    t = df11.encode_multi(mats)
    d = t._bind()
    keep = []
    for name in ("enc", "sm", "gaps", "block_start", "lut"):
        v, owner = _aligned_copy(t.host_array(name))
        keep.append(owner)
        setattr(d, name, v.ctypes.data)
    xbuf, xown = _aligned_copy(np.zeros(4 * 64 + 8, dtype=np.uint16))
    ybuf = np.zeros(4 * 64 + 4, dtype=np.float32)
    X, Y = xbuf.ctypes.data, ybuf.ctypes.data

    def call(descs, T=1, n=None):
        arr = (df11._GemvMat * max(1, len(descs)))(*[df11._GemvMat(*m) for m in descs])
        return lib.df11_decode_gemv(ctypes.byref(d), arr, len(descs) if n is None else n, T, None, None)

    good = [(0, 64, 32, X, Y), (2048, 32, 64, X, Y)]
    assert call(good, n=0) == 0
    assert call(good, T=0) == 2 and call(good, T=5) == 2
    assert call([(0, 1, 16, X, Y)] * 17) == 2
    assert call([(8, 64, 32, X, Y)]) == 1                      # offset not a multiple of 16
    assert call([(0, 64, 24, X, Y)]) == 1                      # cols not a multiple of 16
    assert call([(0, 0, 32, X, Y)]) == 1                       # no rows
    assert call([(0, 64, 32, None, Y)]) == 1                   # NULL x
    assert call([(0, 64, 32, X, None)]) == 1                   # NULL y
    assert call([(0, 64, 32, X + 2, Y)]) == 1                  # x not 16-byte aligned
    assert call([(0, 64, 32, X, Y + 2)]) == 1                  # y not 4-byte aligned
    assert call([good[1], good[0]]) == 1                       # out of order
    assert call([(0, 64, 32, X, Y), (2032, 32, 64, X, Y)]) == 1  # overlapping
    assert call([(2048, 33, 64, X, Y)]) == 1                   # past the tensor's end
    assert call([(0, 0xFFFFFFFF, 0xFFFFFFF0, X, Y)]) == 1      # size far past the end
    del keep, xown


def test_header_compiles_as_plain_c(tmp_path):
    """include/df11.h is a C ABI: it compiles as C99 with -pedantic -Werror
    and every struct the calls take can be declared from C."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_df11.c"
    src.write_text('#include "df11.h"\n'
                   "int main(void) {\n"
                   "    df11_params p; df11_tensor t; df11_gemv_mat m;\n"
                   "    (void)p; (void)t; (void)m;\n"
                   "    return 0;\n"
                   "}\n")
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                        os.path.join(ROOT, "include"), "-c", str(src), "-o", str(tmp_path / "use_df11.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_tile_order_round_trip_and_layout():
    """Tile order against an independent numpy route: the [rows, cols] matrix
    as [rows/128, 128, cols/64, 64], axes (0, 2, 1, 3), flattened; and the
    inverse restores the matrix."""
    w = workloads.normal_matrix(384, 192, 0.02, seed=31)
    t = df11.to_tile_order(w)
    ref = w.reshape(3, 128, 3, 64).transpose(0, 2, 1, 3).reshape(-1)
    np.testing.assert_array_equal(t, ref)
    np.testing.assert_array_equal(df11.from_tile_order(t, 384, 192), w)
    lib = df11._lib()
    buf = np.zeros(64 * 64, dtype=np.uint16)
    assert lib.df11_to_tile_order(ctypes.c_void_p(buf.ctypes.data), 64, 64, ctypes.c_void_p(buf.ctypes.data)) == 2
    assert lib.df11_to_tile_order(None, 128, 64, ctypes.c_void_p(buf.ctypes.data)) == 1


def test_encode_multi_tile_order_flags():
    mats = [workloads.normal_matrix(256, 128, 0.02, seed=1), workloads.normal_matrix(1, 128, 0.02, seed=2)[0],
            workloads.normal_matrix(100, 64, 0.02, seed=3)]
    blk = df11.encode_multi(mats, tile_order=True)
    assert blk.tiled == [True, False, False]
    flat = np.concatenate([df11.to_tile_order(mats[0]), mats[1].reshape(-1), mats[2].reshape(-1)])
    np.testing.assert_array_equal(blk.host_array("enc"), df11.encode(flat).host_array("enc"))


def test_decode_gemm_argument_checks():
    """df11_decode_gemm refuses bad calls before any GPU work: a tensor
    without per-thread counts, T outside 1..256, rows not a multiple of 128 or
    cols of 64 are unsupported; misaligned, overlapping or out-of-range
    matrices and NULL vectors are invalid; no matrices is a no-op."""
    lib = df11._lib()
    mats = [workloads.normal_matrix(128, 64, 0.02, seed=1), workloads.normal_matrix(256, 128, 0.02, seed=2)]
    t = df11.encode_multi(mats, tile_order=True)
    keep = []

    def bind(tt):
        d = tt._bind()
        for name in tt.arrays:
            v, owner = _aligned_copy(tt.host_array(name))
            keep.append(owner)
            setattr(d, name, v.ctypes.data)
        return d

    d, dn = bind(t), bind(t.without_counts())
    xbuf, xown = _aligned_copy(np.zeros(256 * 128 + 8, dtype=np.uint16))
    ybuf = np.zeros(256 * 256 + 4, dtype=np.float32)
    X, Y = xbuf.ctypes.data, ybuf.ctypes.data

    def call(descs, T=16, n=None, dd=None):
        arr = (df11._GemvMat * max(1, len(descs)))(*[df11._GemvMat(*m) for m in descs])
        return lib.df11_decode_gemm(ctypes.byref(dd or d), arr, len(descs) if n is None else n, T, None, None)

    good = [(0, 128, 64, X, Y), (8192, 256, 128, X, Y)]
    assert call(good, n=0) == 0
    assert call(good, dd=dn) == 2                              # no stored counts
    assert call(good, T=0) == 2 and call(good, T=257) == 2
    assert call([(0, 64, 128, X, Y)]) == 2                     # rows not a multiple of 128
    assert call([(0, 128, 32, X, Y)]) == 2                     # cols not a multiple of 64
    assert call([(8, 128, 64, X, Y)]) == 1                     # offset not a multiple of 16
    assert call([(0, 128, 64, X + 2, Y)]) == 1                 # x not 16-byte aligned
    assert call([(0, 128, 64, None, Y)]) == 1                  # NULL x
    assert call([(8192, 256, 128, X, Y), (0, 128, 64, X, Y)]) == 1   # out of order
    assert call([(16384, 256, 128, X, Y)]) == 1                # runs past the tensor's end
    assert call(good * 9) == 2                                 # more than 16 matrices


def test_gemm_multi_argument_checks():
    """df11_gemm_bf16_multi refuses bad calls before any GPU work: no
    products is a no-op; more than 16 products, T outside 1..256, out not a
    multiple of 128 or in of 64 are unsupported; NULL or misaligned pointers
    are invalid."""
    lib = df11._lib()
    buf, own = _aligned_copy(np.zeros(4096, dtype=np.uint16))
    A = buf.ctypes.data

    def call(descs, T=16, n=None):
        arr = (df11._GemmMat * max(1, len(descs)))(*[df11._GemmMat(*m) for m in descs])
        return lib.df11_gemm_bf16_multi(arr, len(descs) if n is None else n, T, None, None)

    good = (A, A, A, 128, 64)
    assert call([good], n=0) == 0
    assert call([good] * 17) == 2
    assert call([good], T=0) == 2 and call([good], T=257) == 2
    assert call([(A, A, A, 100, 64)]) == 2                     # out not a multiple of 128
    assert call([(A, A, A, 128, 32)]) == 2                     # in not a multiple of 64
    assert call([(0, A, A, 128, 64)]) == 1                     # NULL x
    assert call([(A + 2, A, A, 128, 64)]) == 1                 # x not 16-byte aligned
    assert call([(A, A + 8, A, 128, 64)]) == 1                 # w not 16-byte aligned
    assert call([(A, A, A + 2, 128, 64)]) == 1                 # y not 4-byte aligned
    assert lib.df11_gemm_bf16_multi(None, 1, 16, None, None) == 1


def test_call_descriptor_follows_the_arrays():
    """The descriptor the binding passes to the library is reused while the
    arrays stay where they are and rebuilt as soon as one moves; _bind()
    always returns a fresh copy (callers may edit it)."""
    t = df11.encode(workloads.normal_matrix(64, 64, 0.02, seed=3))
    d1 = t._desc_for_call()
    assert t._desc_for_call() is d1
    assert d1.enc == t.host_array("enc").ctypes.data
    b = t._bind()
    assert b is not d1 and b.enc == d1.enc
    b.enc = 0  # editing a fresh copy leaves the call descriptor alone
    assert t._desc_for_call().enc == d1.enc
    t.arrays["enc"] = np.array(t.host_array("enc"), copy=True)  # the array moves
    d2 = t._desc_for_call()
    assert d2 is not d1 and d2.enc == t.arrays["enc"].ctypes.data
