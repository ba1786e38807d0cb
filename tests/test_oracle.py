"""Pins for the oracle: each check ties it to something other than itself --
printed examples, closed forms, brute force on tiny alphabets, and an
independent numpy route to the same bits.  All CPU-only."""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _bits_to_str(code: int, length: int) -> str:
    return format(code, f"0{length}b") if length else ""


# ---------------------------------------------------------------- goldens

def test_rfc1951_canonical_example(golden_dir):
    g = _load(golden_dir, "rfc1951_canonical.json")
    lengths = np.zeros(256, dtype=np.uint8)
    lengths[: len(g["lengths"])] = g["lengths"]
    codes = oracle.canonical_codes(lengths)
    got = [_bits_to_str(int(codes[i]), int(lengths[i])) for i in range(len(g["symbols"]))]
    assert got == g["codes"]


def test_clrs_huffman_example(golden_dir):
    g = _load(golden_dir, "clrs_huffman.json")
    count = np.zeros(256, dtype=np.uint64)
    count[: len(g["counts"])] = g["counts"]
    for lengths in (oracle.huffman_lengths(count), oracle.package_merge_lengths(count, 32)):
        cost = int(np.sum(count.astype(np.int64) * lengths.astype(np.int64)))
        assert cost == g["optimal_cost"]
        # the printed lengths are one optimal assignment; ties may permute
        # lengths among equal counts only, and this example has none
        assert list(lengths[:6]) == g["optimal_lengths"]


def test_df11_worked_example(golden_dir):
    g = _load(golden_dir, "df11_worked_example.json")
    w = np.array([int(x, 16) for x in g["weights_hex"]], dtype=np.uint16)
    count = oracle.histogram(w)
    lengths = oracle.package_merge_lengths(count, 32)
    for e, l in g["exponent_lengths"].items():
        assert lengths[int(e)] == l
    assert int(np.count_nonzero(lengths)) == len(g["exponent_lengths"])
    codes = oracle.canonical_codes(lengths)
    for e, c in g["exponent_codes"].items():
        assert _bits_to_str(int(codes[int(e)]), int(lengths[int(e)])) == c
    enc, sm, bits = oracle.encode(w, lengths)
    assert bits == g["total_bits"]
    assert [int(x) for x in enc] == [int(x, 16) for x in g["enc_hex"]]
    assert [int(x) for x in sm] == [int(x, 16) for x in g["sm_hex"]]
    out = oracle.decode(enc, bits, sm, w.size, lengths)
    assert np.array_equal(out, w)
    a1 = oracle.aux(enc, bits, w.size, lengths, bytes_per_thread=1, threads_per_block=1)
    assert list(a1["gaps"]) == g["aux_n1_T1"]["gaps"]
    assert list(a1["counts"]) == g["aux_n1_T1"]["counts"]
    assert list(a1["block_start"]) == g["aux_n1_T1"]["block_start"]
    assert [int(x) for x in oracle.pack_gaps(a1["gaps"])] == [
        int(x, 16) for x in g["aux_n1_T1"]["packed_gaps_hex"]]
    a2 = oracle.aux(enc, bits, w.size, lengths, bytes_per_thread=1, threads_per_block=2)
    assert list(a2["gaps"]) == g["aux_n1_T2"]["gaps"]
    assert list(a2["block_start"]) == g["aux_n1_T2"]["block_start"]
    h, k, mean = oracle.exponent_stats(count, lengths)
    assert k == 4 and math.isclose(h, 1.75) and math.isclose(mean, 1.75)


# ---------------------------------------------------------- brute force

def _brute_force_cost(counts, cap):
    """Minimum of sum(count * len) over all length vectors with every length
    in [1, cap] and Kraft sum <= 1 (enumerated exhaustively)."""
    k = len(counts)
    best = None
    c = np.array(counts, dtype=np.int64)
    for ls in itertools.product(range(1, cap + 1), repeat=k):
        if sum(2.0 ** -l for l in ls) > 1.0 + 1e-12:
            continue
        cost = int(np.dot(c, ls))
        if best is None or cost < best:
            best = cost
    return best


@pytest.mark.parametrize("k", [2, 3, 4, 5, 6])
def test_package_merge_optimal_brute_force(k):
    rng = np.random.default_rng(100 + k)
    for trial in range(6):
        counts = rng.integers(1, 60, size=k)
        if trial == 0:
            counts = np.array([2 ** i for i in range(k)])  # skewed
        syms = rng.choice(256, size=k, replace=False)
        full = np.zeros(256, dtype=np.uint64)
        full[syms] = counts
        min_cap = max(1, math.ceil(math.log2(k)))
        for cap in range(min_cap, k + 1):
            pm = oracle.package_merge_lengths(full, cap)
            assert pm[syms].max() <= cap
            assert np.all(pm[np.setdiff1d(np.arange(256), syms)] == 0)
            cost = int(np.dot(full.astype(np.int64), pm.astype(np.int64)))
            assert cost == _brute_force_cost(list(counts), cap), (counts, cap)
        hu = oracle.huffman_lengths(full)
        cost_h = int(np.dot(full.astype(np.int64), hu.astype(np.int64)))
        assert cost_h == _brute_force_cost(list(counts), k)


def test_package_merge_seven_symbols_brute_force():
    counts = [31, 1, 7, 2, 13, 3, 5]
    full = np.zeros(256, dtype=np.uint64)
    syms = [3, 17, 100, 126, 127, 200, 255]
    full[syms] = counts
    for cap in (3, 4, 5):
        pm = oracle.package_merge_lengths(full, cap)
        cost = int(np.dot(full.astype(np.int64), pm.astype(np.int64)))
        assert cost == _brute_force_cost(counts, cap)


def test_cap_too_small_is_an_error():
    full = np.zeros(256, dtype=np.uint64)
    full[:5] = 1
    with pytest.raises(oracle.OracleError):
        oracle.package_merge_lengths(full, 2)


# ------------------------------------------------------------ closed forms

def test_dyadic_lengths_equal_minus_log2_p():
    # p = 1/2, 1/4, 1/8, 1/16, 1/32, 1/32  -> lengths 1,2,3,4,5,5, mean = H
    counts = [16, 8, 4, 2, 1, 1]
    full = np.zeros(256, dtype=np.uint64)
    syms = [126, 125, 127, 124, 128, 0]
    full[syms] = counts
    for lengths in (oracle.huffman_lengths(full), oracle.package_merge_lengths(full, 32)):
        assert list(lengths[syms]) == [1, 2, 3, 4, 5, 5]
        h, k, mean = oracle.exponent_stats(full, lengths)
        assert math.isclose(h, mean)


def test_uniform_256_exponents_identity_code():
    w = workloads.adversarial("uniform_exponents")
    c = oracle.compress(w)
    assert np.all(c["lengths"] == 8)
    assert np.array_equal(oracle.canonical_codes(c["lengths"]), np.arange(256, dtype=np.uint32))
    # every code is the exponent byte itself, so the stream is the exponents
    expo = ((w >> 7) & 0xFF).astype(np.uint8)
    assert np.array_equal(c["enc"], expo)
    assert c["total_bits"] == 8 * w.size


def test_two_symbols_get_one_bit_each():
    w = workloads.adversarial("two_values")
    c = oracle.compress(w)
    assert sorted(int(x) for x in c["lengths"][c["lengths"] > 0]) == [1, 1]
    assert c["total_bits"] == w.size


def test_single_symbol_gets_code_zero():
    w = workloads.adversarial("all_equal")
    c = oracle.compress(w)
    e = 0x3F80 >> 7
    assert c["lengths"][e] == 1 and int(np.count_nonzero(c["lengths"])) == 1
    assert oracle.canonical_codes(c["lengths"])[e] == 0
    assert np.all(c["enc"] == 0) and c["total_bits"] == w.size
    assert oracle.kraft_sum_2p32(c["lengths"]) == 1 << 31
    assert np.array_equal(oracle.decode(c["enc"], c["total_bits"], c["sm"], w.size, c["lengths"]), w)


def test_fibonacci_depth_and_cap():
    w = workloads.adversarial("fibonacci_exponents")
    count = oracle.histogram(w)
    hu = oracle.huffman_lengths(count)
    assert hu.max() == 25  # K - 1 for 26 Fibonacci weights
    for cap in (8, 12, 16, 24):
        pm = oracle.package_merge_lengths(count, cap)
        assert pm.max() == cap
        assert oracle.kraft_sum_2p32(pm) == 1 << 32
        # capped cost can only be >= the unlimited optimum
        assert np.dot(count.astype(np.int64), pm.astype(np.int64)) >= np.dot(
            count.astype(np.int64), hu.astype(np.int64))
    pm25 = oracle.package_merge_lengths(count, 25)
    assert np.dot(count.astype(np.int64), pm25.astype(np.int64)) == np.dot(
        count.astype(np.int64), hu.astype(np.int64))


def test_entropy_bounds_mean_length():
    w = workloads.normal_matrix(256, 256, 0.02, seed=3)
    count = oracle.histogram(w)
    lengths = oracle.package_merge_lengths(count, 32)
    h, k, mean = oracle.exponent_stats(count, lengths)
    assert h <= mean < h + 1


# --------------------------------------------------- invariants on streams

CASES = ["all_bf16_patterns", "all_zero", "all_equal", "two_values", "random_u16",
         "neg_zero_and_nan", "single", "empty", "subnormals", "uniform_exponents",
         "fibonacci_exponents"]


@pytest.mark.parametrize("name", CASES)
def test_roundtrip_identity_and_kraft(name):
    w = workloads.adversarial(name)
    for cap in (32, 12):
        count = oracle.histogram(w)
        k = int(np.count_nonzero(count))
        if k > (1 << cap):
            continue
        c = oracle.compress(w, cap)
        lengths = c["lengths"]
        assert lengths.max(initial=0) <= cap
        assert oracle.is_prefix_free(lengths)
        kraft = oracle.kraft_sum_2p32(lengths)
        if k >= 2:
            assert kraft == 1 << 32
        elif k == 1:
            assert kraft == 1 << 31
        out = oracle.decode(c["enc"], c["total_bits"], c["sm"], w.size, lengths)
        assert out.dtype == np.uint16 and np.array_equal(out, w)


def _lengths(values):
    out = np.zeros(256, dtype=np.uint8)
    out[: len(values)] = values
    return out


@pytest.mark.parametrize("bad", [[1, 1, 1], [1, 2, 2, 2], [2, 2, 2, 2, 3], [1, 1, 2]])
def test_over_full_lengths_are_rejected(bad):
    """Lengths whose Kraft sum exceeds 1 admit no prefix code: the canonical
    assignment refuses them and the prefix check says no.  {1,1,1} sums to
    3/2 and {1,2,2,2} to 5/4."""
    lengths = _lengths(bad)
    assert oracle.kraft_sum_2p32(lengths) > 1 << 32
    assert not oracle.is_prefix_free(lengths)
    with pytest.raises(oracle.OracleError):
        oracle.canonical_codes(lengths)


def test_shortening_one_length_of_a_complete_code_overflows_kraft():
    """Every length vector of a complete code (Kraft sum exactly 1) turns
    into an over-full one when any single length is shortened by one bit."""
    w = workloads.normal_matrix(64, 64, 0.02, seed=5)
    lengths = oracle.package_merge_lengths(oracle.histogram(w), 32)
    assert oracle.kraft_sum_2p32(lengths) == 1 << 32
    for s in np.flatnonzero(lengths):
        if lengths[s] < 2:
            continue
        short = lengths.copy()
        short[s] -= 1
        assert oracle.kraft_sum_2p32(short) > 1 << 32
        assert not oracle.is_prefix_free(short)
        with pytest.raises(oracle.OracleError):
            oracle.canonical_codes(short)


def test_length_above_32_is_rejected():
    lengths = _lengths([1, 2, 33])
    assert not oracle.is_prefix_free(lengths)
    with pytest.raises(oracle.OracleError):
        oracle.canonical_codes(lengths)


@pytest.mark.parametrize("codes,lengths,ok", [
    # RFC 1951 section 3.2.2 example: A..H with lengths 3,3,3,3,3,2,4,4
    ([0b010, 0b011, 0b100, 0b101, 0b110, 0b00, 0b1110, 0b1111], [3, 3, 3, 3, 3, 2, 4, 4], True),
    ([0b0, 0b10, 0b11], [1, 2, 2], True),
    ([0b0, 0b01], [1, 2], False),            # "0" is a prefix of "01"
    ([0b01, 0b0], [2, 1], False),            # same, longer code inserted first
    ([0b10, 0b101, 0b11], [2, 3, 2], False),  # "10" is a prefix of "101"
    ([0b110, 0b110], [3, 3], False),         # the same code twice
    ([0b1, 0b0111, 0b0110, 0b010], [1, 4, 4, 3], True),
    ([0b1, 0b0111, 0b01111], [1, 4, 5], False),  # "0111" is a prefix of "01111"
])
def test_explicit_code_sets_prefix_check(codes, lengths, ok):
    """The tree-insertion check on explicit code sets, including ones whose
    lengths satisfy Kraft but whose codes collide; canonical codes from
    lengths alone can never reach these cases."""
    assert oracle.codes_prefix_free(codes, lengths) is ok


def test_canonical_codes_of_lengths_pass_the_explicit_check(golden_dir):
    g = _load(golden_dir, "rfc1951_canonical.json")
    lengths = _lengths(g["lengths"])
    assert oracle.codes_prefix_free(oracle.canonical_codes(lengths), lengths)


def test_encoded_bits_match_independent_bitstring():
    """The stream is the concatenation of the canonical codes, MSB-first;
    rebuilt here with Python strings and numpy.packbits."""
    w = workloads.normal_matrix(64, 96, 0.02, seed=11)
    c = oracle.compress(w)
    codes = oracle.canonical_codes(c["lengths"])
    expo = (w.reshape(-1) >> 7) & 0xFF
    s = "".join(_bits_to_str(int(codes[e]), int(c["lengths"][e])) for e in expo)
    assert len(s) == c["total_bits"]
    bits = np.array([ch == "1" for ch in s], dtype=np.uint8)
    assert np.array_equal(np.packbits(bits), c["enc"])
    sm = (((w.reshape(-1) >> 8) & 0x80) | (w.reshape(-1) & 0x7F)).astype(np.uint8)
    assert np.array_equal(sm, c["sm"])


@pytest.mark.parametrize("n_bytes,T", [(8, 256), (8, 32), (4, 64), (1, 3)])
def test_aux_matches_cumulative_sum_closed_form(n_bytes, T):
    """Code start positions are prefix sums of code lengths; gaps, counts and
    block starts follow from them with searchsorted / bincount."""
    w = workloads.adversarial("ragged_normal")[:200_000]
    c = oracle.compress(w)
    lens = c["lengths"][((w >> 7) & 0xFF)].astype(np.int64)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    bits = c["total_bits"]
    span = 8 * n_bytes
    n_threads = -(-bits // span)
    n_blocks = -(-n_threads // T)
    a = oracle.aux(c["enc"], bits, w.size, c["lengths"], n_bytes, T)
    assert a["n_threads"] == n_threads and a["n_blocks"] == n_blocks
    ext = np.concatenate([starts, [bits]])
    t0 = np.arange(n_threads, dtype=np.int64) * span
    first = ext[np.searchsorted(ext, t0, side="left")]
    gaps = np.zeros(n_blocks * T, dtype=np.int64)
    gaps[:n_threads] = first - t0
    assert np.array_equal(a["gaps"].astype(np.int64), gaps)
    assert a["gaps"].max() <= 31  # 5-bit gap field
    counts = np.bincount(starts // span, minlength=n_blocks * T)
    assert np.array_equal(a["counts"].astype(np.int64), counts)
    bs = np.concatenate([[0], np.cumsum(counts.reshape(n_blocks, T).sum(axis=1))])
    assert np.array_equal(a["block_start"].astype(np.int64), bs)
    assert a["block_start"][-1] == w.size


def test_pack_gaps_matches_packbits():
    rng = np.random.default_rng(5)
    g = rng.integers(0, 32, size=1001).astype(np.uint8)
    s = "".join(format(int(x), "05b") for x in g)
    bits = np.array([ch == "1" for ch in s], dtype=np.uint8)
    assert np.array_equal(oracle.pack_gaps(g), np.packbits(bits))
    p = oracle.pack_gaps(g)
    assert all(oracle.read_gap(p, t) == g[t] for t in range(0, 1001, 37))


def test_decode_rejects_truncated_and_corrupt_streams():
    w = workloads.normal_matrix(32, 32, 0.02, seed=2)
    c = oracle.compress(w)
    with pytest.raises(oracle.OracleError):
        oracle.decode(c["enc"], c["total_bits"] - 1, c["sm"], w.size, c["lengths"])
    with pytest.raises(oracle.OracleError):
        oracle.decode(c["enc"], c["total_bits"] + 3, c["sm"], w.size, c["lengths"])


def test_mistake_in_lengths_is_caught():
    """A plausible slip -- swapping the lengths of two exponents -- keeps a
    valid code but loses optimality, and the brute-force pin sees it."""
    counts = [40, 10, 5, 3]
    full = np.zeros(256, dtype=np.uint64)
    full[[10, 11, 12, 13]] = counts
    good = oracle.package_merge_lengths(full, 32)
    bad = good.copy()
    bad[10], bad[13] = good[13], good[10]
    best = _brute_force_cost(counts, 4)
    assert int(np.dot(full.astype(np.int64), good.astype(np.int64))) == best
    assert int(np.dot(full.astype(np.int64), bad.astype(np.int64))) > best


def test_llm_like_statistics_near_the_pages():
    """The pages report ~2.6 bits of exponent entropy, ~40 exponent values in
    use and ~11 bits per weight for LLM weights.  Gaussian stand-ins land in
    the same region (a plausibility check, not a parity item)."""
    w = workloads.normal_matrix(1024, 1024, 0.02, seed=0)
    count = oracle.histogram(w)
    lengths = oracle.package_merge_lengths(count, 32)
    h, k, mean = oracle.exponent_stats(count, lengths)
    assert 2.2 < h < 3.0
    assert 15 <= k <= 45
    assert 10.0 < 8 + mean < 12.0


def test_decode_range_pieces_at_block_starts():
    """The stream cut at thread-block starts (bit 16384*b plus the gap of the
    block's first thread; element block_start[b]) decodes piece by piece to
    the same weights as the whole stream; a cut one bit off does not."""
    w = workloads.normal_matrix(300, 256, 0.02, seed=13).reshape(-1)
    c = oracle.compress(w, 12)
    a = oracle.aux(c["enc"], c["total_bits"], w.size, c["lengths"], 8, 256)
    bs, gaps, nb = a["block_start"], a["gaps"], a["n_blocks"]
    assert nb >= 5

    def first_bit(b):
        return c["total_bits"] if b >= nb else 16384 * b + int(gaps[256 * b])

    cuts = [0, 1, 3, nb - 1, nb]
    got = np.concatenate([
        oracle.decode_range(c["enc"], first_bit(b0), first_bit(b1), c["sm"][bs[b0]:bs[b1]], int(bs[b1] - bs[b0]),
                            c["lengths"]) for b0, b1 in zip(cuts[:-1], cuts[1:])])
    np.testing.assert_array_equal(got, w)
    b = 2
    n = int(bs[b + 1] - bs[b])
    try:
        bad = oracle.decode_range(c["enc"], first_bit(b) + 1, first_bit(b + 1), c["sm"][bs[b]:bs[b + 1]], n,
                                  c["lengths"])
        assert not np.array_equal(bad, w[bs[b]:bs[b + 1]])
    except oracle.OracleError:
        pass  # the shifted piece does not even end on its last code
