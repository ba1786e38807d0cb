"""GPU parity: the sm_100a decode through the C ABI against the oracle,
element by element, bit-exact (compared as uint16 bit patterns so that -0.0,
subnormals and NaN payloads count)."""
import ctypes

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import huffman_decode_02_b200 as df11  # noqa: E402


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _bits(x: torch.Tensor) -> np.ndarray:
    return x.view(torch.int16).cpu().numpy().view(np.uint16)


def _oracle_decode(t: df11.DF11Tensor) -> np.ndarray:
    """The oracle's bit-serial decode of the product's stream."""
    enc = t.host_array("enc")
    sm = t.host_array("sm")
    return oracle.decode(enc, t.total_bits, sm, t.n_elems, t.code_len)


def _gpu_roundtrip(w, params=None, check_oracle=True):
    """Both decode paths: with the stored per-thread counts (one decoding
    pass) and without them (count pass, then decoding pass)."""
    dev = _dev()
    w = np.ascontiguousarray(w).reshape(-1).view(np.uint16)
    t = df11.encode(w, params)
    assert t.has_counts
    d = t.to(dev)
    ref = _oracle_decode(t) if check_oracle else w
    if check_oracle:
        assert np.array_equal(ref, w)  # the oracle reproduces the input
    got = None
    for dd in (d, d.without_counts()):
        out = df11.decode(dd)
        torch.cuda.synchronize()
        got = _bits(out)
        np.testing.assert_array_equal(got, ref)
    return t, d, got


@pytest.mark.parametrize("name", workloads.ADVERSARIAL_NAMES)
def test_adversarial_bit_exact(name):
    _gpu_roundtrip(workloads.adversarial(name))


@pytest.mark.parametrize("cap", [8, 12, 16, 24, 32])
def test_length_cap_bit_exact(cap):
    _gpu_roundtrip(workloads.adversarial("fibonacci_exponents"), df11.Params(max_code_len=cap))


def test_long_codes_bit_exact():
    rng = np.random.default_rng(21)
    e = np.minimum(rng.geometric(0.42, size=3_000_001), 31) + 100
    w = ((e << 7) | rng.integers(0, 128, e.size) | (rng.integers(0, 2, e.size) << 15)).astype(np.uint16)
    t, _, _ = _gpu_roundtrip(w, df11.Params(max_code_len=32))
    assert t.code_len.max() > 20  # the long-code instance
    t, _, _ = _gpu_roundtrip(w)
    assert t.code_len.max() == 12  # default cap: the short-code instance


def test_config1_1024x1024_seed0():
    w = workloads.normal_matrix(1024, 1024, 0.02, seed=0)
    t, _, _ = _gpu_roundtrip(w)
    assert t.n_blocks > 4 * 148 // 8  # several tiles per CTA group


def test_config2_4096x4096_seed1():
    _gpu_roundtrip(workloads.normal_matrix(4096, 4096, 0.02, seed=1))
    _gpu_roundtrip(workloads.normal_matrix(4096, 4096, 0.02, seed=1), df11.Params(max_code_len=32))


@pytest.mark.parametrize("n", [1, 7, 15, 16, 17, 255, 4096 + 3, 131_071, 2_000_003])
def test_ragged_sizes(n):
    w = workloads.adversarial("ragged_normal")
    w = np.concatenate([w, w])[:n] if n > w.size else w[:n]
    _gpu_roundtrip(w)


def test_block_decode_small_and_views():
    dev = _dev()
    mats = [workloads.normal_matrix(r, c, s, seed=i) for i, (r, c, s) in
            enumerate([(256, 128, 0.02), (64, 128, 0.03), (3, 7, 0.5), (128, 256, 0.01)])]
    blk = df11.encode_multi(mats)
    d = blk.to(dev)
    scratch = torch.full((blk.n_elems + 100,), float("nan"), dtype=torch.bfloat16, device=dev)
    df11.decode_block(d, scratch)
    for m, v in zip(mats, d.views(scratch)):
        assert tuple(v.shape) == m.shape
        np.testing.assert_array_equal(_bits(v).reshape(-1), m.reshape(-1))
    # reuse of the same scratch for a second block
    mats2 = [workloads.normal_matrix(300, 100, 0.02, seed=77)]
    blk2 = df11.encode_multi(mats2).to(dev)
    df11.decode_block(blk2, scratch)
    np.testing.assert_array_equal(_bits(scratch[: blk2.n_elems]), mats2[0].reshape(-1))


def test_decode_on_side_stream_and_repeat():
    dev = _dev()
    w = workloads.normal_matrix(2048, 1024, 0.02, seed=5)
    d = df11.encode(w).to(dev)
    s = torch.cuda.Stream(device=dev)
    out = torch.empty(w.size, dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    with torch.cuda.stream(s):
        for _ in range(3):
            df11.decode(d, out, err, stream=s)
    s.synchronize()
    assert df11.read_error(err, s) == 0
    np.testing.assert_array_equal(_bits(out), w.reshape(-1))


@pytest.mark.parametrize("counts", [True, False])
def test_corrupt_block_start_is_reported(counts):
    dev = _dev()
    w = workloads.normal_matrix(512, 512, 0.02, seed=6)
    d = df11.encode(w).to(dev)
    d = d if counts else d.without_counts()
    bs = d.arrays["block_start"].view(torch.int32)
    bs[3] += 5  # block 2 claims 5 more elements, block 3 5 fewer
    with pytest.raises(df11.CorruptStreamError):
        df11.decode(d)


@pytest.mark.parametrize("counts", [True, False])
def test_corrupt_stream_bits_are_reported(counts):
    dev = _dev()
    w = workloads.normal_matrix(512, 512, 0.02, seed=8)
    d = df11.encode(w).to(dev)
    d = d if counts else d.without_counts()
    enc = d.arrays["enc"]
    enc[1000:1100] ^= 0x5A  # scramble 100 bytes of codes
    with pytest.raises(df11.CorruptStreamError):
        df11.decode(d)


@pytest.mark.parametrize("thread", [0, 5, 300, 1000])
def test_corrupt_stored_count_is_reported(thread):
    """A stored count off by one breaks its block's sum (reported by the
    block check); two counts moved in opposite directions keep the sum, and
    the chain's bit check reports them."""
    dev = _dev()
    w = workloads.normal_matrix(512, 512, 0.02, seed=10)
    d = df11.encode(w).to(dev)
    cnt = d.arrays["counts"]
    cnt[thread] += 1
    with pytest.raises(df11.CorruptStreamError):
        df11.decode(d)
    cnt[thread + 1] -= 1  # same block: the block's sum is right again
    with pytest.raises(df11.CorruptStreamError):
        df11.decode(d)
    cnt[thread] -= 1
    cnt[thread + 1] += 1  # restored
    np.testing.assert_array_equal(_bits(df11.decode(d)), w.reshape(-1))


def test_sign_mantissa_flip_changes_only_that_weight():
    dev = _dev()
    w = workloads.normal_matrix(256, 256, 0.02, seed=9).reshape(-1)
    d = df11.encode(w).to(dev)
    d.arrays["sm"][12345] ^= 0x81
    got = _bits(df11.decode(d))
    exp = w.copy()
    exp[12345] ^= 0x8001  # sign bit and mantissa bit 0
    np.testing.assert_array_equal(got, exp)


def test_bad_arguments_rejected():
    dev = _dev()
    w = workloads.normal_matrix(64, 64, 0.02, seed=1)
    d = df11.encode(w).to(dev)
    out = torch.empty(w.size + 8, dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    with pytest.raises(df11.DF11Error):
        df11.decode(d, out[1:], err)  # not 16-byte aligned
    bad = df11.DF11Tensor(df11._Tensor.from_buffer_copy(d.desc), d.arrays, d.device, d.shapes, d.offsets)
    bad.desc.n_threads += 1
    with pytest.raises(df11.DF11Error):
        df11.decode(bad, out, err)
    offs = (ctypes.c_uint64 * 2)(0, w.size - 1)
    st = df11._lib().df11_decode_block(ctypes.byref(d._bind()), offs, 1, ctypes.c_void_p(out.data_ptr()),
                                       ctypes.c_void_p(err.data_ptr()), ctypes.c_void_p(0))
    assert st == 1


@pytest.mark.slow
@pytest.mark.parametrize("cap", [12, 32])
def test_config3_llama8b_block_full_size(cap):
    """The benchmark's workload, in the benchmark's launch configuration
    (cap 12, the default, stored counts), with uncapped codes (cap 32,
    long-code path), and without the stored counts (count pass): every
    element compared with the oracle's decode of the same stream."""
    dev = _dev()
    mats = workloads.llama8b_block(seed=0)
    blk = df11.encode_multi(mats, df11.Params(max_code_len=cap))
    assert blk.n_elems == 218_112_000
    d = blk.to(dev)
    ref = _oracle_decode(blk)
    np.testing.assert_array_equal(ref, np.concatenate([m.reshape(-1) for m in mats]))
    scratch = torch.empty(blk.n_elems, dtype=torch.bfloat16, device=dev)
    for dd in (d, d.without_counts()):
        scratch.fill_(float("nan"))
        df11.decode_block(dd, scratch)
        np.testing.assert_array_equal(_bits(scratch), ref)


@pytest.mark.slow
@pytest.mark.parametrize("cap", [32, 12])
def test_config4_heavy_tail_full_size(cap):
    """Long codes (cap 32: up to 27 bits, through the long-code path) and the
    default 12-bit cap; with and without the stored counts."""
    dev = _dev()
    w = workloads.heavy_tail_matrix(seed=4)
    t = df11.encode(w, df11.Params(max_code_len=cap))
    assert t.code_len.max() >= (20 if cap == 32 else 12)
    d = t.to(dev)
    ref = _oracle_decode(t)
    np.testing.assert_array_equal(ref, w.reshape(-1))
    for dd in (d, d.without_counts()):
        np.testing.assert_array_equal(_bits(df11.decode(dd)), ref)


@pytest.mark.parametrize("offset_elems", [8, 16])
def test_output_alignment_paths(offset_elems):
    """Whole-chunk stores are 32 bytes when the output is 32-byte aligned and
    two 16-byte stores otherwise: both paths bit-exact, nothing written
    outside the output range."""
    dev = _dev()
    w = workloads.normal_matrix(777, 301, 0.02, seed=12)
    d = df11.encode(w).to(dev)
    buf = torch.full((w.size + 64,), -1, dtype=torch.int16, device=dev)
    out = buf[offset_elems: offset_elems + w.size].view(torch.bfloat16)
    df11.decode(d, out)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_bits(out), w.reshape(-1))
    rest = torch.cat([buf[:offset_elems], buf[offset_elems + w.size:]])
    assert bool((rest == -1).all())


@pytest.mark.slow
def test_maximum_size_tensor():
    """The largest tensor the format holds: 2^32 - 1 elements (u32 block
    output positions), 8.6 GB of BF16.  The weights repeat a 4096 x 4096
    Gaussian matrix, so the histogram and code are those of the matrix; the
    decoded tensor is compared with the input on 20 M sampled positions and
    on its last 4 M elements, and the last block start must be right below
    2^32.  The row gather, the fused matrix-vector product and the device
    encoder run on the same tensor."""
    dev = _dev()
    n = (1 << 32) - 1
    base = workloads.normal_matrix(4096, 4096, 0.02, seed=2).reshape(-1)
    w = np.tile(base, n // base.size + 1)[:n]
    t = df11.encode(w)
    bs = t.host_array("block_start")
    assert int(bs[t.n_blocks]) == n and int(bs[t.n_blocks - 1]) > n - 20_000
    d = t.to(dev)
    del t
    out = df11.decode(d)
    torch.cuda.synchronize()
    rng = np.random.default_rng(6)
    idx = np.concatenate([rng.integers(0, n, 20_000_000), np.arange(n - 4_000_000, n)])
    got = out.view(torch.int16)[torch.from_numpy(idx).to(dev)].cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got, w[idx])
    del out
    # row gather at the far end (65537 divides 2^32 - 1): rows 0, the middle and the last
    rows = np.array([0, 32768, 65533, 65534], dtype=np.int32)
    got = df11.decode_rows(d, 65537, torch.from_numpy(rows).to(dev))
    np.testing.assert_array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16),
                                  w.reshape(65535, 65537)[rows])
    # the fused matrix-vector product over the whole range (a [1048575, 4096]
    # matrix: chunk indices up to 2^28 - 256) and over a 1024 x 4096 matrix
    # that ends within 16 elements of 2^32 - 1; sampled rows (the last ones
    # among them) against FP64, within the FP32 rounding bound
    xb = workloads.round_to_bf16(rng.standard_normal((1, 4096), dtype=np.float32))
    x64 = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).double()
    far = ((n - 1024 * 4096) // 16) * 16
    for off, rows_m in ((0, n // 4096), (far, 1024)):
        view = df11.DF11Tensor(d.desc, d.arrays, d.device, [(rows_m, 4096)], [off, off + rows_m * 4096])
        y = df11.decode_gemv(view, {0: torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)})[0]
        r = np.unique(np.concatenate([rng.integers(0, rows_m, 300), np.arange(rows_m - 8, rows_m)]))
        W = torch.from_numpy(np.stack([w[off + int(i) * 4096: off + (int(i) + 1) * 4096] for i in r])
                             .view(np.int16)).view(torch.bfloat16).double()
        ref, mag = x64 @ W.T, x64.abs() @ W.abs().T
        got = y.cpu().double()[:, torch.from_numpy(r)]
        assert bool(torch.all((got - ref).abs() <= (4096 + 32) * 2.0 ** -24 * mag + 1e-30)), off
    # the device encoder on the same weights: arrays identical to the host encoder's
    e = df11.encode_device(torch.from_numpy(w.view(np.int16)).to(dev).view(torch.bfloat16))
    for k in ("enc", "sm", "gaps", "block_start", "lut", "counts"):
        nb = d.nbytes(k)
        assert e.nbytes(k) == nb and torch.equal(e.arrays[k][:nb], d.arrays[k][:nb]), k


def test_two_streams_at_once():
    """Two decodes in flight on two streams (no shared device state): both
    bit-exact."""
    dev = _dev()
    w1 = workloads.normal_matrix(3000, 1024, 0.02, seed=21)
    rng = np.random.default_rng(22)
    x = (rng.standard_t(3, (2000, 1024)) * 0.015).astype(np.float32)
    x[rng.random(x.shape) < 0.001] *= 1000.0
    w2 = workloads.round_to_bf16(x)  # heavy tail: long codes
    d1 = df11.encode(w1).to(dev)
    d2 = df11.encode(w2, df11.Params(max_code_len=32)).to(dev)
    s1, s2 = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    o1 = torch.empty(w1.size, dtype=torch.bfloat16, device=dev)
    o2 = torch.empty(w2.size, dtype=torch.bfloat16, device=dev)
    e1 = torch.zeros(1, dtype=torch.int32, device=dev)
    e2 = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    for _ in range(4):
        df11.decode(d1, o1, e1, stream=s1)
        df11.decode(d2, o2, e2, stream=s2)
    torch.cuda.synchronize()
    assert df11.read_error(e1, s1) == 0 and df11.read_error(e2, s2) == 0
    np.testing.assert_array_equal(_bits(o1), w1.reshape(-1))
    np.testing.assert_array_equal(_bits(o2), w2.reshape(-1))
