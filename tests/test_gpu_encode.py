"""The device encoder against the host encoder: the same code lengths and
byte-identical arrays (EncodedExponent, PackedSignMantissa, Gaps, block
starts, decode tables) and descriptor fields, so every property pinned for
the host encoder (and the oracle's agreement with it) carries over."""
import numpy as np
import pytest

import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import huffman_decode_02_b200 as df11  # noqa: E402

FIELDS = ["n_elems", "total_bits", "n_threads", "n_blocks", "max_block_codes", "enc_bytes", "sm_bytes",
          "gaps_bytes", "block_start_bytes", "lut_bytes", "counts_bytes"]


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _to_dev(m, dev):
    return torch.from_numpy(np.ascontiguousarray(m).view(np.int16)).to(dev).view(torch.bfloat16)


def _same(host: df11.DF11Tensor, d: df11.DF11Tensor):
    for f in FIELDS:
        assert getattr(host.desc, f) == getattr(d.desc, f), f
    assert bytes(host.desc.code_len) == bytes(d.desc.code_len)
    for k in ("enc", "sm", "gaps", "block_start", "lut", "counts"):
        a = host.host_array(k).view(np.uint8)[: host.nbytes(k)]
        b = d.host_array(k).view(np.uint8)[: d.nbytes(k)]
        np.testing.assert_array_equal(a, b, err_msg=k)


@pytest.mark.parametrize("name", workloads.ADVERSARIAL_NAMES)
def test_adversarial_identical(name):
    dev = _dev()
    w = workloads.adversarial(name)
    if w.size == 0:
        pytest.skip("empty input: covered by test_empty")
    _same(df11.encode(w), df11.encode_device(_to_dev(w, dev)))


@pytest.mark.parametrize("cap", [8, 12, 32])
def test_caps_identical(cap):
    dev = _dev()
    w = workloads.adversarial("fibonacci_exponents")
    p = df11.Params(max_code_len=cap)
    _same(df11.encode(w, p), df11.encode_device(_to_dev(w, dev), p))


@pytest.mark.parametrize("n", [1, 7, 8, 9, 8191, 8192, 8193, 100_003])
def test_ragged_identical_and_decodes(n):
    dev = _dev()
    w = workloads.adversarial("ragged_normal")
    w = np.concatenate([w] * (1 + n // max(1, w.size)))[:n]
    d = df11.encode_device(_to_dev(w, dev))
    _same(df11.encode(w), d)
    np.testing.assert_array_equal(df11.decode(d).view(torch.int16).cpu().numpy().view(np.uint16), w)


def test_block_of_matrices_identical():
    dev = _dev()
    mats = [workloads.normal_matrix(r, c, s, seed=i) for i, (r, c, s) in
            enumerate([(256, 128, 0.02), (64, 128, 0.03), (3, 7, 0.5), (128, 256, 0.01)])]
    d = df11.encode_device([_to_dev(m, dev) for m in mats])
    _same(df11.encode_multi(mats), d)
    scratch = df11.decode_block(d)
    for m, v in zip(mats, d.views(scratch)):
        np.testing.assert_array_equal(v.view(torch.int16).cpu().numpy().view(np.uint16), m)


def test_empty():
    dev = _dev()
    d = df11.encode_device(torch.empty(0, dtype=torch.bfloat16, device=dev))
    assert d.n_elems == 0 and d.total_bits == 0


@pytest.mark.slow
def test_llama_block_full_size_identical():
    dev = _dev()
    mats = workloads.llama8b_block(seed=0)
    d = df11.encode_device([_to_dev(m, dev) for m in mats])
    _same(df11.encode_multi(mats), d)
