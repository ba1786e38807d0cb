"""Row gather (embedding lookup): only the requested rows of a compressed
[R, row_len] matrix are decoded; each output row bit-exact against the
original matrix."""
import numpy as np
import pytest

import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import huffman_decode_02_b200 as df11  # noqa: E402


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _rows_bits(x):
    return x.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("shape", [(3000, 512), (1001, 333), (64, 4096), (5, 16)])
def test_rows_bit_exact(shape):
    dev = _dev()
    w = workloads.normal_matrix(*shape, 0.02, seed=shape[0])
    d = df11.encode(w).to(dev)
    rng = np.random.default_rng(shape[1])
    rows = np.concatenate([[0, shape[0] - 1, shape[0] // 2, shape[0] // 2],
                           rng.integers(0, shape[0], 200)]).astype(np.int32)
    for dd in (d, d.without_counts()):  # stored counts, and the count pass
        out = df11.decode_rows(dd, shape[1], torch.from_numpy(rows).to(dev))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(_rows_bits(out), w[rows])


def test_rows_heavy_tail_long_codes():
    """Long codes (uncapped) through the gather path."""
    dev = _dev()
    rng = np.random.default_rng(3)
    x = (rng.standard_t(3, (600, 1024)) * 0.015).astype(np.float32)
    x[rng.random(x.shape) < 0.001] *= 1000.0
    w = workloads.round_to_bf16(x)
    t = df11.encode(w, df11.Params(max_code_len=32))
    assert t.code_len.max() > 12  # the long-code instance
    d = t.to(dev)
    rows = torch.from_numpy(rng.integers(0, 600, 100).astype(np.int32)).to(dev)
    for dd in (d, d.without_counts()):  # stored counts, and the count pass
        out = df11.decode_rows(dd, w.shape[1], rows)
        np.testing.assert_array_equal(_rows_bits(out), w[rows.cpu().numpy()])


def test_bad_row_index_reported_other_rows_written():
    dev = _dev()
    w = workloads.normal_matrix(100, 256, 0.02, seed=7)
    d = df11.encode(w).to(dev)
    rows = torch.tensor([3, 100, 99], dtype=torch.int32, device=dev)
    out = torch.zeros(3, 256, dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    df11.decode_rows(d, 256, rows, out, err)
    with pytest.raises(df11.CorruptStreamError):
        df11.read_error(err)
    assert int(err.item()) & df11.KERR_BAD_ROW
    got = _rows_bits(out)
    np.testing.assert_array_equal(got[0], w[3])
    np.testing.assert_array_equal(got[2], w[99])
    assert not got[1].any()  # the bad row is left untouched


def test_rows_argument_checks():
    dev = _dev()
    w = workloads.normal_matrix(10, 30, 0.02, seed=1)
    d = df11.encode(w).to(dev)
    rows = torch.zeros(2, dtype=torch.int32, device=dev)
    with pytest.raises(df11.DF11Error):
        df11.decode_rows(d, 7, rows)  # 7 does not divide 300
    empty = df11.decode_rows(d, 30, torch.zeros(0, dtype=torch.int32, device=dev))
    assert tuple(empty.shape) == (0, 30)


@pytest.mark.slow
def test_lm_head_full_decode_and_gather():
    """Llama-3.1-8B LM head / embedding shape (128256 x 4096, 525M weights):
    full single-matrix decode checked on sampled elements against the
    original, and a 256-token row gather checked row by row."""
    dev = _dev()
    w = workloads.normal_matrix(128256, 4096, 0.02, seed=5)
    t = df11.encode(w)
    d = t.to(dev)
    full = df11.decode(d)
    rng = np.random.default_rng(8)
    idx = rng.integers(0, w.size, 1_000_000)
    got = full.view(torch.int16)[torch.from_numpy(idx).to(dev)].cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got, w.reshape(-1)[idx])
    del full
    rows = rng.integers(0, 128256, 256).astype(np.int32)
    out = df11.decode_rows(d, 4096, torch.from_numpy(rows).to(dev))
    np.testing.assert_array_equal(_rows_bits(out), w[rows])


@pytest.mark.parametrize("kind", ["dense", "wide"])
def test_rows_other_instances(kind):
    """Gather through the instances for blocks with more codes: 1-bit codes
    (a two-valued matrix, up to 16384 codes per block) and a five-exponent
    matrix (about 7500 codes per block)."""
    dev = _dev()
    rng = np.random.default_rng(17)
    if kind == "dense":
        e = rng.choice([100, 126], p=[0.2, 0.8], size=(4000, 96))
    else:
        e = rng.choice([120, 121, 122, 123, 124], p=[0.3, 0.3, 0.2, 0.1, 0.1], size=(4000, 96))
    w = ((e << 7) | rng.integers(0, 128, e.shape) | (rng.integers(0, 2, e.shape) << 15)).astype(np.uint16)
    t = df11.encode(w)
    need = t.desc.max_block_codes + 15
    assert (need > 8192) if kind == "dense" else (7152 < need <= 8192)
    d = t.to(dev)
    rows = torch.from_numpy(rng.integers(0, 4000, 300).astype(np.int32)).to(dev)
    for dd in (d, d.without_counts()):  # stored counts, and the count pass
        out = df11.decode_rows(dd, 96, rows)
        np.testing.assert_array_equal(_rows_bits(out), w[rows.cpu().numpy()])
        np.testing.assert_array_equal(_rows_bits(df11.decode(dd)).reshape(w.shape), w)
