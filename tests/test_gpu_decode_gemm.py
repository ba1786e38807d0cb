"""The fused decode -> tensor-core GEMM (df11_decode_gemm) against an FP64 CPU
product of the original weights: every output within the bound of FP32
accumulation, and the relative Frobenius error within 2e-3.  The matrices are
stored in tile order (encode_multi(..., tile_order=True)); the decoded
weights themselves never leave the GPU's shared memory."""
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


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def _x(T: int, cols: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return workloads.round_to_bf16(rng.standard_normal((T, cols), dtype=np.float32))


def _check(y: torch.Tensor, w: np.ndarray, xb: np.ndarray, rows=None):
    """Every output within (K + 64) * 2^-23 * sum |w x| of the FP64 product
    (BF16 products are exact in FP32; the tensor cores and the cross-CTA
    atomics add with FP32 roundings), and the relative Frobenius error within
    2e-3.  `rows`: check only these output rows."""
    W = _bf16(w).double()
    X = _bf16(xb).double()
    got = y.cpu().double()
    if rows is not None:
        W = W[torch.as_tensor(rows)]
        got = got[:, torch.as_tensor(rows)]
    ref, mag = X @ W.T, X.abs() @ W.abs().T
    k = w.shape[1]
    assert bool(torch.all((got - ref).abs() <= (k + 64) * 2.0 ** -23 * mag + 1e-30))
    assert float((got - ref).norm() / ref.norm()) <= 2e-3


def _block():
    """Matrices of several tile shapes, a 1-D vector between two of them (not
    in tile order, skipped by the product), and a matrix too small to be
    tiled."""
    return [workloads.normal_matrix(256, 128, 0.02, seed=1), workloads.normal_matrix(128, 320, 0.03, seed=2),
            workloads.normal_matrix(1, 512, 0.05, seed=3).reshape(-1), workloads.normal_matrix(384, 192, 0.02, seed=4),
            workloads.normal_matrix(100, 64, 0.02, seed=5)]


@pytest.mark.parametrize("T", [1, 5, 16, 64, 200, 256])
def test_fused_gemm_small_block(T):
    dev = _dev()
    mats = _block()
    d = df11.encode_multi(mats, tile_order=True).to(dev)
    idx = [j for j in range(len(mats)) if d.tiled[j]]
    assert idx == [0, 1, 3]
    xs = {j: _x(T, mats[j].shape[1], 100 + j) for j in idx}
    ys = df11.decode_gemm(d, {j: _bf16(xs[j]).to(dev) for j in idx})
    for j in idx:
        assert ys[j].shape == (T, mats[j].shape[0])
        _check(ys[j], mats[j], xs[j])


@pytest.mark.parametrize("T", [16, 64])
def test_fused_gemm_row_tiles_shared_by_ctas(T):
    """Enough k-tiles that each CTA's range starts and ends inside row tiles
    (partial sums added by two CTAs) and the tile ring wraps many times: a
    1024 x 4096 and a 4096 x 1024 matrix (1024 k-tiles over at most 148 CTAs)."""
    dev = _dev()
    mats = [workloads.normal_matrix(1024, 4096, 0.02, seed=11), workloads.normal_matrix(4096, 1024, 0.03, seed=12)]
    d = df11.encode_multi(mats, tile_order=True).to(dev)
    xs = {j: _x(T, mats[j].shape[1], 200 + j) for j in (0, 1)}
    ys = df11.decode_gemm(d, {j: _bf16(xs[j]).to(dev) for j in (0, 1)})
    for j in (0, 1):
        _check(ys[j], mats[j], xs[j])
    # only the second matrix, added into a y that already holds values
    y1 = torch.full((T, 4096), 0.5, dtype=torch.float32, device=dev)
    df11.decode_gemm(d, {1: _bf16(xs[1]).to(dev)}, ys={1: y1})
    ref = _bf16(xs[1]).double() @ _bf16(mats[1]).double().T + 0.5
    assert float((y1.cpu().double() - ref).norm() / ref.norm()) <= 2e-3


def test_fused_gemm_long_codes():
    """Uncapped codes (up to about 27 bits) through the long-code instance."""
    dev = _dev()
    rng = np.random.default_rng(3)
    x = (rng.standard_t(3, (512, 1024)) * 0.015).astype(np.float32)
    x[rng.random(x.shape) < 0.001] *= 1000.0
    w = workloads.round_to_bf16(x)
    t = df11.encode_multi([w], df11.Params(max_code_len=32), tile_order=True)
    assert t.code_len.max() > 12
    d = t.to(dev)
    for T in (8, 64):
        xb = _x(T, 1024, 40 + T)
        y = df11.decode_gemm(d, {0: _bf16(xb).to(dev)})[0]
        _check(y, w, xb)


def test_fused_gemm_matches_decode_then_gemm():
    """The fused product equals (to FP32 rounding) the unfused path: decode
    the tile-ordered block, put the matrix back in row order, run the
    consumer GEMM."""
    dev = _dev()
    w = workloads.normal_matrix(512, 1024, 0.02, seed=21)
    d = df11.encode_multi([w], tile_order=True).to(dev)
    dec = df11.decode(d).view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(df11.from_tile_order(dec, 512, 1024), w)
    xb = _x(32, 1024, 7)
    yf = df11.decode_gemm(d, {0: _bf16(xb).to(dev)})[0]
    yu = df11.gemm(_bf16(xb).to(dev), _bf16(w).to(dev))
    assert float((yf - yu).norm() / yu.norm()) <= 1e-5


def test_fused_gemm_corrupt_stream_reported():
    """Scrambled code bytes: the decoder's checks report it, the kernel still
    finishes (every tile completes)."""
    dev = _dev()
    w = workloads.normal_matrix(512, 512, 0.02, seed=8)
    d = df11.encode_multi([w], tile_order=True).to(dev)
    d.arrays["enc"][1000:1100] ^= 0x5A
    with pytest.raises(df11.CorruptStreamError):
        df11.decode_gemm(d, {0: _bf16(_x(16, 512, 1)).to(dev)})


def test_fused_gemm_bad_block_start_aborts_quickly():
    """A block start that breaks the order of the block starts: the block
    cannot be placed, the CTA gives up its waits at once and the error is
    reported (no wait runs into its limit)."""
    import time
    dev = _dev()
    w = workloads.normal_matrix(512, 512, 0.02, seed=6)
    d = df11.encode_multi([w], tile_order=True).to(dev)
    bs = d.arrays["block_start"].view(torch.int32)
    bs[3] = bs[5] + 100  # block 2 ends after block 3 does
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    t0 = time.time()
    df11.decode_gemm(d, {0: _bf16(_x(16, 512, 1)).to(dev)}, err=err)
    torch.cuda.synchronize()
    assert time.time() - t0 < 5.0
    assert int(err.item()) != 0


@pytest.mark.slow
@pytest.mark.parametrize("T", [16, 64, 256])
def test_fused_gemm_llama_block(T):
    """The Llama-3.1-8B-shaped block (seven matrices in tile order, the two
    norm vectors between them), one launch for all seven products; 256
    sampled rows of each output (the first and last among them) against FP64."""
    dev = _dev()
    mats = workloads.llama8b_block(seed=0)
    d = df11.encode_multi(mats, tile_order=True).to(dev)
    idx = [j for j in range(len(mats)) if d.tiled[j]]
    assert len(idx) == 7
    xs = {j: _x(T, mats[j].shape[1], 1000 + T + j) for j in idx}
    ys = df11.decode_gemm(d, {j: _bf16(xs[j]).to(dev) for j in idx})
    rng = np.random.default_rng(T)
    for j in idx:
        rows = np.unique(np.concatenate([[0, mats[j].shape[0] - 1], rng.integers(0, mats[j].shape[0], 254)]))
        _check(ys[j], mats[j], xs[j], rows)
