"""Fused decode -> matrix-vector products (df11_decode_gemv, T <= 4) against
an FP64 CPU product of the original weights (the codec is lossless, so the
decoded weights are the original ones).

Every output is held to the FP32 rounding bound of a sum in any order: the
products of two BF16 values are exact in FP32 and only the additions round,
so |y - ref| <= (n + 32) * 2^-24 * sum_c |w_rc x_c| for n = cols terms (the
32 covers the warp reduction and the atomic adds into y).  A dropped, doubled
or misplaced weight breaks the bound by orders of magnitude."""
import numpy as np
import pytest

import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import huffman_decode_02_b200 as df11  # noqa: E402

U = 2.0 ** -24


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _f64(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double()


def _bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _x(T: int, cols: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return workloads.round_to_bf16(rng.standard_normal((T, cols), dtype=np.float32))


def _check(y: torch.Tensor, w_bits: np.ndarray, x_bits: np.ndarray, y0: torch.Tensor | None = None,
           rows=None):
    """y (device, [T, rows]) against x W^T (+ y0) in FP64, within the bound."""
    W = _f64(w_bits if rows is None else w_bits[rows])
    X = _f64(x_bits)
    ref = X @ W.T
    mag = X.abs() @ W.abs().T
    got = y.cpu().double()
    if rows is not None:
        got = got[:, rows]
    if y0 is not None:
        base = y0.cpu().double() if rows is None else y0.cpu().double()[:, rows]
        ref = ref + base
        mag = mag + base.abs()
    n = w_bits.shape[1]
    bound = (n + 32) * U * mag + 1e-30
    err = (got - ref).abs()
    assert bool(torch.all(err <= bound)), f"max err/bound {float((err / bound).max()):.3g}"


def _block():
    """Matrices of several shapes with a 1-D vector between them (skipped by
    the product), a one-row matrix and a 16-column one; about 50 format
    blocks with a ragged last one."""
    return [workloads.normal_matrix(512, 256, 0.02, seed=1), workloads.normal_matrix(256, 512, 0.03, seed=2),
            workloads.normal_matrix(1, 256, 0.05, seed=3).reshape(-1), workloads.normal_matrix(48, 1024, 0.02, seed=4),
            workloads.normal_matrix(1, 1024, 0.02, seed=5), workloads.normal_matrix(300, 16, 0.02, seed=6)]


@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_fused_block_all_matrices(T):
    dev = _dev()
    mats = _block()
    d = df11.encode_multi(mats).to(dev)
    idx = [j for j, m in enumerate(mats) if m.ndim == 2]
    xs_np = {j: _x(T, mats[j].shape[1], 100 + j) for j in idx}
    for dd in (d, d.without_counts()):  # stored counts, and the count pass
        ys = df11.decode_gemv(dd, {j: _bf16(xs_np[j]).to(dev) for j in idx})
        torch.cuda.synchronize()
        assert sorted(ys) == idx
        for j in idx:
            assert ys[j].shape == (T, mats[j].shape[0]) and ys[j].dtype == torch.float32
            _check(ys[j], mats[j], xs_np[j])


def test_fused_subset_accumulates_into_y():
    """Only matrices 1 and 3; y holds values on entry and the product is
    added to them."""
    dev = _dev()
    mats = _block()
    d = df11.encode_multi(mats).to(dev)
    T = 2
    xs_np = {j: _x(T, mats[j].shape[1], 200 + j) for j in (1, 3)}
    y0 = {j: torch.randn(T, mats[j].shape[0], dtype=torch.float32) for j in (1, 3)}
    ys = {j: y0[j].clone().to(dev) for j in (1, 3)}
    out = df11.decode_gemv(d, {j: _bf16(xs_np[j]).to(dev) for j in (1, 3)}, ys)
    torch.cuda.synchronize()
    for j in (1, 3):
        assert out[j].data_ptr() == ys[j].data_ptr()
        _check(out[j], mats[j], xs_np[j], y0=y0[j])


def test_fused_matches_decode_then_gemv():
    """The fused call and the unfused path (decode, then the T <= 4 GEMM)
    agree within the sum of their bounds on one matrix of a block."""
    dev = _dev()
    mats = _block()
    d = df11.encode_multi(mats).to(dev)
    x_np = _x(4, 512, 7)
    x = _bf16(x_np).to(dev)
    fused = df11.decode_gemv(d, {1: x})[1]
    w = d.views(df11.decode_block(d))[1]
    y = df11.gemm(x, w.contiguous())
    torch.cuda.synchronize()
    mag = _f64(x_np).abs() @ _f64(mats[1]).abs().T
    assert bool(torch.all((fused.cpu().double() - y.cpu().double()).abs() <= 2 * (512 + 32) * U * mag + 1e-30))


def test_fused_long_codes():
    """Codes longer than the table windows (uncapped heavy tail): the
    long-code instance."""
    dev = _dev()
    rng = np.random.default_rng(3)
    x = (rng.standard_t(3, (600, 1024)) * 0.015).astype(np.float32)
    x[rng.random(x.shape) < 0.001] *= 1000.0
    w = workloads.round_to_bf16(x)
    t = df11.encode(w, df11.Params(max_code_len=32))
    assert t.code_len.max() > 12
    d = t.to(dev)
    for T in (1, 3):
        xb = _x(T, 1024, 30 + T)
        y = df11.decode_gemv(d, {0: _bf16(xb).to(dev)})[0]
        _check(y, w, xb)


@pytest.mark.parametrize("kind", ["dense", "wide"])
def test_fused_other_instances(kind):
    """Blocks with more codes than the typical instance holds: 1-bit codes
    (a two-valued matrix) and a five-exponent matrix."""
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
    for dd in (d, d.without_counts()):  # stored counts, and the count pass
        for T in (1, 4):
            xb = _x(T, 96, 40 + T)
            y = df11.decode_gemv(dd, {0: _bf16(xb).to(dev)})[0]
            _check(y, w, xb)


def test_fused_argument_checks():
    dev = _dev()
    mats = _block()
    d = df11.encode_multi(mats).to(dev)
    x = torch.zeros(5, 256, dtype=torch.bfloat16, device=dev)
    with pytest.raises(df11.DF11Error):
        df11.decode_gemv(d, {0: x})  # T = 5
    with pytest.raises(TypeError):
        df11.decode_gemv(d, {0: torch.zeros(1, 255, dtype=torch.bfloat16, device=dev)})  # wrong in
    with pytest.raises(ValueError):
        df11.decode_gemv(d, {2: torch.zeros(1, 256, dtype=torch.bfloat16, device=dev)})  # a 1-D vector
    # a matrix whose offset is not a multiple of 16
    odd = [workloads.normal_matrix(1, 8, 0.02, seed=1).reshape(-1), workloads.normal_matrix(32, 64, 0.02, seed=2)]
    d2 = df11.encode_multi(odd).to(dev)
    with pytest.raises(df11.DF11Error):
        df11.decode_gemv(d2, {1: torch.zeros(1, 64, dtype=torch.bfloat16, device=dev)})
    # more than 16 matrices in one call
    many = [workloads.normal_matrix(16, 16, 0.02, seed=s) for s in range(17)]
    d3 = df11.encode_multi(many).to(dev)
    with pytest.raises(df11.DF11Error):
        df11.decode_gemv(d3, {j: torch.zeros(1, 16, dtype=torch.bfloat16, device=dev) for j in range(17)})
    # 16 matrices are accepted
    xs16 = {j: _bf16(_x(1, 16, j)).to(dev) for j in range(16)}
    ys16 = df11.decode_gemv(d3, xs16)
    for j in range(16):
        _check(ys16[j], many[j], _x(1, 16, j))
    assert df11.decode_gemv(d, {}) == {}


def test_fused_corrupt_stream_reported():
    dev = _dev()
    w = workloads.normal_matrix(512, 512, 0.02, seed=8)
    d = df11.encode(w).to(dev)
    d.arrays["enc"][1000:1100] ^= 0x5A
    with pytest.raises(df11.CorruptStreamError):
        df11.decode_gemv(d, {0: torch.zeros(1, 512, dtype=torch.bfloat16, device=dev)})


@pytest.mark.slow
@pytest.mark.parametrize("T", [1, 4])
def test_fused_llama_block(T):
    """The Llama-3.1-8B-shaped block: all seven matrices in one call (the
    bench's launch), 256 sampled rows of each checked; then each matrix on
    its own (only its thread blocks decoded)."""
    dev = _dev()
    mats = workloads.llama8b_block(seed=0)
    d = df11.encode_multi(mats).to(dev)
    idx = [j for j, m in enumerate(mats) if m.ndim == 2]
    xs_np = {}
    for j in idx:
        xs_np.setdefault(mats[j].shape[1], _x(T, mats[j].shape[1], 1000 + T))
    xs = {j: _bf16(xs_np[mats[j].shape[1]]).to(dev) for j in idx}
    ys = df11.decode_gemv(d, xs)
    torch.cuda.synchronize()
    rng = np.random.default_rng(11)
    for j in idx:
        rows = np.sort(rng.choice(mats[j].shape[0], 256, replace=False))
        _check(ys[j], mats[j], xs_np[mats[j].shape[1]], rows=rows)
    for j in (idx[1], idx[-1]):
        yj = df11.decode_gemv(d, {j: xs[j]})[j]
        rows = np.sort(rng.choice(mats[j].shape[0], 256, replace=False))
        _check(yj, mats[j], xs_np[mats[j].shape[1]], rows=rows)


@pytest.mark.slow
def test_fused_lm_head_shape():
    """The LM-head / embedding shape (128256 x 4096, 525 M weights, one
    matrix): T = 1 and 4, 512 sampled rows (the last ones among them)."""
    dev = _dev()
    w = workloads.normal_matrix(128256, 4096, 0.02, seed=5)
    d = df11.encode(w).to(dev)
    rng = np.random.default_rng(13)
    rows = np.unique(np.concatenate([rng.choice(128256, 504, replace=False), np.arange(128248, 128256)]))
    for T in (1, 4):
        xb = _x(T, 4096, 50 + T)
        y = df11.decode_gemv(d, {0: _bf16(xb).to(dev)})[0]
        _check(y, w, xb, rows=rows)
