"""The consumer GEMM (tcgen05 for T > 4, a CUDA-core matrix-vector stream
for T <= 4; FP32 accumulation) against a CPU GEMM: the relative Frobenius
error must stay within 2e-3.  Inputs are BF16, so every
product is exact in FP32 and the two sides differ only in summation order."""
import numpy as np
import pytest

import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import huffman_decode_02_b200 as df11  # noqa: E402

TOL = 2e-3


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def _rel_fro(y, ref):
    return float(np.linalg.norm(y - ref) / np.linalg.norm(ref))


def _check(T, out, inn, seed):
    dev = _dev()
    rng = np.random.default_rng(seed)
    x = workloads.round_to_bf16(rng.standard_normal((T, inn), dtype=np.float32))
    w = workloads.round_to_bf16(rng.standard_normal((out, inn), dtype=np.float32) * np.float32(0.02))
    xt, wt = _bf16(x), _bf16(w)
    ref = xt.double() @ wt.double().T  # CPU reference
    y = df11.gemm(xt.to(dev), wt.to(dev))
    torch.cuda.synchronize()
    assert y.shape == (T, out) and y.dtype == torch.float32
    assert _rel_fro(y.cpu().double().numpy(), ref.numpy()) <= TOL


@pytest.mark.parametrize("T", [1, 16, 64, 256])
def test_gemm_q_proj_shape(T):
    _check(T, 4096, 4096, seed=1000 + T)


@pytest.mark.parametrize("T,out,inn", [(5, 1024, 4096), (33, 128, 64), (256, 14336, 4096), (16, 4096, 14336),
                                       (200, 256, 128), (1, 14336, 4096), (2, 4096, 14336), (3, 1024, 4096),
                                       (4, 128, 64), (4, 256, 128)])
def test_gemm_other_shapes(T, out, inn):
    _check(T, out, inn, seed=T + out)


def test_gemm_rejects_unsupported():
    dev = _dev()
    x = torch.zeros(4, 100, dtype=torch.bfloat16, device=dev)
    w = torch.zeros(128, 100, dtype=torch.bfloat16, device=dev)
    with pytest.raises(df11.DF11Error):
        df11.gemm(x, w)  # in not a multiple of 64
    x = torch.zeros(300, 64, dtype=torch.bfloat16, device=dev)
    w = torch.zeros(128, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(df11.DF11Error):
        df11.gemm(x, w)  # T > 256


def test_decode_then_gemm_from_scratch():
    """Decode a small block into a scratch buffer, multiply straight from the
    matrix views (the decode -> consumer path)."""
    dev = _dev()
    mats = [workloads.normal_matrix(512, 256, 0.02, seed=1), workloads.normal_matrix(256, 512, 0.03, seed=2)]
    blk = df11.encode_multi(mats).to(dev)
    scratch = df11.decode_block(blk)
    views = blk.views(scratch)
    rng = np.random.default_rng(9)
    for w, v in zip(mats, views):
        x = workloads.round_to_bf16(rng.standard_normal((64, w.shape[1]), dtype=np.float32))
        xt = _bf16(x)
        y = df11.gemm(xt.to(dev), v.contiguous())
        ref = xt.double() @ _bf16(w).double().T
        assert _rel_fro(y.cpu().double().numpy(), ref.numpy()) <= TOL


@pytest.mark.slow
def test_config5_decode_then_gemm_full_blocks():
    """Llama-8B-shaped blocks (seeds 0 and 31 of the 32-block sequence) decoded
    one after the other into the same scratch, each matrix multiplied by
    N(0,1) BF16 activations [T, in] (seed 1000 + T) for T in {1, 16, 64, 256};
    512 sampled output columns per product are checked against an FP64 CPU
    GEMM of the original weights."""
    dev = _dev()
    names = ["q", "k", "v", "o", "gate", "up", "down"]
    scratch = None
    rng_cols = np.random.default_rng(5)
    for seed in (0, 31):
        mats = workloads.llama8b_block(seed=seed)
        blk = df11.encode_multi(mats).to(dev)
        if scratch is None:
            scratch = torch.empty(blk.n_elems, dtype=torch.bfloat16, device=dev)
        df11.decode_block(blk, scratch)
        views = blk.views(scratch)
        for T in (1, 16, 64, 256):
            xs = {}
            for name, w, v in zip(names, mats, views):
                inn = w.shape[1]
                if inn not in xs:
                    r = np.random.default_rng(1000 + T)
                    xs[inn] = _bf16(workloads.round_to_bf16(r.standard_normal((T, inn), dtype=np.float32)))
                y = df11.gemm(xs[inn].to(dev), v).cpu().double().numpy()
                cols = rng_cols.choice(w.shape[0], 512, replace=False)
                ref = (xs[inn].double() @ _bf16(w[cols]).double().T).numpy()
                assert _rel_fro(y[:, cols], ref) <= TOL, (seed, T, name)


@pytest.mark.slow
@pytest.mark.parametrize("T", [1, 16])
def test_gemm_lm_head_shape(T):
    """The LM-head shape (128256 x 4096): the widest grid of either path
    (64128 GEMV CTAs at T = 1; 1002 row tiles on tcgen05 at T = 16).  1024
    sampled output columns against an FP64 CPU GEMM."""
    dev = _dev()
    g = torch.Generator(device=dev).manual_seed(40 + T)
    w = (torch.randn(128256, 4096, device=dev, generator=g) * 0.02).to(torch.bfloat16)
    x = torch.randn(T, 4096, device=dev, generator=g).to(torch.bfloat16)
    y = df11.gemm(x, w)
    cols = torch.from_numpy(np.random.default_rng(T).choice(128256, 1024, replace=False)).to(dev)
    ref = (x.double() @ w[cols].double().T).cpu().numpy()
    assert _rel_fro(y[:, cols].double().cpu().numpy(), ref) <= TOL


def _mats(shapes, T, seed):
    rng = np.random.default_rng(seed)
    out = []
    for o, i in shapes:
        x = workloads.round_to_bf16(rng.standard_normal((T, i), dtype=np.float32))
        w = workloads.round_to_bf16(rng.standard_normal((o, i), dtype=np.float32) * np.float32(0.02))
        out.append((x, w))
    return out


def _check_multi(shapes, T, seed, rows=None):
    """gemm_multi against FP64 per product: every output within the FP32
    accumulation bound (K + 64) * 2^-23 * sum |w x| and the relative
    Frobenius error within 2e-3.  `rows`: sampled output rows per product."""
    dev = _dev()
    data = _mats(shapes, T, seed)
    pairs = [(_bf16(x).to(dev), _bf16(w).to(dev)) for x, w in data]
    ys = df11.gemm_multi(pairs)
    torch.cuda.synchronize()
    for (x, w), y in zip(data, ys):
        X, W = _bf16(x).double(), _bf16(w).double()
        got = y.cpu().double()
        if rows is not None:
            r = np.unique(np.concatenate([[0, w.shape[0] - 1], np.random.default_rng(seed).integers(0, w.shape[0], rows)]))
            W, got = W[torch.as_tensor(r)], got[:, torch.as_tensor(r)]
        ref, mag = X @ W.T, X.abs() @ W.abs().T
        assert bool(torch.all((got - ref).abs() <= (w.shape[1] + 64) * 2.0 ** -23 * mag + 1e-30))
        assert float((got - ref).norm() / ref.norm()) <= TOL


@pytest.mark.parametrize("T", [5, 16, 17, 64, 200, 256])
def test_gemm_multi_mixed_shapes(T):
    """Products of several shapes in one launch: row tiles split between
    CTAs (partial sums added), matrices smaller than a CTA's share, a
    single-tile matrix, T not a multiple of 16."""
    _check_multi([(256, 128), (128, 64), (1024, 4096), (384, 192), (128, 1024)], T, seed=T)


@pytest.mark.parametrize("T", [5, 16, 33, 64, 128])
def test_gemm_multi_two_tiles_per_stage(T):
    """Every product with an even number of k-tiles per row tile: stages of
    two k-tiles (a stage may end one row tile and start the next)."""
    _check_multi([(256, 128), (1024, 4096), (128, 1024), (512, 256), (128, 128)], T, seed=50 + T)


@pytest.mark.parametrize("T", [1, 4])
def test_gemm_multi_matrix_vector(T):
    _check_multi([(256, 128), (1024, 4096)], T, seed=10 + T)


@pytest.mark.slow
@pytest.mark.parametrize("T", [16, 64, 256])
def test_gemm_multi_llama_block(T):
    """The seven Llama-3.1-8B block shapes in one launch; 256 sampled rows
    of each output (first and last among them) against FP64."""
    shapes = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096), (4096, 14336)]
    _check_multi(shapes, T, seed=100 + T, rows=254)


def test_gemm_multi_overwrites_y():
    """Y is overwritten (zeroed, then the partial sums added), not added into."""
    dev = _dev()
    data = _mats([(512, 2048)], 32, 7)
    x, w = (_bf16(a).to(dev) for a in data[0])
    y = torch.full((32, 512), 3.0, dtype=torch.float32, device=dev)
    df11.gemm_multi([(x, w)], outs=[y])
    ref = _bf16(data[0][0]).double() @ _bf16(data[0][1]).double().T
    assert float((y.cpu().double() - ref).norm() / ref.norm()) <= TOL


def test_gemm_multi_rejects_unsupported():
    dev = _dev()
    x = torch.zeros(16, 64, dtype=torch.bfloat16, device=dev)
    w = torch.zeros(100, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(df11.DF11Error):
        df11.gemm_multi([(x, w)])
    x2 = torch.zeros(300, 64, dtype=torch.bfloat16, device=dev)
    w2 = torch.zeros(128, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(df11.DF11Error):
        df11.gemm_multi([(x2, w2)])
