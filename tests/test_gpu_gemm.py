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
