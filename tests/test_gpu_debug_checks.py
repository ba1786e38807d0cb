"""The decode, block-decode, row-gather and fused decode -> matrix-vector
kernels built with every
data-dependent shared-memory index and global store address checked
(libdf11_debug.so): on adversarial inputs, all length caps, ragged sizes and
the long-code path, no check fails and the output stays bit-exact."""
import ctypes

import numpy as np
import pytest

import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import huffman_decode_02_b200 as df11  # noqa: E402
from huffman_decode_02_b200 import build as df11_build  # noqa: E402


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(scope="module")
def debug_lib():
    _dev()
    path = df11_build.build(debug=True)
    saved_lib, saved_path = df11._LIB, df11_build.LIB_PATH
    df11._LIB = None
    df11_build.LIB_PATH = path
    lib = df11._lib()  # same ABI checks as the product library
    lib.df11_debug_bounds_errors.restype = ctypes.c_uint32
    lib.df11_debug_bounds_errors.argtypes = [ctypes.c_int]
    lib.df11_debug_bounds_errors(1)
    yield lib
    df11._LIB, df11_build.LIB_PATH = saved_lib, saved_path


def _bits(x):
    return x.view(torch.int16).cpu().numpy().view(np.uint16)


def _cases():
    for name in workloads.ADVERSARIAL_NAMES:
        yield name, workloads.adversarial(name), df11.Params()
    fib = workloads.adversarial("fibonacci_exponents")
    for cap in (8, 16, 32):
        yield f"fib-cap{cap}", fib, df11.Params(max_code_len=cap)
    rng = np.random.default_rng(3)
    x = (rng.standard_t(3, (300, 1024)) * 0.015).astype(np.float32)
    x[rng.random(x.shape) < 0.001] *= 1000.0
    yield "heavy-cap32", workloads.round_to_bf16(x), df11.Params(max_code_len=32)
    yield "normal-1024", workloads.normal_matrix(1024, 1024, 0.02, seed=0), df11.Params()


def test_decode_paths_without_bounds_errors(debug_lib):
    dev = _dev()
    for name, w, p, counts in ((n, w, p, c) for n, w, p in _cases() for c in (True, False)):
        w = np.ascontiguousarray(w).reshape(-1).view(np.uint16)
        d = df11.encode(w, p).to(dev)
        d = d if counts else d.without_counts()  # stored counts, and the count pass
        name = f"{name}-{'counts' if counts else 'count-pass'}"
        np.testing.assert_array_equal(_bits(df11.decode(d)), w, err_msg=name)
        if w.size >= 64 and w.size % 64 == 0:  # as a 64-column matrix: row gather
            rows = torch.arange(0, w.size // 64, 7, dtype=torch.int32, device=dev)
            got = _bits(df11.decode_rows(d, 64, rows))
            np.testing.assert_array_equal(got, w.reshape(-1, 64)[rows.cpu().numpy()], err_msg=name)
            # and the fused matrix-vector product (T = 1, 2 and 3; values are
            # checked elsewhere, adversarial inputs hold NaN and Inf)
            for T in (1, 2, 3):
                x = torch.randn(T, 64, generator=torch.Generator().manual_seed(T)).to(torch.bfloat16).to(dev)
                df11.decode_gemv(df11.DF11Tensor(d.desc, d.arrays, d.device, [(w.size // 64, 64)], [0, w.size]),
                                 {0: x})
        assert debug_lib.df11_debug_bounds_errors(1) == 0, name
    mats = [workloads.normal_matrix(r, c, s, seed=i) for i, (r, c, s) in
            enumerate([(512, 256, 0.02), (64, 128, 0.03), (3, 7, 0.5)])]
    blk = df11.encode_multi(mats).to(dev)
    for b in (blk, blk.without_counts()):
        scratch = df11.decode_block(b)
        for m, v in zip(mats, b.views(scratch)):
            np.testing.assert_array_equal(_bits(v).reshape(m.shape), m)
    for T in (1, 4):  # the fused product over the two 2-D matrices (in = 256, 128)
        xs = {j: torch.randn(T, mats[j].shape[1], generator=torch.Generator().manual_seed(j)).to(torch.bfloat16)
              .to(dev) for j in (0, 1)}
        ys = df11.decode_gemv(blk, xs)
        for j in (0, 1):
            w64 = torch.from_numpy(mats[j].view(np.int16)).view(torch.bfloat16).double()
            ref = xs[j].cpu().double() @ w64.T
            assert float((ys[j].cpu().double() - ref).norm() / ref.norm()) < 1e-5
    assert debug_lib.df11_debug_bounds_errors(1) == 0


def test_fused_gemm_without_bounds_errors(debug_lib):
    """The fused decode -> tensor-core GEMM through the bounds-checked build
    (every data-dependent shared-memory index of its decoder, the tile-ring
    stores included): no failed check, the product within 2e-3."""
    dev = _dev()
    mats = [workloads.normal_matrix(256, 128, 0.02, seed=1), workloads.normal_matrix(1, 64, 0.02, seed=2)[0],
            workloads.normal_matrix(512, 320, 0.03, seed=3)]
    rng = np.random.default_rng(5)
    x = (rng.standard_t(3, (256, 512)) * 0.015).astype(np.float32)
    x[rng.random(x.shape) < 0.001] *= 1000.0
    for blk_mats, p in ((mats, df11.Params()), ([workloads.round_to_bf16(x)], df11.Params(max_code_len=32))):
        blk = df11.encode_multi(blk_mats, p, tile_order=True).to(dev)
        idx = [j for j in range(len(blk_mats)) if blk.tiled[j]]
        for T in (16, 96):
            xs = {j: torch.randn(T, blk_mats[j].shape[1], generator=torch.Generator().manual_seed(j))
                  .to(torch.bfloat16).to(dev) for j in idx}
            ys = df11.decode_gemm(blk, xs)
            for j in idx:
                w64 = torch.from_numpy(np.ascontiguousarray(blk_mats[j]).view(np.int16)).view(torch.bfloat16).double()
                ref = xs[j].cpu().double() @ w64.T
                assert float((ys[j].cpu().double() - ref).norm() / ref.norm()) < 2e-3
    assert debug_lib.df11_debug_bounds_errors(1) == 0
