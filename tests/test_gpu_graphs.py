"""The device calls inside CUDA graphs: each is captured once (after one
ordinary call, which makes the library's one-time settings) and replayed;
the replays give the same results as the ordinary calls.  This is how a
serving loop removes the per-call host cost of launch-bound steps."""
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


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _mats():
    return [workloads.normal_matrix(512, 256, 0.02, seed=1), workloads.normal_matrix(256, 512, 0.03, seed=2),
            workloads.normal_matrix(1, 256, 0.05, seed=3).reshape(-1), workloads.normal_matrix(128, 1024, 0.02, seed=4)]


def test_block_decode_replayed_from_a_graph():
    dev = _dev()
    mats = _mats()
    d = df11.encode_multi(mats).to(dev)
    out = torch.empty(d.n_elems, dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        df11.decode_block(d, out, err)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        df11.decode_block(d, out, err)
    want = np.concatenate([m.reshape(-1) for m in mats])
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), want)
    assert df11.read_error(err) == 0


def test_fused_gemv_replayed_from_a_graph():
    """Zeroing of y and the fused call, captured together."""
    dev = _dev()
    mats = _mats()
    d = df11.encode_multi(mats).to(dev)
    idx = [0, 1, 3]
    rng = np.random.default_rng(5)
    xs_np = {j: workloads.round_to_bf16(rng.standard_normal((2, mats[j].shape[1]), dtype=np.float32)) for j in idx}
    xs = {j: _bf16(xs_np[j]).to(dev) for j in idx}
    ys = {j: torch.zeros(2, mats[j].shape[0], device=dev) for j in idx}
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        df11.decode_gemv(d, xs, ys, err)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for j in idx:
            ys[j].zero_()
        df11.decode_gemv(d, xs, ys, err)
    for _ in range(3):
        for j in idx:
            ys[j].fill_(123.0)  # replaced by the replay's zeroing
        g.replay()
        torch.cuda.synchronize()
        for j in idx:
            W = torch.from_numpy(mats[j].view(np.int16)).view(torch.bfloat16).double()
            X = _bf16(xs_np[j]).double()
            bound = (mats[j].shape[1] + 32) * U * (X.abs() @ W.abs().T) + 1e-30
            assert bool(torch.all((ys[j].cpu().double() - X @ W.T).abs() <= bound))
    assert df11.read_error(err) == 0


@pytest.mark.parametrize("T", [1, 16])
def test_gemm_replayed_from_a_graph(T):
    """Both GEMM paths: the matrix-vector stream (T = 1) and the tcgen05
    kernel with split-K zeroing (T = 16)."""
    dev = _dev()
    rng = np.random.default_rng(T)
    w_np = workloads.normal_matrix(256, 1024, 0.02, seed=T)
    x_np = workloads.round_to_bf16(rng.standard_normal((T, 1024), dtype=np.float32))
    w, x = _bf16(w_np).to(dev), _bf16(x_np).to(dev)
    y = torch.empty(T, 256, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        df11.gemm(x, w, y, err)
    s.synchronize()
    first = y.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        df11.gemm(x, w, y, err)
    ref = _bf16(x_np).double() @ _bf16(w_np).double().T
    for _ in range(3):
        y.fill_(-7.0)
        g.replay()
        torch.cuda.synchronize()
        assert float((y.cpu().double() - ref).norm() / ref.norm()) <= 2e-3
        assert float((y - first).abs().max()) <= 1e-3 * float(first.abs().max())
    assert df11.read_error(err) == 0
