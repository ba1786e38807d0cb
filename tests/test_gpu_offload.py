"""Streaming compressed blocks from pinned host memory (double-buffered
copy / decode): every decoded matrix bit-exact, in any block order."""
import numpy as np
import pytest

import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import huffman_decode_02_b200 as df11  # noqa: E402
from huffman_decode_02_b200.offload import BlockStreamer, RawStreamer  # noqa: E402


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _blocks():
    shapes = [[(256, 128), (64, 128), (3, 7)], [(512, 256), (128, 512)], [(100, 64), (64, 100), (1, 4096)]]
    return [[workloads.normal_matrix(r, c, 0.02 + 0.01 * j, seed=10 * i + j) for j, (r, c) in enumerate(sh)]
            for i, sh in enumerate(shapes)]


def test_block_streamer_bit_exact_any_order():
    dev = _dev()
    mats = _blocks()
    blocks = [df11.encode_multi(m, pinned=True) for m in mats]
    st = BlockStreamer(blocks, dev)
    got = []
    order = [0, 1, 2, 1, 0, 2, 2]
    st.run(order, lambda bi, views: got.append((bi, [v.clone() for v in views])))
    st.check()
    torch.cuda.synchronize()
    assert [bi for bi, _ in got] == order
    for bi, views in got:
        for m, v in zip(mats[bi], views):
            assert tuple(v.shape) == m.shape
            np.testing.assert_array_equal(v.view(torch.int16).cpu().numpy().view(np.uint16), m)


def test_raw_streamer_matches_host_arrays():
    dev = _dev()
    mats = _blocks()
    rs = RawStreamer(mats, dev)
    got = []
    rs.run([2, 0, 1], lambda bi, views: got.append((bi, [v.clone() for v in views])))
    torch.cuda.synchronize()
    for bi, views in got:
        for m, v in zip(mats[bi], views):
            np.testing.assert_array_equal(v.view(torch.int16).cpu().numpy().view(np.uint16), m)


def test_block_streamer_rejects_unpinned_blocks():
    _dev()
    blk = df11.encode_multi(_blocks()[0])  # numpy host arrays, not pinned
    with pytest.raises(ValueError):
        BlockStreamer([blk])
