"""Streaming compressed blocks from pinned host memory (double-buffered
copy / decode): every decoded matrix bit-exact, in any block order."""
import numpy as np
import pytest

import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import huffman_decode_02_b200 as df11  # noqa: E402
from huffman_decode_02_b200.offload import BlockStreamer, RawStreamer  # noqa: E402
from huffman_decode_02_b200.pipeline import BlockPipeline  # noqa: E402


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _bits(x):
    return x.view(torch.int16).cpu().numpy().view(np.uint16)


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


def test_device_pipeline_bit_exact_with_repeats():
    """Device-resident blocks decoded one ahead of their consumer into two
    alternating scratch buffers: every view the consumer sees is the block's
    original matrix, for an order with repeats and both scratch slots reused."""
    dev = _dev()
    blocks = _blocks()
    devs = [df11.encode_multi(mats).to(dev) for mats in blocks]
    pipe = BlockPipeline(devs, dev)
    order = [0, 1, 2, 2, 0, 1, 0]
    seen = []

    def consumer(bi, views):
        seen.append((bi, [v.clone() for v in views]))

    pipe.run(order, consumer)
    pipe.check()
    torch.cuda.synchronize()
    assert [bi for bi, _ in seen] == order
    for bi, views in seen:
        for m, v in zip(blocks[bi], views):
            np.testing.assert_array_equal(_bits(v).reshape(m.shape), m)
    with pytest.raises(ValueError):
        BlockPipeline([df11.encode_multi(blocks[0])], dev)  # host tensors are refused

