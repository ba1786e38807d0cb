"""The no-allocation device-encoder entry points (fixed scratch inside the
library) against the caller-scratch entry points: identical descriptors and
arrays on two different inputs encoded one after the other (the second call
must not see the first one's scratch contents), and inputs beyond the fixed
scratch refused before any GPU work.  Collected last on purpose: it must
pass alone and after every other test."""
import ctypes

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


def _same(a: df11.DF11Tensor, b: df11.DF11Tensor):
    for f in FIELDS:
        assert getattr(a.desc, f) == getattr(b.desc, f), f
    assert bytes(a.desc.code_len) == bytes(b.desc.code_len)
    for k in ("enc", "sm", "gaps", "block_start", "lut", "counts"):
        np.testing.assert_array_equal(a.host_array(k).view(np.uint8)[: a.nbytes(k)],
                                      b.host_array(k).view(np.uint8)[: b.nbytes(k)], err_msg=k)


def test_two_calls_in_a_row_match_caller_scratch():
    dev = _dev()
    first = workloads.normal_matrix(2048, 1024, 0.02, seed=31)            # 2.1M weights
    second = workloads.adversarial("fibonacci_exponents")[:1_000_003]      # other code, ragged size
    for w, p in ((first, df11.Params()), (second, df11.Params(max_code_len=8))):
        t = torch.from_numpy(np.ascontiguousarray(w).reshape(-1).view(np.int16)).to(dev).view(torch.bfloat16)
        got = df11.encode_device_noalloc(t, p)
        _same(df11.encode_device(t, p), got)
        np.testing.assert_array_equal(df11.decode(got).view(torch.int16).cpu().numpy().view(np.uint16),
                                      np.ascontiguousarray(w).reshape(-1))


def test_too_large_refused_before_gpu_work():
    dev = _dev()
    lib = df11._lib()
    cap = int(lib.df11_encode_device_noalloc_max_elems())
    assert cap == 1 << 28
    buf = torch.zeros(16, dtype=torch.int16, device=dev)
    desc = df11._Tensor()
    pc = df11.Params()._c()
    st = lib.df11_encode_device_size_noalloc(ctypes.c_void_p(buf.data_ptr()), cap + 1, ctypes.byref(pc),
                                             ctypes.byref(desc), ctypes.c_void_p(0))
    assert st == 3  # DF11_ERR_TOO_LARGE


def test_too_large_refused_by_the_fill_call():
    """The fill call checks its own size limit too (before any GPU work)."""
    dev = _dev()
    lib = df11._lib()
    cap = int(lib.df11_encode_device_noalloc_max_elems())
    buf = torch.zeros(16, dtype=torch.int16, device=dev)
    desc = df11._Tensor()
    st = lib.df11_encode_device_noalloc(ctypes.c_void_p(buf.data_ptr()), cap + 1, ctypes.byref(desc),
                                        ctypes.c_void_p(0))
    assert st == 3  # DF11_ERR_TOO_LARGE


def test_host_pointer_refused():
    """Weights must be memory of the current device; a host pointer is an
    argument error, reported before anything is enqueued."""
    _dev()
    lib = df11._lib()
    host = np.zeros(4096, dtype=np.uint16)
    desc = df11._Tensor()
    pc = df11.Params()._c()
    st = lib.df11_encode_device_size_noalloc(ctypes.c_void_p(host.ctypes.data), host.size, ctypes.byref(pc),
                                             ctypes.byref(desc), ctypes.c_void_p(0))
    assert st == 1  # DF11_ERR_INVALID_ARG


@pytest.mark.slow
def test_llama_block_near_capacity_matches_caller_scratch():
    """A whole Llama-3.1-8B-shaped block (218,112,000 weights, 81 % of the
    fixed scratch's 2^28-weight limit, so the tile-offset region is filled
    far into its end) encoded without allocation, byte for byte against the
    caller-scratch encoder."""
    dev = _dev()
    mats = workloads.llama8b_block(seed=0)
    flat = np.concatenate([np.ascontiguousarray(m).reshape(-1) for m in mats])
    t = torch.from_numpy(flat.view(np.int16)).to(dev).view(torch.bfloat16)
    got = df11.encode_device_noalloc(t)
    _same(df11.encode_device(t), got)
    del got
    torch.cuda.empty_cache()
