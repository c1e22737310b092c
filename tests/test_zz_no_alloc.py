"""ep_compress_cuda_noalloc: the CUDA encoder with its device scratch in the library's fixed static area.

Collected last on purpose. Two calls in a row, on different tensors, must each write the same bytes as
ep_compress_cuda, so no state is left in the shared area between calls. The file passes alone and after
the rest of the suite.
"""
import ctypes

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ep():
    import decode_ep_b200 as m
    assert torch.cuda.is_available()
    m.lib()
    return m


def test_two_calls_in_a_row_match_the_allocating_entry_point(ep):
    w1 = synth.dit_layer(9, shape=(2048, 2048)).cuda()                       # about 4.2 M parameters
    w2 = synth.lognormal_rows_with_outliers(n=512, seed=21, outlier_frac=1e-3).cuda()  # escapes
    w3 = synth.gaussian(256, 512, seed=22, container="fp32").cuda()          # raw low bits at 9 bpp
    ref1 = ep.compress(w1, ep.EntroPackLossyConfig(4.0, encoder="cuda"))
    ref2 = ep.compress(w2, ep.EntroPackLossyConfig(4.0, encoder="cuda"))
    ref3 = ep.compress(w3, ep.EntroPackLossyConfig(9.0, rounds_per_tile=5, encoder="cuda"))
    a = ep.compress_cuda_noalloc(w1, 4.0)
    b = ep.compress_cuda_noalloc(w2, 4.0)
    c = ep.compress_cuda_noalloc(w3, ep.EntroPackLossyConfig(9.0, rounds_per_tile=5))
    a2 = ep.compress_cuda_noalloc(w1, 4.0)
    assert a.blob == ref1.blob and a2.blob == ref1.blob
    assert b.blob == ref2.blob
    assert c.blob == ref3.blob
    assert a.actual_bpp == ref1.actual_bpp
    y = ep.decompress(b)
    assert y.shape == w2.shape


def test_calls_allocate_no_device_memory(ep):
    """The property the entry point exists for: after a first call (which resolves the static area), further
    calls leave the device's free memory (cudaMemGetInfo) and the reserved size of the device's current
    memory pool unchanged."""
    from cuda.bindings import runtime as rt
    w = synth.gaussian(1024, 1024, seed=23, container="bf16").cuda()
    torch.cuda.synchronize()
    ep.compress_cuda_noalloc(w, 4.0)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    err, pool = rt.cudaDeviceGetMemPool(torch.cuda.current_device())
    assert err == rt.cudaError_t.cudaSuccess

    def pool_bytes():
        e, v = rt.cudaMemPoolGetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrReservedMemCurrent)
        assert e == rt.cudaError_t.cudaSuccess
        return int(v)

    reserved0 = pool_bytes()
    for _ in range(2):
        ep.compress_cuda_noalloc(w, 4.0)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert pool_bytes() == reserved0


def test_input_on_another_device_is_rejected(ep):
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two devices")
    w = synth.quickstart_256().to("cuda:1")
    buf = (ctypes.c_uint8 * (1 << 20))()
    nbytes, bpp = ctypes.c_size_t(), ctypes.c_double()
    opt = ep.EntroPackLossyConfig(3.5)._options()
    with torch.cuda.device(0):
        st = ep.lib().ep_compress_cuda_noalloc(w.data_ptr(), 1, 256, 256, 256, 3.5, ctypes.byref(opt), None, buf,
                                               1 << 20, ctypes.byref(nbytes), ctypes.byref(bpp))
    assert st == -1


def test_oversize_request_is_rejected_and_the_next_call_works(ep):
    big = synth.gaussian(4096, 4096, seed=2, container="bf16").cuda()  # needs far more than the static area
    with pytest.raises(ep.EntroPackError) as e:
        ep.compress_cuda_noalloc(big, 4.0)
    assert e.value.status == -1
    w = synth.quickstart_256().cuda()
    assert ep.compress_cuda_noalloc(w, 3.5).blob == ep.compress(w, ep.EntroPackLossyConfig(3.5, encoder="cuda")).blob


def test_small_output_buffer_is_rejected(ep):
    w = synth.quickstart_256().cuda()
    buf = (ctypes.c_uint8 * 1024)()
    nbytes, bpp = ctypes.c_size_t(), ctypes.c_double()
    opt = ep.EntroPackLossyConfig(3.5)._options()
    st = ep.lib().ep_compress_cuda_noalloc(w.data_ptr(), 1, 256, 256, 256, 3.5, ctypes.byref(opt),
                                           torch.cuda.current_stream().cuda_stream, buf, 1024, ctypes.byref(nbytes),
                                           ctypes.byref(bpp))
    torch.cuda.synchronize()
    assert st == -9
