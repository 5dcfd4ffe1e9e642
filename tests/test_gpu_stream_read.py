"""The read-only streaming kernels (skinny_stream_read) that give the bench its
read-only HBM ceiling: both methods run to completion on buffers that are and
are not whole multiples of their block size, leave the device error word
clear, and never write the sink unless their running XOR hits its magic
value (a buffer of zeros keeps it zero)."""
import ctypes

import pytest
import torch

import fp8_weight_only_w4a16_b200 as sk

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def no_device_errors():
    yield
    assert sk.device_error(clear=True) == 0


@pytest.mark.parametrize("method", [0, 1])
@pytest.mark.parametrize("nbytes", [64 << 20, (64 << 20) + 36864 * 3 + 4096, 36864])
def test_stream_read_runs(method, nbytes):
    buf = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    sink = torch.full((1,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    lib = sk.library()
    stream = torch.cuda.current_stream().cuda_stream
    st = lib.skinny_stream_read(ctypes.c_void_p(buf.data_ptr()), nbytes, method,
                                ctypes.c_void_p(sink.data_ptr()), ctypes.c_void_p(stream))
    assert st == 0, sk.status_string(st)
    torch.cuda.synchronize()
    # The sink is written only when a thread's XOR equals 0x9E3779B9; zeros never do.
    assert int(sink.item()) == 0x5A5A5A5A


def test_stream_read_bulk_rejects_a_buffer_smaller_than_one_block():
    buf = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    st = sk.library().skinny_stream_read(ctypes.c_void_p(buf.data_ptr()), 4096, 1, None, None)
    assert sk.status_string(st) == "SKINNY_ERR_UNSUPPORTED"
