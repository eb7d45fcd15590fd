"""attn_hadamard_quant_fp8_noalloc: the FP8 input preparation for callers that
cannot allocate device memory (their memory belongs to an allocator they
cannot reach, or they must not call cudaMalloc on a hot path).  It uses the
library's static scratch array instead of a caller workspace.  This file is
collected last on purpose, so a run that stops at the first failure has run
every other test before it.

Checked through the C ABI against the workspace entry point, on two calls in a
row: the second input has a smaller absolute maximum, so a maximum left over in
the shared scratch from the first call would show up as a wrong scale."""
import ctypes

import numpy as np
import pytest

import attn_inputs as gen

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_two_calls():
    import torch

    import exact_attention_140_b200 as ea
    lib = ctypes.CDLL(ea.lib_path)
    vp = ctypes.c_void_p
    lib.attn_hadamard_quant_fp8_noalloc.argtypes = [vp, vp, vp, ctypes.c_longlong, ctypes.c_int, vp, vp]
    lib.attn_hadamard_quant_fp8_noalloc.restype = ctypes.c_int
    lib.attn_hadamard_quant_fp8.argtypes = [vp, vp, vp, vp, ctypes.c_longlong, ctypes.c_int, vp, vp]
    lib.attn_hadamard_quant_fp8.restype = ctypes.c_int

    d = 128
    stream = torch.cuda.current_stream().cuda_stream
    signs = torch.from_numpy(gen.hadamard_signs(gen.BASE_SEED + 3, d)).cuda()
    ws = torch.empty(ea.attn_hadamard_quant_fp8_workspace_bytes(), dtype=torch.uint8, device="cuda")
    # first call: outlier columns (large maximum); second: plain N(0,1) (smaller maximum)
    inputs = [gen.normal_bf16(41, (3, 700, 2, d), column_scale=gen.outlier_scale(42, 2, d)),
              gen.normal_bf16(43, (2, 513, 2, d))]
    for call, xb in enumerate(inputs):
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
        rows = x.numel() // d
        for sg in (signs, None):
            sgp = None if sg is None else sg.data_ptr()
            a8 = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
            b8 = torch.full(x.shape, 0xAB, dtype=torch.uint8, device="cuda")
            da = torch.empty(1, dtype=torch.float32, device="cuda")
            db = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
            assert lib.attn_hadamard_quant_fp8(x.data_ptr(), a8.data_ptr(), da.data_ptr(), ws.data_ptr(), rows, d,
                                               sgp, stream) == 0
            assert lib.attn_hadamard_quant_fp8_noalloc(x.data_ptr(), b8.data_ptr(), db.data_ptr(), rows, d, sgp,
                                                       stream) == 0
            torch.cuda.synchronize()
            # same kernels, same inputs: codes and scale are identical (the
            # tolerance the quantiser tests use for codes is bit-exact)
            assert torch.equal(a8, b8), (call, sg is None)
            assert da.item() == db.item(), (call, da.item(), db.item())
            assert db.item() > 0
    rc, word = ea.attn_get_last_device_error()
    assert rc == 0, hex(word)


def test_noalloc_rejects_bad_arguments():
    import exact_attention_140_b200 as ea
    FAKE = 1 << 20
    assert ea.attn_hadamard_quant_fp8_noalloc(FAKE, FAKE, FAKE, 4, 64, stream=0, raise_on_error=False) == 2
    assert ea.attn_hadamard_quant_fp8_noalloc(FAKE, FAKE, None, 4, 128, stream=0, raise_on_error=False) == 1
    assert ea.attn_hadamard_quant_fp8_noalloc(FAKE + 4, FAKE, FAKE, 4, 128, stream=0, raise_on_error=False) == 3
