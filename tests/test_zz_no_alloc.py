"""The allocation-free HCA entry point, hca_compress_noalloc, against hca_compress.

hca_compress_noalloc serves callers that cannot allocate device memory while they run (a
serving loop whose memory is all handed out at start-up, a host program with no
allocator to provide a workspace): the library keeps the prepared bias in a fixed scratch
array of its own.  Here it is called through the C ABI twice in a row on one stream, the
second call with another bias, shape and dtype, so it runs on the scratch the first call
left behind; each result must match hca_compress on the same inputs within the GPU
tests' parity tolerance.  This file is collected last, so that a run stopping at the
first failure has run every other test before it."""

from __future__ import annotations

import pytest
import torch

from gpu_util import check_close, dev, host64, tdtype
from kv_token_compressor_b200 import kvc, synth

pytestmark = pytest.mark.gpu


def _code(dt):
    return kvc.KVC_BF16 if dt == torch.bfloat16 else kvc.KVC_F32


def _noalloc(C, Z, B, m, out):
    """One call of the C entry point with raw device pointers."""
    batch, n, c = C.shape
    return kvc.lib().hca_compress_noalloc(C.data_ptr(), Z.data_ptr(), _code(C.dtype), B.data_ptr(),
                                          batch, n, c, m, out.data_ptr(), _code(out.dtype),
                                          torch.cuda.current_stream().cuda_stream)


def _case(batch, n, c, m, in_dt, out_dt, seed):
    d = synth.stream_inputs("hca", batch, n, c, m, in_dt, seed=seed)
    C, Z, B = dev(d["C"], in_dt), dev(d["Z"], in_dt), dev(d["B"], "f32")
    ref = kvc.hca_compress(C, Z, B, m=m, out_dtype=tdtype(out_dt))
    out = torch.empty_like(ref)
    return C, Z, B, m, out, ref


def test_noalloc_matches_hca_compress_twice():
    first = _case(1, 128 * 300 + 5, 512, 128, "bf16", "bf16", seed=1)
    second = _case(2, 64 * 100 + 3, 256, 64, "f32", "f32", seed=2)
    torch.cuda.synchronize()
    assert _noalloc(*first[:5]) == kvc.KVC_OK
    assert kvc.last_kernel() == "window_tma_kernel/prepared"
    assert _noalloc(*second[:5]) == kvc.KVC_OK
    assert kvc.device_status() == kvc.KVC_OK
    for (C, Z, B, m, out, ref), dt in ((first, "bf16"), (second, "f32")):
        check_close(out, host64(ref), dt, f"noalloc m={m} {dt}")


def test_noalloc_repeat_call_allocates_no_device_memory():
    C, Z, B, m, out, ref = _case(1, 128 * 200, 512, 128, "bf16", "bf16", seed=3)
    assert _noalloc(C, Z, B, m, out) == kvc.KVC_OK
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    assert _noalloc(C, Z, B, m, out) == kvc.KVC_OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert kvc.device_status() == kvc.KVC_OK
    check_close(out, host64(ref), "bf16", "noalloc repeat")


def test_noalloc_rejects_a_bias_beyond_its_scratch():
    """c = 2048 at m = 128 needs about 2 MB of workspace: refused before any launch."""
    C = torch.zeros((1, 256, 2048), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((128, 2048), dtype=torch.float32, device="cuda")
    out = torch.full((1, 2, 2048), -1280.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(C, C, B, 128, out) == kvc.KVC_ERR_TOO_LARGE
    assert "fixed scratch" in kvc.status_string(kvc.KVC_ERR_TOO_LARGE)
    torch.cuda.synchronize()
    assert bool(torch.all(out == -1280.0))
