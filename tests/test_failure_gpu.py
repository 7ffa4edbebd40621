"""Failure detection on the GPU without a fault: a bounded wait that nothing completes gives
up after its limit, raises the CTA's abort flag (which releases the CTA's other waiters) and
the device error word; the host reads KVC_ERR_TIMEOUT once, and the context keeps working."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import check_close, dev
from kv_token_compressor_b200 import kvc, synth
from oracle import compressor as O

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_context_survives():
    assert kvc.device_status() == kvc.KVC_OK  # nothing pending from earlier tests
    flags = kvc.selftest_bounded_wait()
    assert kvc.device_status() == kvc.KVC_ERR_TIMEOUT
    assert flags.cpu().tolist() == [1, 1]
    assert kvc.device_status() == kvc.KVC_OK  # the report cleared the word
    # the same process, stream and context still compute correctly
    d = synth.stream_inputs("hca", 1, 128 * 40, 256, 128, "bf16", seed=21)
    out = kvc.hca_compress(dev(d["C"], "bf16"), dev(d["Z"], "bf16"), dev(d["B"], "f32"), m=128)
    torch.cuda.synchronize()
    assert kvc.device_status() == kvc.KVC_OK
    check_close(out, O.hca_compress(d["C"], d["Z"], d["B"], 128), "bf16", "after the self-test")


def test_selftest_rejects_host_pointer():
    host = np.zeros(2, dtype=np.int32)
    st = kvc.lib().kvc_selftest_bounded_wait(host.ctypes.data, None)
    assert st == kvc.KVC_ERR_POINTER
