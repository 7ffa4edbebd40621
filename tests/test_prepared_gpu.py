"""GPU parity of the prepared-bias HCA compressor (hca_prepare_bias + hca_compress_prepared):
bit for bit the result of hca_compress with the same bias, on the TMA-fed window kernel
(which copies the prepared slabs) and on the kernels that read the workspace's raw copy,
and against the fp64 oracle; a workspace made for another problem is refused on the
device."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import check_close, dev, tdtype
from kv_token_compressor_b200 import kvc, synth
from oracle import compressor as O

pytestmark = pytest.mark.gpu

CASES = [
    # kernel, batch, n, c, m, in, out
    ("window_tma_kernel/prepared", 1, 65536, 512, 128, "bf16", "bf16"),
    ("window_tma_kernel/prepared", 2, 128 * 37 + 5, 520, 128, "bf16", "f32"),
    ("window_tma_kernel/prepared", 1, 64 * 300 + 9, 256, 64, "f32", "f32"),
    ("window_tma_kernel/prepared", 3, 32 * 200, 136, 32, "f32", "bf16"),
    # windows the TMA-fed kernel does not take: the raw copy in the workspace
    ("window_pipe_kernel/rg16", 1, 16 * 100, 64, 16, "f32", "f32"),
    ("window_pipe_kernel/rg16", 1, 256 * 20, 128, 256, "bf16", "bf16"),
]


@pytest.mark.parametrize("kernel,batch,n,c,m,in_dt,out_dt", CASES,
                         ids=[f"{k}-{b}x{n}x{c}-m{m}-{i}-{o}" for k, b, n, c, m, i, o in CASES])
def test_prepared_equals_unprepared(kernel, batch, n, c, m, in_dt, out_dt):
    d = synth.stream_inputs("hca", batch, n, c, m, in_dt, seed=n + m)
    C, Z, B = dev(d["C"], in_dt), dev(d["Z"], in_dt), dev(d["B"], "f32")
    plain = kvc.hca_compress(C, Z, B, m=m, out_dtype=tdtype(out_dt))
    ws = kvc.hca_prepare_bias(B, tdtype(in_dt))
    assert kvc.last_kernel() == "prepare_bias_kernel"
    B.fill_(float("nan"))  # the workspace keeps its own copy
    prepared = kvc.hca_compress_prepared(C, Z, ws, m=m, out_dtype=tdtype(out_dt))
    assert kvc.last_kernel() == kernel
    assert kvc.device_status() == kvc.KVC_OK
    assert torch.equal(prepared, plain)
    check_close(prepared, O.hca_compress(d["C"], d["Z"], d["B"], m), out_dt, kernel)


@pytest.mark.parametrize("spread", [38.0, 90.0])
def test_prepared_bias_spread_paths(spread):
    """Both softmax-reference paths (bias spread within and beyond the fast-bound limit)
    are selected from the prepared flag exactly as from the staged bias."""
    m, c = 128, 256
    d = synth.stream_inputs("hca", 1, m * 300 + 3, c, m, "bf16", seed=int(spread))
    rng = np.random.default_rng(int(spread))
    d["B"] = rng.uniform(-spread / 2, spread / 2, size=(m, c)).astype(np.float32)
    C, Z, B = dev(d["C"], "bf16"), dev(d["Z"], "bf16"), dev(d["B"], "f32")
    plain = kvc.hca_compress(C, Z, B, m=m, out_dtype=torch.float32)
    ws = kvc.hca_prepare_bias(B, torch.bfloat16)
    prepared = kvc.hca_compress_prepared(C, Z, ws, m=m, out_dtype=torch.float32)
    assert kvc.device_status() == kvc.KVC_OK
    assert torch.equal(prepared, plain)
    check_close(prepared, O.hca_compress(d["C"], d["Z"], d["B"], m), "f32", f"spread {spread}")


def test_workspace_of_another_problem_is_refused():
    m, c = 128, 512
    d = synth.stream_inputs("hca", 1, m * 50, c, m, "bf16", seed=1)
    C, Z = dev(d["C"], "bf16"), dev(d["Z"], "bf16")
    ws = kvc.hca_prepare_bias(dev(d["B"], "f32"), torch.float32)  # prepared for fp32 streams
    big = torch.zeros(kvc.hca_bias_workspace_bytes(c, m, torch.bfloat16) + 4096, dtype=torch.uint8,
                      device="cuda")
    big[:ws.numel()].copy_(ws)
    out = torch.full((1, 50, c), -1280.0, dtype=torch.bfloat16, device="cuda")
    kvc.hca_compress_prepared(C, Z, big, m=m, out=out)
    assert kvc.last_kernel() == "window_tma_kernel/prepared"
    assert kvc.device_status() == kvc.KVC_ERR_WORKSPACE
    assert bool(torch.all(out == -1280.0))  # nothing was written
    assert kvc.device_status() == kvc.KVC_OK  # reported once
    # a zeroed workspace (never prepared) is refused the same way
    big.zero_()
    kvc.hca_compress_prepared(C, Z, big, m=m, out=out)
    assert kvc.device_status() == kvc.KVC_ERR_WORKSPACE


def test_prepared_long_n1048576_every_entry():
    """The long-context HCA workload through the prepared path: every entry equals the
    unprepared call's bit for bit (which the stream tests compare with the oracle)."""
    n, c, m = 1 << 20, 512, 128
    t = synth.stream_inputs_torch("hca", 1, n, c, m, "bf16", seed=5, z_row_offset=4.0)
    plain = kvc.hca_compress(t["C"], t["Z"], t["B"], m=m)
    ws = kvc.hca_prepare_bias(t["B"], torch.bfloat16)
    prepared = kvc.hca_compress_prepared(t["C"], t["Z"], ws, m=m)
    assert kvc.device_status() == kvc.KVC_OK
    assert torch.equal(prepared, plain)
    del t
    torch.cuda.empty_cache()
