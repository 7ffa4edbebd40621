"""Seeded synthetic inputs for the compressor workloads.

This module only draws random numbers and rounds them to the storage dtype; it holds
none of the compressor's arithmetic.  Both the fp64 oracle (via the tests and the
bench) and the CUDA path consume the buffers it produces, so parity never depends on
the generator.

Distributions (N(mu, var) notation, second argument = variance):

* streams C^a, C^b, Z^a, Z^b (or C, Z for HCA): N(0, 1), drawn in fp32, then rounded to
  bf16 (round-to-nearest-even) where the workload stores bf16;
* optional per-row logit offsets U(-lo, lo): one offset per (stream, token row), drawn
  independently for Z^a and Z^b, added to all c channels of that row in fp32 before the
  bf16 rounding (the long-context workload, lo = 4, stresses the softmax range);
* position biases B^a, B^b (m x c) and B (m' x c): N(0, 0.1), fp32;
* hidden states H: N(0, 1) -> bf16; projections W (d x c): N(0, 1/d) -> bf16;
* lightning indexer: queries q [T, H, 128] and compressed indexer keys K [rows, 128]
  N(0, 1) -> bf16, head weights w [T, H] N(0, 1/H) fp32 (the pages give no
  distributions; these keep every head's dot product O(sqrt(128)) and the scores O(1)).

Draw order for a given seed (numpy ``default_rng(seed)``): the streams in the order
listed in the returned dict, then the offsets, then the biases.  Large workloads can be
generated directly on the GPU with a seeded ``torch.Generator`` (same distributions,
different bit stream); that path is used by the full-size parity tests and the bench.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "round_to_bf16",
    "stream_inputs",
    "fused_inputs",
    "stream_inputs_torch",
    "fused_inputs_torch",
    "stream_rows_torch",
    "fused_scalar_inputs",
    "fused_scalar_inputs_torch",
    "bias_torch",
    "ROW_CHUNK",
    "scalar_inputs",
    "scalar_inputs_torch",
    "indexer_inputs",
    "indexer_inputs_torch",
    "WORKLOADS",
]


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32 holding them."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # u + 0x7FFF + lsb, then the low half cleared: in 32 bits this wraps only for bit
    # patterns above 0xFFFF7FFF, which are all NaNs and are restored below.
    r = (u >> 16) & np.uint32(1)
    r += u
    r += np.uint32(0x7FFF)
    r &= np.uint32(0xFFFF0000)
    out = r.view(np.float32)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = np.nan
    return out


def _normal(rng, shape, var=1.0):
    a = rng.standard_normal(shape, dtype=np.float32)
    a *= np.float32(np.sqrt(var))
    return a


def stream_inputs(mode: str, batch: int, n: int, c: int, m: int, dtype: str = "f32",
                  seed: int = 0, z_row_offset: float = 0.0, bias_var: float = 0.1):
    """Host (numpy fp32) inputs for the streaming compressor.

    mode "csa": keys Ca, Cb, Za, Zb ([batch, n, c]) and Ba, Bb ([m, c]).
    mode "hca": keys C, Z ([batch, n, c]) and B ([m, c]).
    dtype "bf16" rounds the streams to bf16 values (still stored as fp32 here).
    """
    rng = np.random.default_rng(seed)
    names = ("Ca", "Cb", "Za", "Zb") if mode == "csa" else ("C", "Z")
    out = {}
    for k in names:
        out[k] = _normal(rng, (batch, n, c))
    if z_row_offset:
        for k in names:
            if k.startswith("Z"):
                off = rng.uniform(-z_row_offset, z_row_offset, size=(batch, n, 1)).astype(np.float32)
                out[k] += off
    if dtype == "bf16":
        for k in names:
            out[k] = round_to_bf16(out[k])
    elif dtype != "f32":
        raise ValueError(dtype)
    bias_names = ("Ba", "Bb") if mode == "csa" else ("B",)
    for k in bias_names:
        out[k] = _normal(rng, (m, c), bias_var)
    return out


def fused_inputs(mode: str, batch: int, n: int, d: int, c: int, m: int, seed: int = 0,
                 bias_var: float = 0.1):
    """Host inputs for the fused projection path: H [batch*n, d] and the W's [d, c]
    rounded to bf16 (stored as fp32), biases fp32."""
    rng = np.random.default_rng(seed)
    out = {"H": round_to_bf16(_normal(rng, (batch * n, d)))}
    wn = ("W_kva", "W_kvb", "W_za", "W_zb") if mode == "csa" else ("W_kv", "W_z")
    for k in wn:
        out[k] = round_to_bf16(_normal(rng, (d, c), 1.0 / d))
    for k in (("Ba", "Bb") if mode == "csa" else ("B",)):
        out[k] = _normal(rng, (m, c), bias_var)
    return out


def fused_scalar_inputs(mode: str, batch: int, n: int, d: int, c: int, m: int, seed: int = 0,
                        z_scale: float = 2.0, bias_var: float = 0.1):
    """Host inputs of the fused scalar-logit form: H [batch*n, d] and the value projections
    W [d, c] as in fused_inputs, score vectors w [d] ~ N(0, z_scale^2 / d) (scores of
    spread z_scale, as scalar_inputs draws them), all rounded to bf16 (stored as fp32);
    biases [m] fp32.  mode "csa": H, W_kva, W_kvb, w_za, w_zb, ba, bb; "hca": H, W_kv, w_z, b."""
    rng = np.random.default_rng(seed)
    out = {"H": round_to_bf16(_normal(rng, (batch * n, d)))}
    for k in (("W_kva", "W_kvb") if mode == "csa" else ("W_kv",)):
        out[k] = round_to_bf16(_normal(rng, (d, c), 1.0 / d))
    for k in (("w_za", "w_zb") if mode == "csa" else ("w_z",)):
        out[k] = round_to_bf16(_normal(rng, (d,), z_scale * z_scale / d))
    for k in (("ba", "bb") if mode == "csa" else ("b",)):
        out[k] = _normal(rng, (m,), bias_var)
    return out


def fused_scalar_inputs_torch(mode: str, batch: int, n: int, d: int, c: int, m: int,
                              seed: int = 0, z_scale: float = 2.0, bias_var: float = 0.1,
                              device="cuda"):
    """Same distributions as :func:`fused_scalar_inputs`, generated on ``device``."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    bf = torch.bfloat16
    out = {"H": torch.randn((batch * n, d), generator=g, device=device).to(bf)}
    for k in (("W_kva", "W_kvb") if mode == "csa" else ("W_kv",)):
        out[k] = (torch.randn((d, c), generator=g, device=device) * float(1.0 / np.sqrt(d))).to(bf)
    for k in (("w_za", "w_zb") if mode == "csa" else ("w_z",)):
        out[k] = (torch.randn((d,), generator=g, device=device) * float(z_scale / np.sqrt(d))).to(bf)
    for k in (("ba", "bb") if mode == "csa" else ("b",)):
        out[k] = torch.randn((m,), generator=g, device=device) * float(np.sqrt(bias_var))
    return out


def stream_inputs_torch(mode: str, batch: int, n: int, c: int, m: int, dtype: str,
                        seed: int = 0, z_row_offset: float = 0.0, bias_var: float = 0.1,
                        device="cuda"):
    """Same distributions as :func:`stream_inputs`, generated on ``device`` with a
    seeded torch.Generator (for workloads too large to draw on the host quickly)."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    names = ("Ca", "Cb", "Za", "Zb") if mode == "csa" else ("C", "Z")
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = {}
    for k in names:
        x = torch.randn((batch, n, c), generator=g, device=device, dtype=torch.float32)
        if z_row_offset and k.startswith("Z"):
            off = torch.rand((batch, n, 1), generator=g, device=device, dtype=torch.float32)
            x += off * (2 * z_row_offset) - z_row_offset
        out[k] = x.to(tdt)
        del x
    for k in (("Ba", "Bb") if mode == "csa" else ("B",)):
        out[k] = torch.randn((m, c), generator=g, device=device, dtype=torch.float32) * float(np.sqrt(bias_var))
    return out


ROW_CHUNK = 1 << 16  # rows per independently seeded piece of stream_rows_torch


def stream_rows_torch(row0: int, row1: int, c: int, dtype: str, seed: int = 0,
                      z_row_offset: float = 0.0, device="cuda"):
    """Rows [row0, row1) of one long sequence's four CSA streams Ca, Cb, Za, Zb ([1, rows,
    c], the distributions of stream_inputs_torch), drawn in pieces of ROW_CHUNK rows, each
    from its own generator seeded by (seed, piece index): any process can draw any rows of
    the same sequence and gets the same values (for a given device type), which lets ranks
    that each hold a slice of one sequence, and a checker that redraws a few windows,
    agree."""
    import torch

    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    names = ("Ca", "Cb", "Za", "Zb")
    out = {k: torch.empty((1, row1 - row0, c), dtype=tdt, device=device) for k in names}
    g = torch.Generator(device=device)
    for piece in range(row0 // ROW_CHUNK, (max(row1, row0 + 1) - 1) // ROW_CHUNK + 1):
        p0 = piece * ROW_CHUNK
        g.manual_seed(seed * 1000003 + piece)
        lo, hi = max(row0, p0), min(row1, p0 + ROW_CHUNK)
        for k in names:
            x = torch.randn((ROW_CHUNK, c), generator=g, device=device, dtype=torch.float32)
            if z_row_offset and k.startswith("Z"):
                off = torch.rand((ROW_CHUNK, 1), generator=g, device=device, dtype=torch.float32)
                x += off * (2 * z_row_offset) - z_row_offset
            if hi > lo:
                out[k][0, lo - row0:hi - row0] = x[lo - p0:hi - p0].to(tdt)
    return out


def bias_torch(m: int, c: int, seed: int, bias_var: float = 0.1, device="cuda"):
    """One position bias [m, c] fp32 ~ N(0, bias_var), from its own seeded generator."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn((m, c), generator=g, device=device, dtype=torch.float32) * float(np.sqrt(bias_var))


def fused_inputs_torch(mode: str, batch: int, n: int, d: int, c: int, m: int, seed: int = 0,
                       bias_var: float = 0.1, device="cuda"):
    """Same distributions as :func:`fused_inputs`, generated on ``device``."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = {}
    H = torch.empty((batch * n, d), device=device, dtype=torch.bfloat16)
    rows = max(1, (1 << 28) // d)          # draw in slabs to bound fp32 temporaries
    for r0 in range(0, batch * n, rows):
        r1 = min(batch * n, r0 + rows)
        H[r0:r1] = torch.randn((r1 - r0, d), generator=g, device=device, dtype=torch.float32)
    out["H"] = H
    wn = ("W_kva", "W_kvb", "W_za", "W_zb") if mode == "csa" else ("W_kv", "W_z")
    for k in wn:
        out[k] = (torch.randn((d, c), generator=g, device=device, dtype=torch.float32)
                  * float(1.0 / np.sqrt(d))).to(torch.bfloat16)
    for k in (("Ba", "Bb") if mode == "csa" else ("B",)):
        out[k] = torch.randn((m, c), generator=g, device=device, dtype=torch.float32) * float(np.sqrt(bias_var))
    return out


def scalar_inputs(mode: str, batch: int, n: int, c: int, m: int, dtype: str = "f32", seed: int = 0,
                  z_scale: float = 2.0, bias_var: float = 0.1):
    """Host inputs for the scalar-logit form: value streams [batch, n, c] N(0, 1), one logit
    per token and stream [batch, n] N(0, z_scale^2), biases [m] N(0, bias_var).
    mode "csa": Ca, Cb, za, zb, ba, bb;  mode "hca": C, z, b."""
    rng = np.random.default_rng(seed)
    vals = ("Ca", "Cb") if mode == "csa" else ("C",)
    logs = ("za", "zb") if mode == "csa" else ("z",)
    out = {k: _normal(rng, (batch, n, c)) for k in vals}
    for k in logs:
        out[k] = (_normal(rng, (batch, n)) * np.float32(z_scale)).astype(np.float32)
    if dtype == "bf16":
        for k in vals + logs:
            out[k] = round_to_bf16(out[k])
    for k in (("ba", "bb") if mode == "csa" else ("b",)):
        out[k] = _normal(rng, (m,), bias_var)
    return out


def scalar_inputs_torch(mode: str, batch: int, n: int, c: int, m: int, dtype: str, seed: int = 0,
                        z_scale: float = 2.0, bias_var: float = 0.1, device="cuda"):
    """Same distributions as :func:`scalar_inputs`, generated on ``device``."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    vals = ("Ca", "Cb") if mode == "csa" else ("C",)
    logs = ("za", "zb") if mode == "csa" else ("z",)
    out = {k: torch.randn((batch, n, c), generator=g, device=device).to(tdt) for k in vals}
    for k in logs:
        out[k] = (torch.randn((batch, n), generator=g, device=device) * z_scale).to(tdt)
    for k in (("ba", "bb") if mode == "csa" else ("b",)):
        out[k] = torch.randn((m,), generator=g, device=device) * float(np.sqrt(bias_var))
    return out


def indexer_inputs(T: int, H: int, rows: int, D: int = 128, seed: int = 0):
    """Host inputs of the lightning indexer: q [T, H, D], w [T, H], K [rows, D] (fp32
    arrays holding bf16 values for q and K).  Draw order: q, K, w."""
    rng = np.random.default_rng(seed)
    q = round_to_bf16(_normal(rng, (T, H, D)))
    K = round_to_bf16(_normal(rng, (rows, D)))
    w = _normal(rng, (T, H), 1.0 / H)
    return dict(q=q, K=K, w=w)


def indexer_inputs_torch(T: int, H: int, rows: int, D: int = 128, seed: int = 0, device="cuda"):
    """Same distributions as :func:`indexer_inputs`, generated on ``device``."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    q = torch.randn((T, H, D), generator=g, device=device).to(torch.bfloat16)
    K = torch.randn((rows, D), generator=g, device=device).to(torch.bfloat16)
    w = torch.randn((T, H), generator=g, device=device) * float(np.sqrt(1.0 / H))
    return dict(q=q, K=K, w=w)


# The five workloads, named by what they are.
WORKLOADS = {
    "csa_f32_n1024": dict(kind="stream", mode="csa", batch=1, n=1024, c=512, m=4,
                          in_dtype="f32", out_dtype="f32"),
    "hca_bf16_n65536": dict(kind="stream", mode="hca", batch=1, n=65536, c=512, m=128,
                            in_dtype="bf16", out_dtype="bf16"),
    "csa_fused_n32768_d7168": dict(kind="fused", mode="csa", batch=1, n=32768, d=7168, c=512,
                                   m=4, out_dtype="bf16"),
    "hca_fused_4x131072_d4096": dict(kind="fused", mode="hca", batch=4, n=131072, d=4096,
                                     c=512, m=128, out_dtype="bf16"),
    "csa_long_n1048576": dict(kind="stream", mode="csa", batch=1, n=1 << 20, c=512, m=4,
                              in_dtype="bf16", out_dtype="bf16", z_row_offset=4.0),
    "hca_long_n1048576": dict(kind="stream", mode="hca", batch=1, n=1 << 20, c=512, m=128,
                              in_dtype="bf16", out_dtype="bf16", z_row_offset=4.0),
}
