"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that the pins
reject every one of them: a dropped term, a wrong sign, an off-by-one index, swapped or
transposed operands, a wrong boundary, a wrong normalisation."""

import os
import types

import pytest

import oracle_pins

SRC = os.path.join(os.path.dirname(__file__), os.pardir, "oracle", "compressor.py")

# (name, text in the oracle, replacement)
MUTANTS = [
    ("b_range_off_by_one", "return range(m * i, m * (i + 1)), range(m * (i - 1), m * i)",
     "return range(m * i, m * (i + 1)), range(m * (i - 1) + 1, m * i + 1)"),
    ("a_bias_dropped", "La = _f64(Za[a_rows.start:a_rows.stop]) + _f64(Ba)",
     "La = _f64(Za[a_rows.start:a_rows.stop])"),
    ("a_bias_reversed", "La = _f64(Za[a_rows.start:a_rows.stop]) + _f64(Ba)",
     "La = _f64(Za[a_rows.start:a_rows.stop]) + _f64(Ba)[::-1]"),
    ("b_bias_dropped", "Lb = Zb_rows + Bb", "Lb = Zb_rows"),
    ("b_logits_from_a_block", "Zb_rows = _f64(Zb[b_rows.start:b_rows.stop])",
     "Zb_rows = _f64(Zb[a_rows.start:a_rows.stop])"),
    ("softmax_sign_flipped", "w = np.exp(L - M)", "w = np.exp(M - L)"),
    ("values_a_b_swapped", "V = np.concatenate([Va, Cb_rows], axis=0)",
     "V = np.concatenate([Cb_rows, Va], axis=0)"),
    ("boundary_logit_zero", "Zb_rows = np.full((m, c), -np.inf)", "Zb_rows = np.zeros((m, c))"),
    ("separate_normalisation", "    L, V = csa_window(Ca, Cb, Za, Zb, Ba, Bb, i, m, overlap)\n    return pool_window(L, V)",
     "    L, V = csa_window(Ca, Cb, Za, Zb, Ba, Bb, i, m, overlap)\n"
     "    if overlap and i > 0:\n        return pool_window(L[:m], V[:m]) + pool_window(L[m:], V[m:])\n"
     "    return pool_window(L, V)"),
    ("normaliser_dropped", "return w / np.sum(w, axis=0, keepdims=True)", "return w"),
    ("hca_bias_dropped", "L = _f64(Z[lo:hi]) + _f64(B)", "L = _f64(Z[lo:hi])"),
    ("hca_segment_shift", "lo, hi = m * i, m * (i + 1)\n    L = _f64(Z[lo:hi])",
     "lo, hi = m * i + 1, m * (i + 1) + 1\n    L = _f64(Z[lo:hi])"),
    ("scalar_hca_segment_shift", "lo, hi = m * i, m * (i + 1)\n    L = _f64(z[lo:hi])",
     "lo, hi = m * i + 1, m * (i + 1) + 1\n    L = _f64(z[lo:hi])"),
    ("entries_ceil", "    return n // m", "    return -(-n // m)"),
    ("projection_transposed", "return _f64(H) @ _f64(W)", "return _f64(H) @ _f64(W).T"),
    ("projection_k_misaligned", "return _f64(H) @ _f64(W)", "return _f64(H) @ _f64(W)[::-1]"),
    ("fused_streams_swapped", "Ca, Za = stream(W_kva), stream(W_za)", "Ca, Za = stream(W_za), stream(W_kva)"),
    ("fused_b_streams_swapped", "Cb = stream(W_kvb) if overlap else None", "Cb = stream(W_zb) if overlap else None"),
    ("scalar_a_bias_dropped", "la = _f64(za[a_rows.start:a_rows.stop]) + _f64(ba)",
     "la = _f64(za[a_rows.start:a_rows.stop])"),
    ("scalar_b_rows_from_a_block", "lb = _f64(zb[b_rows.start:b_rows.stop]) + _f64(bb)",
     "lb = _f64(zb[a_rows.start:a_rows.stop]) + _f64(bb)"),
    ("scalar_boundary_zero_logit", "lb = np.full(m, -np.inf)", "lb = np.zeros(m)"),
    ("scalar_separately_normalised", "    w = np.exp(L - np.max(L))\n    s = w / np.sum(w)                                # one",
     "    w = np.exp(L - np.max(L))\n    s = w / (np.sum(w[:m]) if len(w) == m else np.sum(w[m:]) + 0 * np.sum(w[:m]))  # one"),
    ("scalar_hca_bias_dropped", "L = _f64(z[lo:hi]) + _f64(bvec)", "L = _f64(z[lo:hi])"),
    ("e4m3_two_mantissa_bits", "np.maximum(lead, -6) - 3)", "np.maximum(lead, -6) - 2)"),
    ("e4m3_subnormal_boundary", "np.maximum(lead, -6) - 3)", "np.maximum(lead, -7) - 3)"),
    ("e4m3_no_saturation", "    q = np.minimum(q, E4M3_MAX)\n", "\n"),
    ("rope_angle_sign", "np.exp(1j * ang)", "np.exp(-1j * ang)"),
    ("rope_pairs_halves", "z = (x[..., 0::2] + 1j * x[..., 1::2])", "z = (x[..., :r // 2] + 1j * x[..., r // 2:])"),
    ("cache_position_shift", "pos = pos_offset + pos_stride * np.arange(ne, dtype=np.float64)",
     "pos = pos_offset + pos_stride * np.arange(1, ne + 1, dtype=np.float64)"),
    ("cache_scale_dropped", "nope = round_e4m3(entries[..., :c - r] * scale)", "nope = round_e4m3(entries[..., :c - r])"),
    ("fused_hca_streams_swapped", "C = project(Hs, W_kv)\n        Z = project(Hs, W_z)",
     "C = project(Hs, W_z)\n        Z = project(Hs, W_kv)"),
]


def _mutant_module(old, new):
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) == 1, f"mutation anchor not unique/present: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


# A broken oracle may divide by zero or produce NaN on the way to failing a pin; the
# warnings that numpy raises then are expected.
@pytest.mark.filterwarnings("ignore::RuntimeWarning")
@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(name, old, new):
    mod = _mutant_module(old, new)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mod)
        except Exception:  # noqa: BLE001 - any failure counts as a rejection
            failed.append(pin.__name__)
    assert failed, f"no pin rejects mutant {name}"
