"""Pins of the oracle's density-field state representation (CPU only).

The pages describe the representation in one sentence (gist.science technical summary of DF-SSM, §2.D
"Density Field State Representation": a binary field per state element with K^2 about 4 d_state cells;
normalization, sigma-delta injection with error feedback, binarization, popcount readout).  The oracle
states its reading; these tests hold it to things fixed outside the oracle:
  - rows worked by hand (tests/golden/density_field.txt);
  - the closed form of a first-order sigma-delta modulator: after cells 0..j the count of ones is
    floor(P_j + 1/2), P_j the exact sum of the densities fed so far (an integer computation here);
  - the five readout levels c {-1, -1/2, 0, 1/2, 1} come back exactly;
  - error feedback bounds the running readout error by c / 4 (plus the normalization's rounding).
"""
import os

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import oracle
from bit_quantized_mamba_b200 import inputs


def _golden_rows():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "density_field.txt")
    rows, cur = [], None
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            if key == "row":
                cur = dict(name=vals[0], N=int(vals[1]))
                rows.append(cur)
            elif key in ("state", "readout"):
                cur[key] = np.array([float(v) for v in vals], np.float32)
            elif key == "scale":
                cur[key] = np.float32(float(vals[0]))
            elif key == "words":
                cur[key] = np.array([int(v, 16) for v in vals], np.uint32)
    return rows


@pytest.mark.parametrize("row", _golden_rows(), ids=lambda r: r["name"])
def test_hand_worked_rows(row):
    field, scale = oracle.field_encode(row["state"][None, :])
    assert scale[0] == row["scale"]
    assert np.array_equal(field[0], row["words"]), [hex(w) for w in field[0]]
    back = oracle.field_decode(field, scale, row["N"])
    assert np.array_equal(back[0], row["readout"])


def _densities_units(S):
    """The densities d_n = fl32(fl32(S_n / c) + 1) / 2 of each row as integers in units of 2^-25
    (numpy fp32 arithmetic is IEEE single precision)."""
    S = S.astype(np.float32)
    c = np.max(np.abs(S), axis=1, keepdims=True).astype(np.float32)
    with np.errstate(invalid="ignore", divide="ignore"):
        x = np.where(c > 0, S / np.where(c > 0, c, np.float32(1)), np.float32(0)).astype(np.float32)
    d = ((x + np.float32(1)).astype(np.float32) * np.float32(0.5)).astype(np.float32)
    D = d.astype(np.float64) * 2.0 ** 25
    assert np.all(D == np.floor(D)), "densities are multiples of 2^-25"
    return D.astype(np.int64), c[:, 0]


def _cells(field, N):
    w = field.astype(np.uint64)
    bits = (w[:, :, None] >> np.arange(32, dtype=np.uint64)) & np.uint64(1)
    return bits.reshape(field.shape[0], N * 4).astype(np.int64)


@pytest.mark.parametrize("N,rows", [(8, 300), (16, 200), (24, 130), (64, 129), (128, 260), (256, 70)])
def test_sigma_delta_closed_form(N, rows):
    """Ones among cells 0..j equal floor(P_j + 1/2) for every j (P_j in units of 2^-25, integers)."""
    S = inputs.ssm_state_rows(seed=40 + N, rows=rows, d_state=N)
    field, scale = oracle.field_encode(S)
    D, c = _densities_units(S)
    assert np.array_equal(scale, c)
    P = np.cumsum(np.repeat(D, 4, axis=1), axis=1)          # after each cell
    ones = (P + (1 << 24)) >> 25                             # floor(P + 1/2)
    assert np.array_equal(np.cumsum(_cells(field, N), axis=1), ones)


def test_levels_round_trip_exactly():
    g = np.random.default_rng(7)
    rows, N = 64, 128
    c = (10.0 ** g.uniform(-3, 3, size=(rows, 1))).astype(np.float32)
    lev = g.integers(0, 5, size=(rows, N)).astype(np.float32) * np.float32(0.5) - np.float32(1)
    lev[:, 0] = np.where(g.integers(0, 2, size=rows) == 0, -1.0, 1.0)  # each row reaches +-c
    S = (lev * c).astype(np.float32)
    field, scale = oracle.field_encode(S)
    assert np.array_equal(scale, c[:, 0])
    assert np.array_equal(oracle.field_decode(field, scale, N), S)


@pytest.mark.parametrize("N", [8, 64, 128, 256])
def test_running_error_bounded_by_feedback(N):
    """sum_{m<=n} (S^_m - S_m) stays within c / 4 (plus the rounding of S / c and of x + 1): without
    the error feedback, or with it reset per value, these sums drift far outside the bound."""
    S = inputs.ssm_state_rows(seed=90 + N, rows=400, d_state=N).astype(np.float64)
    field, scale = oracle.field_encode(S.astype(np.float32))
    back = oracle.field_decode(field, scale, N).astype(np.float64)
    c = scale.astype(np.float64)[:, None]
    run = np.cumsum(back - S, axis=1)
    assert np.all(np.abs(run) <= c / 4 + c * N * 2.0 ** -22)
    assert np.all(np.abs(back) <= c)


def test_readout_levels_of_arbitrary_fields():
    """Any field decodes to c (popcount / 2 - 1) per value, levels in {-c, -c/2, 0, c/2, c}."""
    g = np.random.default_rng(11)
    N, rows = 64, 50
    field = g.integers(0, 2 ** 32, size=(rows, N // 8), dtype=np.uint64).astype(np.uint32)
    scale = g.uniform(0.1, 10, size=rows).astype(np.float32)
    back = oracle.field_decode(field, scale, N)
    p = _cells(field, N).reshape(rows, N, 4).sum(axis=2)
    assert np.array_equal(back / scale[:, None], p * 0.5 - 1.0)


_f32 = st.floats(width=32, allow_nan=False, allow_infinity=False)


@settings(max_examples=300, deadline=None)
@given(st.sampled_from([8, 16, 24, 32, 64]).flatmap(lambda n: st.lists(_f32, min_size=n, max_size=n)))
def test_closed_form_on_arbitrary_rows(vals):
    """Any finite fp32 row, extremes and subnormals included: the closed form holds cell by cell and
    every readout lies on one of the five levels of the row's absmax."""
    S = np.array([vals], np.float32)
    N = S.shape[1]
    field, scale = oracle.field_encode(S)
    D, c = _densities_units(S)
    assert scale[0] == c[0]
    P = np.cumsum(np.repeat(D, 4, axis=1), axis=1)
    assert np.array_equal(np.cumsum(_cells(field, N), axis=1), (P + (1 << 24)) >> 25)
    back = oracle.field_decode(field, scale, N)
    levels = np.array([-1.0, -0.5, 0.0, 0.5, 1.0], np.float32) * scale[0]
    assert np.all(np.isin(back[0], levels))
