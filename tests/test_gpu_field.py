"""GPU parity of the density-field state representation against the oracle (bit-exact).

The oracle runs the sigma-delta modulator cell after cell (technical summary §2.D "Density Field State
Representation", under the reading its header states); the kernels compute each value's four cells from
exact integer prefix sums of the densities, one warp per row.  Fields, scales and readouts must be equal
bit for bit: every step is integer or a single correctly rounded fp32 operation on both sides.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_mamba_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dfssm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_mamba_b200 import build, dfssm as lib
    build.build()
    lib.lib()
    return lib


DEV = torch.device("cuda:0")


def _check_all(dfssm, S):
    """encode, decode and both round-trip forms against the oracle on the rows S [rows][N]."""
    N = S.shape[1]
    f_ref, s_ref = oracle.field_encode(S)
    back_ref = oracle.field_decode(f_ref, s_ref, N)
    st = torch.from_numpy(S).to(DEV)
    field, scale = dfssm.state_field_encode(st)
    got_f = field.cpu().numpy().view(np.uint32)
    assert np.array_equal(scale.cpu().numpy(), s_ref)
    bad = np.nonzero((got_f != f_ref).any(axis=1))[0]
    assert len(bad) == 0, f"{len(bad)} rows' fields differ, first {bad[:5]}"
    back = dfssm.state_field_decode(field, scale, N)
    assert np.array_equal(back.cpu().numpy(), back_ref)
    # in place, with and without the field stored
    st2 = st.clone()
    f2 = torch.full_like(field, -1)
    s2 = torch.full_like(scale, -1.0)
    dfssm.state_field_roundtrip(st2, f2, s2)
    assert np.array_equal(st2.cpu().numpy(), back_ref)
    assert np.array_equal(f2.cpu().numpy().view(np.uint32), f_ref)
    assert np.array_equal(s2.cpu().numpy(), s_ref)
    st3 = st.clone()
    dfssm.state_field_roundtrip(st3)
    assert np.array_equal(st3.cpu().numpy(), back_ref)
    torch.cuda.synchronize()


@pytest.mark.parametrize("N", [8, 16, 24, 40, 72, 104, 128, 160, 176, 200, 256])
@pytest.mark.parametrize("rows", [1, 37, 1029])
def test_field_matches_oracle(dfssm, N, rows):
    """Every lane split (1 to 8 values per lane, ranges cut short at N) over ragged row counts."""
    S = inputs.ssm_state_rows(seed=1000 + N + rows, rows=rows, d_state=N)
    _check_all(dfssm, S)


def test_field_full_state_of_the_48_layer_stack(dfssm):
    """The whole SSM state of the 48-layer Mamba-2-1.3B stack at batch 1 (196,608 rows of 128), the
    configuration bench.py times, compared in full."""
    S = inputs.ssm_state_rows(seed=77, rows=48 * 64 * 64, d_state=128)
    _check_all(dfssm, S)


def test_field_edge_rows(dfssm):
    """Zero rows, the five levels (exact round trip), rows at the top and bottom of the fp32 range,
    denormal quotients, a single nonzero value, a constant row and its negation."""
    g = np.random.default_rng(5)
    N = 128
    rows = []
    rows.append(np.zeros(N, np.float32))
    lev = (g.integers(0, 5, N).astype(np.float32) * np.float32(0.5) - np.float32(1)) * np.float32(3.0)
    lev[7] = 3.0
    rows.append(lev)
    rows.append((g.standard_normal(N) * 1e37).astype(np.float32))
    rows.append((g.standard_normal(N) * 1e-38).astype(np.float32))
    den = (g.standard_normal(N) * 1e-10).astype(np.float32)
    den[0] = 1e30
    rows.append(den)                                        # x = S / c below the normal range
    one = np.zeros(N, np.float32)
    one[N - 1] = -0.75
    rows.append(one)
    rows.append(np.full(N, 2.5, np.float32))
    rows.append(np.full(N, -2.5, np.float32))
    negz = np.zeros(N, np.float32)
    negz[::2] = -0.0
    negz[3] = 1.0
    rows.append(negz)
    S = np.stack(rows).astype(np.float32)
    _check_all(dfssm, S)
    st = torch.from_numpy(S[1:2].copy()).to(DEV)
    dfssm.state_field_roundtrip(st)
    assert np.array_equal(st.cpu().numpy(), S[1:2])          # levels come back exactly


def test_field_zero_rows_launch_nothing(dfssm):
    st = torch.zeros((0, 128), dtype=torch.float32, device=DEV)
    field, scale = dfssm.state_field_encode(st)
    assert field.shape == (0, 16) and scale.shape == (0,)
    out = dfssm.state_field_decode(field, scale, 128)
    assert out.shape == (0, 128)
    dfssm.state_field_roundtrip(st)
    torch.cuda.synchronize()


def test_field_of_a_decoded_state(dfssm):
    """States produced by the oracle's own decode of a small stack (real recurrence statistics)."""
    dims = dict(d_model=256, nheads=4, headdim=32, d_state=64, ngroups=1)
    model = inputs.decode_model(seed=8, n_layers=2, n_tokens=6, batch=1, rank=16, **dims)
    conv, ssm = inputs.zero_states(1, 2, 4, 32, 64, 1)
    layers = [dict(l, in_proj=oracle.Linear.from_dict(l["in_proj"]),
                   out_proj=oracle.Linear.from_dict(l["out_proj"])) for l in model["layers"]]
    for t in range(6):
        h = np.array(model["emb"][t], dtype=np.float32)
        for i, L in enumerate(layers):
            oracle.layer_decode(L, h, conv[i], ssm[i])
    _check_all(dfssm, np.ascontiguousarray(ssm.reshape(-1, 64)))
