"""The host-CPU (AVX-512 VNNI) engine against the oracle, on the CPU (no GPU involved).

The engine (include/dfssm_cpu.h) computes the library's definitions on host memory with the scaffold
GEMV on vpdpbusd; every integer and every fp32 value must equal the oracle's.  Skipped on a CPU without
AVX-512 VNNI.
"""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st
import torch

import oracle
from bit_quantized_mamba_b200 import build, dfssm, inputs


@pytest.fixture(scope="module")
def engine():
    build.build_cpu()
    if not dfssm.cpu_available():
        pytest.skip("host CPU has no AVX-512 VNNI")
    dfssm.cpu_set_threads(0)
    return dfssm


def _host_linear(d):
    return dfssm.Linear.from_host(d, "cpu")


@pytest.mark.parametrize("d_out,d_in,rank,B", [
    (512, 256, 16, 1), (300, 96, 5, 3), (257, 2048, 16, 4), (130, 4096, 0, 16), (64, 32, 7, 2),
    (200, 8192, 16, 5), (96, 160, 1, 16)])
def test_linear_matches_oracle(engine, d_out, d_in, rank, B):
    """Codes, scales, scaffold accumulators, LoRA-down t and outputs bit-identical; d_in % 64 == 32
    cases (96, 160) exercise the half chunk; rank 0 the scaffold alone; an all-zero token the s = 0 row."""
    gen = np.random.default_rng(1000 + d_in + B)
    lin = inputs.linear(gen, d_out, d_in, rank)
    x = inputs.normal(gen, (B, d_in)) * np.float32(3)
    if B > 2:
        x[1] = 0.0
    L = _host_linear(lin)
    dbg = dict(acc=torch.zeros((B, d_out), dtype=torch.int32), lora_t=torch.zeros((B, max(rank, 1)), dtype=torch.int32),
               xq=torch.zeros((B, d_in), dtype=torch.int8), xscale=torch.zeros(B, dtype=torch.float32))
    y = engine.cpu_linear_decode(L, torch.from_numpy(x), debug=dbg).numpy()
    ref = oracle.linear_decode(oracle.Linear.from_dict(lin), x)
    assert np.array_equal(dbg["xq"].numpy(), ref["xq"])
    assert np.array_equal(dbg["xscale"].numpy(), ref["xscale"])
    assert np.array_equal(dbg["acc"].numpy(), ref["acc"])
    if rank:
        assert np.array_equal(dbg["lora_t"].numpy()[:, :rank], ref["t"])
    assert np.array_equal(y, ref["y"]), f"{(y != ref['y']).sum()} outputs differ"


def test_linear_ties(engine):
    """Values exactly halfway between two codes after the division (s = 1 exactly): round half to even."""
    d_in = 256
    x = np.zeros((2, d_in), np.float32)
    x[:, 0] = 127.0
    x[0, 1:64] = np.arange(63, dtype=np.float32) + np.float32(0.5)
    x[1, 1:64] = -(np.arange(63, dtype=np.float32) + np.float32(0.5))
    gen = np.random.default_rng(7)
    lin = inputs.linear(gen, 64, d_in, 16)
    dbg = dict(xq=torch.zeros((2, d_in), dtype=torch.int8))
    y = engine.cpu_linear_decode(_host_linear(lin), torch.from_numpy(x), debug=dbg).numpy()
    ref = oracle.linear_decode(oracle.Linear.from_dict(lin), x)
    assert np.array_equal(dbg["xq"].numpy(), ref["xq"])
    assert np.array_equal(y, ref["y"])


def _stack(model, conv, ssm, dims):
    layers = [dfssm.Layer.from_host(d, "cpu") for d in model["layers"]]
    n = len(layers)
    cs = [torch.from_numpy(conv[i]) for i in range(n)]
    ss = [torch.from_numpy(ssm[i]) for i in range(n)]
    return dfssm.LayerStack(layers, dims, cs, ss), cs, ss


@pytest.mark.parametrize("dims,B,n_layers,n_tokens", [
    (dict(d_model=256, nheads=4, headdim=32, d_state=16, ngroups=1, rank=16), 1, 3, 4),
    (dict(d_model=128, nheads=4, headdim=32, d_state=24, ngroups=2, rank=5), 3, 2, 3),
    (dict(d_model=2048, nheads=64, headdim=64, d_state=128, ngroups=1, rank=16), 1, 2, 2),
    (dict(d_model=64, nheads=8, headdim=28, d_state=12, ngroups=2, rank=3), 2, 2, 3),
])
def test_layer_decode_matches_oracle(engine, dims, B, n_layers, n_tokens):
    """Several tokens through a stack: the residual stream and both states bit-identical to the oracle
    after every token (the 1.3B layer shape included; headdim 28 and d_state 12 take every branch of
    the SSM step: sixteen rows, eight rows, single rows, and state columns past the eight-wide blocks)."""
    d = dict(dims)
    model = inputs.decode_model(seed=21, n_layers=n_layers, n_tokens=n_tokens, batch=B, **d)
    conv, ssm = inputs.zero_states(B, n_layers, d["nheads"], d["headdim"], d["d_state"], d["ngroups"])
    run_dims = {k: d[k] for k in ("d_model", "nheads", "headdim", "d_state", "ngroups")}
    stack, cs, ss = _stack(model, conv.copy(), ssm.copy(), run_dims)
    olayers = [dict(l, in_proj=oracle.Linear.from_dict(l["in_proj"]),
                    out_proj=oracle.Linear.from_dict(l["out_proj"])) for l in model["layers"]]
    oconv, ossm = conv.copy(), ssm.copy()
    for t in range(n_tokens):
        hr = np.array(model["emb"][t], dtype=np.float32)
        h = torch.from_numpy(hr.copy())
        engine.cpu_layer_decode(stack, h)
        for i, ol in enumerate(olayers):
            oracle.layer_decode(ol, hr, oconv[i], ossm[i])
        assert np.array_equal(h.numpy(), hr), f"token {t}: {(h.numpy() != hr).sum()} hidden values differ"
        for i in range(n_layers):
            assert np.array_equal(cs[i].numpy(), oconv[i]), f"token {t} layer {i}: conv state differs"
            assert np.array_equal(ss[i].numpy(), ossm[i]), f"token {t} layer {i}: SSM state differs"


def test_rejects_bad_arguments(engine):
    gen = np.random.default_rng(3)
    L = _host_linear(inputs.linear(gen, 64, 100 * 32 // 32 * 32, 4))
    x = torch.zeros((17, L.d_in), dtype=torch.float32)
    with pytest.raises(dfssm.DfssmError):
        engine.cpu_linear_decode(L, x)  # B > 16
    dev_like = _host_linear(inputs.linear(gen, 64, 64, 4))
    with pytest.raises(ValueError):
        dfssm.linear_decode(dev_like, x[:1, :64])  # a host linear on the CUDA entry point


@pytest.mark.parametrize("N,rows", [(8, 65), (24, 130), (72, 33), (128, 4097), (200, 70), (256, 129)])
def test_state_field_matches_oracle(engine, N, rows):
    """Density-field encode, readout and round trip bit-identical to the oracle's sigma-delta loop."""
    S = inputs.ssm_state_rows(seed=500 + N, rows=rows, d_state=N)
    f_ref, s_ref = oracle.field_encode(S)
    back_ref = oracle.field_decode(f_ref, s_ref, N)
    field, scale = engine.cpu_state_field_encode(torch.from_numpy(S))
    assert np.array_equal(field.numpy().view(np.uint32), f_ref)
    assert np.array_equal(scale.numpy(), s_ref)
    assert np.array_equal(engine.cpu_state_field_decode(field, scale, N).numpy(), back_ref)
    st = torch.from_numpy(S.copy())
    f2, s2 = torch.zeros_like(field), torch.zeros_like(scale)
    engine.cpu_state_field_roundtrip(st, f2, s2)
    assert np.array_equal(st.numpy(), back_ref)
    assert np.array_equal(f2.numpy().view(np.uint32), f_ref) and np.array_equal(s2.numpy(), s_ref)
    st = torch.from_numpy(S.copy())
    engine.cpu_state_field_roundtrip(st)
    assert np.array_equal(st.numpy(), back_ref)


def test_state_field_edge_rows(engine):
    g = np.random.default_rng(6)
    N = 128
    rows = [np.zeros(N, np.float32),
            ((g.integers(0, 5, N) * 0.5 - 1) * 3.0).astype(np.float32),
            (g.standard_normal(N) * 1e37).astype(np.float32),
            (g.standard_normal(N) * 1e-38).astype(np.float32),
            np.full(N, -2.5, np.float32)]
    den = (g.standard_normal(N) * 1e-10).astype(np.float32)
    den[0] = 1e30
    rows.append(den)
    S = np.stack(rows)
    f_ref, s_ref = oracle.field_encode(S)
    field, scale = engine.cpu_state_field_encode(torch.from_numpy(S))
    assert np.array_equal(field.numpy().view(np.uint32), f_ref)
    assert np.array_equal(scale.numpy(), s_ref)
    assert np.array_equal(engine.cpu_state_field_decode(field, scale, N).numpy(),
                          oracle.field_decode(f_ref, s_ref, N))


def test_state_field_binding_rejects_wrong_dtypes(engine):
    with pytest.raises(ValueError):
        engine.cpu_state_field_encode(torch.zeros((4, 128), dtype=torch.float64))
    with pytest.raises(ValueError):
        engine.cpu_state_field_decode(torch.zeros((4, 16), dtype=torch.int64), torch.zeros(4), 128)
    with pytest.raises(ValueError):
        engine.cpu_state_field_decode(torch.zeros((4, 16), dtype=torch.int32),
                                      torch.zeros(4, dtype=torch.float64), 128)
    with pytest.raises(ValueError):
        engine.state_field_encode(torch.zeros((4, 128)))  # a host tensor on the CUDA entry point


@settings(max_examples=200, deadline=None)
@given(st.sampled_from([8, 16, 40, 128]).flatmap(
    lambda n: st.lists(st.floats(width=32, allow_nan=False, allow_infinity=False), min_size=n, max_size=n)))
def test_state_field_arbitrary_rows(vals):
    """The engine's integer closed form against the oracle's loop on arbitrary finite fp32 rows."""
    build.build_cpu()
    if not dfssm.cpu_available():
        pytest.skip("host CPU has no AVX-512 VNNI")
    S = np.array([vals], np.float32)
    N = S.shape[1]
    f_ref, s_ref = oracle.field_encode(S)
    field, scale = dfssm.cpu_state_field_encode(torch.from_numpy(S))
    assert np.array_equal(field.numpy().view(np.uint32), f_ref)
    assert np.array_equal(scale.numpy(), s_ref)


def test_decode_with_field_round_trips_at_chunk_boundaries(engine):
    """The density field applied at chunk boundaries of a decode: every 3 tokens each layer's SSM state
    is replaced by the readout of its encoding, on the engine (dfssm_cpu_state_field_roundtrip) and on
    the oracle (its encode, then its readout).  Residual stream and states stay bit-identical."""
    dims = dict(d_model=256, nheads=4, headdim=32, d_state=64, ngroups=1)
    n_layers, n_tokens, chunk = 2, 7, 3
    model = inputs.decode_model(seed=31, n_layers=n_layers, n_tokens=n_tokens, batch=1, rank=16, **dims)
    conv, ssm = inputs.zero_states(1, n_layers, 4, 32, 64, 1)
    stack, cs, ss = _stack(model, conv.copy(), ssm.copy(), dims)
    olayers = [dict(l, in_proj=oracle.Linear.from_dict(l["in_proj"]),
                    out_proj=oracle.Linear.from_dict(l["out_proj"])) for l in model["layers"]]
    oconv, ossm = conv.copy(), ssm.copy()
    for t in range(n_tokens):
        hr = np.array(model["emb"][t], dtype=np.float32)
        h = torch.from_numpy(hr.copy())
        engine.cpu_layer_decode(stack, h)
        for i, ol in enumerate(olayers):
            oracle.layer_decode(ol, hr, oconv[i], ossm[i])
        if (t + 1) % chunk == 0:
            for i in range(n_layers):
                engine.cpu_state_field_roundtrip(ss[i])
                f, sc = oracle.field_encode(ossm[i])
                ossm[i][...] = oracle.field_decode(f, sc, 64).reshape(ossm[i].shape)
        assert np.array_equal(h.numpy(), hr), f"token {t}: hidden rows differ"
        for i in range(n_layers):
            assert np.array_equal(ss[i].numpy(), ossm[i]), f"token {t} layer {i}: SSM state differs"


@settings(max_examples=40, deadline=None)
@given(d_out=st.integers(1, 300), d_in_words=st.integers(1, 48), rank=st.integers(0, 16),
       B=st.integers(1, 16), seed=st.integers(0, 2 ** 31 - 1))
def test_linear_random_shapes(d_out, d_in_words, rank, B, seed):
    """Random linear shapes (d_out across partial 64-row chunks, d_in = 32..1536 with odd 32-word tails,
    every rank and token count): codes, scales, accumulators, t and outputs bit-identical to the oracle."""
    build.build_cpu()
    if not dfssm.cpu_available():
        pytest.skip("host CPU has no AVX-512 VNNI")
    d_in = 32 * d_in_words
    gen = np.random.default_rng(seed)
    lin = inputs.linear(gen, d_out, d_in, rank)
    x = inputs.normal(gen, (B, d_in)) * np.float32(2)
    dbg = dict(acc=torch.zeros((B, d_out), dtype=torch.int32),
               lora_t=torch.zeros((B, max(rank, 1)), dtype=torch.int32))
    y = dfssm.cpu_linear_decode(dfssm.Linear.from_host(lin, "cpu"), torch.from_numpy(x), debug=dbg).numpy()
    ref = oracle.linear_decode(oracle.Linear.from_dict(lin), x)
    assert np.array_equal(dbg["acc"].numpy(), ref["acc"])
    if rank:
        assert np.array_equal(dbg["lora_t"].numpy()[:, :rank], ref["t"])
    assert np.array_equal(y, ref["y"])
