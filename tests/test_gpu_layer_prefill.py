"""Parity of the layer prefill (dfssm_layer_prefill: in_proj GEMM with the pre-norm folded in, the conv
and the SSM recurrence over the whole prompt, gate, out_proj GEMM with the gated norm folded in and the
residual add) with the CPU oracle, which runs the decode step token after token.

Bar: the residual stream and the conv / SSM states within max|d| <= 1e-3 * (1 + |ref|).  The linears
and the conv follow the decode definition exactly and the SSM state its rounding sequence; the SSM
readout sum is accumulated in about 48 bits instead of the oracle's fp64 serial sum, so rare last-bit
differences are possible.  After a prefill, decode continues from the states it left.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_mamba_b200 import inputs

pytestmark = pytest.mark.gpu

RTOL = 1e-3
FULL = dict(d_model=2048, nheads=64, headdim=64, d_state=128, ngroups=1)
MID = dict(d_model=256, nheads=4, headdim=32, d_state=32, ngroups=1)


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_mamba_b200 import build, dfssm
    build.build()
    dfssm.lib()
    return torch.device("cuda:0")


def to_dev(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def assert_tol(gpu, ref, what):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, what
    bad = np.abs(gpu - ref) > RTOL * (1 + np.abs(ref))
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance, max |d| {np.abs(gpu - ref).max():.3e}"


def _prefill_compare(dev, dims, n_layers, M, seed, decode_after=2):
    from bit_quantized_mamba_b200 import dfssm
    rank = dims.get("rank", 16)
    d = {k: v for k, v in dims.items() if k != "rank"}
    m = inputs.decode_model(seed=seed, n_layers=n_layers, n_tokens=M + decode_after, rank=rank, **d)
    conv, ssm = inputs.zero_states(1, n_layers, d["nheads"], d["headdim"], d["d_state"], d["ngroups"])
    layers = [dfssm.Layer.from_host(l, dev) for l in m["layers"]]
    stack = dfssm.LayerStack(layers, d, [to_dev(c, dev) for c in conv], [to_dev(s, dev) for s in ssm])
    olayers = []
    for l in m["layers"]:
        ol = dict(l)
        ol["in_proj"] = oracle.Linear.from_dict(l["in_proj"])
        ol["out_proj"] = oracle.Linear.from_dict(l["out_proj"])
        olayers.append(ol)
    prompt = np.ascontiguousarray(m["emb"][:M, 0, :])
    h = to_dev(prompt, dev)
    dfssm.layer_prefill(stack, h)
    ref = oracle.layer_prefill(olayers, prompt.copy(), conv, ssm)
    torch.cuda.synchronize()
    assert_tol(h.cpu().numpy(), ref, f"hidden after prefill of {M}")
    for l in range(n_layers):
        assert_tol(stack.ssm_states[l].cpu().numpy(), ssm[l], f"ssm state layer {l}")
        assert_tol(stack.conv_states[l].cpu().numpy(), conv[l], f"conv state layer {l}")
    # decoding continues from the prefilled states
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LAYER_DECODE, 1, d["d_model"],
                                              d["nheads"] * d["headdim"]), dev)
    for t in range(M, M + decode_after):
        h_ref = np.ascontiguousarray(m["emb"][t][:1])
        hd = to_dev(h_ref, dev)
        dfssm.layer_decode(stack, hd, ws)
        for l in range(n_layers):
            oracle.layer_decode(olayers[l], h_ref, conv[l], ssm[l])
        torch.cuda.synchronize()
        assert_tol(hd.cpu().numpy(), h_ref, f"decode token {t} after prefill")


@pytest.mark.parametrize("M", [1, 2, 17, 200])
def test_layer_prefill_mid_dims(dev, M):
    """d_model 256, 4 heads x 32, d_state 32: prompt lengths below the conv width, one past a staging
    chunk, and a ragged multi-tile prompt; three layers."""
    _prefill_compare(dev, MID, 3, M, seed=70 + M)


def test_layer_prefill_two_groups_wide_state(dev):
    """ngroups 2 (B/C offsets per group) and d_state 160 (two state chunks per lane for some lanes)."""
    dims = dict(d_model=256, nheads=4, headdim=32, d_state=160, ngroups=2, rank=8)
    _prefill_compare(dev, dims, 2, 45, seed=75)


def test_layer_prefill_full_dims(dev):
    """The 1.3B layer shape, 2 layers, a 300-token prompt."""
    _prefill_compare(dev, FULL, 2, 300, seed=76)


def test_layer_prefill_full_2048(dev):
    """The 1.3B layer shape, one layer, the 2048-token prompt of the prefill workload."""
    _prefill_compare(dev, FULL, 1, 2048, seed=77, decode_after=1)


def test_layer_prefill_rejects_unsupported(dev):
    from bit_quantized_mamba_b200 import dfssm
    dims = dict(d_model=64, nheads=4, headdim=16, d_state=16, ngroups=1)  # d_model not a multiple of 128
    m = inputs.decode_model(seed=78, n_layers=1, n_tokens=4, rank=4, **dims)
    conv, ssm = inputs.zero_states(1, 1, 4, 16, 16, 1)
    stack = dfssm.LayerStack([dfssm.Layer.from_host(m["layers"][0], dev)], dims, [to_dev(conv[0], dev)],
                             [to_dev(ssm[0], dev)])
    h = to_dev(np.ascontiguousarray(m["emb"][:, 0, :]), dev)
    ws = dfssm.workspace(1 << 20, dev)
    with pytest.raises(dfssm.DfssmError) as ei:
        dfssm.layer_prefill(stack, h, ws)
    assert ei.value.status == -3
