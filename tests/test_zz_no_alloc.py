"""dfssm_linear_decode_noalloc — the linear decode for callers that cannot allocate device memory
(for example a plugin whose host process owns every device allocation, or a real-time loop that must
not call cudaMalloc) — gives the same results as dfssm_linear_decode, which takes a caller workspace.

Collected last on purpose, so that a run stopping at its first failure has already run the rest; it also
passes when run alone in a fresh process."""
import numpy as np
import pytest
import torch

from bit_quantized_mamba_b200 import inputs

pytestmark = pytest.mark.gpu

RTOL = 1e-3


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_mamba_b200 import build, dfssm
    build.build()
    dfssm.lib()
    return torch.device("cuda:0")


def _taps(B, L, dev):
    return dict(acc=torch.zeros((B, L.d_out), dtype=torch.int32, device=dev),
                lora_t=torch.zeros((B, L.rank), dtype=torch.int32, device=dev),
                xq=torch.zeros((B, L.d_in), dtype=torch.int8, device=dev),
                xscale=torch.zeros(B, dtype=torch.float32, device=dev))


def test_noalloc_matches_workspace_entry_point_on_two_calls(dev):
    from bit_quantized_mamba_b200 import dfssm
    # calls in a row: an in_proj-shaped token (streaming kernel, no scratch), then eight tokens of a
    # d_in = 8192 linear and three of a d_in = 384 linear (both through the shared scratch array)
    for seed, (d_out, d_in, B) in enumerate([(8512, 2048, 1), (1000, 8192, 8), (1000, 384, 3)]):
        g = np.random.default_rng(100 + seed)
        L = dfssm.Linear.from_host(inputs.linear(g, d_out, d_in), dev)
        x = torch.from_numpy(inputs.normal(g, (B, d_in)) * np.float32(1.5)).to(dev)
        ref_taps, got_taps = _taps(B, L, dev), _taps(B, L, dev)
        y_ref = dfssm.linear_decode(L, x, debug=ref_taps)
        y = dfssm.linear_decode_noalloc(L, x, debug=got_taps)
        torch.cuda.synchronize()
        for k in ("acc", "lora_t", "xq", "xscale"):
            assert torch.equal(got_taps[k], ref_taps[k]), (seed, k)
        yr, yg = y_ref.cpu().numpy().astype(np.float64), y.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(yg - yr) <= RTOL * (1 + np.abs(yr))), seed


def test_noalloc_rejects_sizes_beyond_its_array(dev):
    from bit_quantized_mamba_b200 import dfssm
    g = np.random.default_rng(7)
    L = dfssm.Linear.from_host(inputs.linear(g, 64, 256), dev)
    x = torch.zeros((17, 256), dtype=torch.float32, device=dev)
    with pytest.raises(dfssm.DfssmError) as e:
        dfssm.linear_decode_noalloc(L, x)
    assert e.value.status == -3  # DFSSM_EUNSUPPORTED: more than 16 tokens
