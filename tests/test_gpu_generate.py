"""Parity of greedy generation (tied int8 embedding, the layer stack, final RMSNorm + int8 LM head,
greedy choice) through the C ABI with the CPU oracle, on the same seeded inputs.

Bar: embeddings, LM-head accumulators, logits and chosen tokens bit-exact for the same fp32 input;
the residual stream after the layers within max|d| <= 1e-3 * (1 + |ref|) (the layer-decode bar).
Generation is checked teacher-forced: the oracle runs the layers on the GPU's tokens, and its head runs
on the GPU's own hidden state, so that a last-bit difference inside the layers can never flip a greedy
choice between the two sides.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_mamba_b200 import inputs

pytestmark = pytest.mark.gpu

RTOL = 1e-3
FULL = dict(d_model=2048, nheads=64, headdim=64, d_state=128, ngroups=1)
SMALL = dict(d_model=64, nheads=4, headdim=16, d_state=16, ngroups=1)


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
    bad = np.abs(gpu - ref) > RTOL * (1 + np.abs(ref))
    assert not bad.any(), f"{what}: {bad.sum()} outside tolerance, max |d| {np.abs(gpu - ref).max():.3e}"
    return int((gpu != ref).sum())


@pytest.fixture(scope="module")
def vocab(dev):
    """The tied 50288 x 2048 int8 matrix, its row scales and the final norm weight."""
    m = inputs.generation_model(seed=5, n_layers=0)
    return m, to_dev(m["emb_w"], dev), to_dev(m["emb_s"], dev), to_dev(m["final_norm_w"], dev)


def test_embed_bit_exact(dev, vocab):
    from bit_quantized_mamba_b200 import dfssm
    m, W, sr, _ = vocab
    V = m["emb_w"].shape[0]
    tok = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_EMBED, 0, 0, 0), dev)
    for t in (0, 1, V - 1, m["first_token"], 31337):
        tok.fill_(t)
        h = dfssm.embed(W, sr, tok, ws=ws).cpu().numpy()
        assert np.array_equal(h, oracle.embed(m["emb_w"], m["emb_s"], t)), t
    assert dfssm.device_status(ws) == 0


def test_embed_rejects_out_of_range_token(dev, vocab):
    """An id outside [0, V) is caught by the kernel's own check: zeros and a reported EINVAL."""
    from bit_quantized_mamba_b200 import dfssm
    m, W, sr, _ = vocab
    V = m["emb_w"].shape[0]
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_EMBED, 0, 0, 0), dev)
    for bad in (V, -1):
        h = torch.full((2048,), 7.0, device=dev)
        dfssm.embed(W, sr, torch.tensor([bad], dtype=torch.int32, device=dev), h, ws=ws)
        assert dfssm.device_status(ws) == -1
        assert not h.any()
    assert dfssm.device_status(ws) == 0  # the status word was cleared by the read


@pytest.mark.parametrize("norm", [True, False])
def test_head_greedy_bit_exact(dev, vocab, norm):
    """Full vocabulary: accumulators, logits and the greedy token equal the oracle's; two calls on one
    workspace (the greedy scratch is left zero by each call)."""
    from bit_quantized_mamba_b200 import dfssm
    m, W, sr, fw = vocab
    V, d = m["emb_w"].shape
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_HEAD_GREEDY, 1, d, V), dev)
    g = np.random.default_rng(60 + norm)
    for call in range(2):
        h = (inputs.normal(g, (d,)) * (0.3 + 2 * call)).astype(np.float32)
        acc = torch.zeros(V, dtype=torch.int32, device=dev)
        tok, logits = dfssm.head_greedy(W, sr, to_dev(h, dev), fw if norm else None, acc=acc, ws=ws)
        rl, racc = oracle.final_head(m["emb_w"], m["emb_s"], h, m["final_norm_w"] if norm else None)
        assert np.array_equal(acc.cpu().numpy(), racc)
        assert np.array_equal(logits.cpu().numpy(), rl)
        assert int(tok.item()) == oracle.greedy(rl)
    assert not ws.any()


def test_head_greedy_ties_take_the_smallest_index(dev):
    """Three identical rows with the largest possible sum: the first of them is chosen."""
    from bit_quantized_mamba_b200 import dfssm
    V, d = 60001, 2048
    g = np.random.default_rng(61)
    W = g.integers(-127, 128, size=(V, d), dtype=np.int8)
    s_row = g.uniform(1e-4, 9e-4, size=V).astype(np.float32)
    h = inputs.normal(g, (d,))
    nw = g.uniform(0.5, 1.5, d).astype(np.float32)
    best = (127 * np.sign(h)).astype(np.int8)
    for r in (40000, 7, 1000):
        W[r] = best
        s_row[r] = 1e-3
    tok, logits = dfssm.head_greedy(to_dev(W, dev), to_dev(s_row, dev), to_dev(h, dev), to_dev(nw, dev))
    rl, _ = oracle.final_head(W, s_row, h, nw)
    assert np.array_equal(logits.cpu().numpy(), rl)
    assert rl[7] == rl[1000] == rl[40000] == rl.max()
    assert int(tok.item()) == 7 == oracle.greedy(rl)


@pytest.mark.parametrize("V,d", [(1, 16), (5, 64), (1187, 4096)])
def test_head_greedy_small_vocabularies(dev, V, d):
    """Fewer rows than warps (most warps own no row) and other widths."""
    from bit_quantized_mamba_b200 import dfssm
    g = np.random.default_rng(V + d)
    W = g.integers(-127, 128, size=(V, d), dtype=np.int8)
    s_row = g.uniform(1e-4, 1e-3, size=V).astype(np.float32)
    h = inputs.normal(g, (d,))
    nw = g.uniform(0.5, 1.5, d).astype(np.float32)
    tok, logits = dfssm.head_greedy(to_dev(W, dev), to_dev(s_row, dev), to_dev(h, dev), to_dev(nw, dev))
    rl, _ = oracle.final_head(W, s_row, h, nw)
    assert np.array_equal(logits.cpu().numpy(), rl)
    assert int(tok.item()) == oracle.greedy(rl)


def _generate_compare(dev, m, dims, n_tokens):
    from bit_quantized_mamba_b200 import dfssm
    n = len(m["layers"])
    conv, ssm = inputs.zero_states(1, n, dims["nheads"], dims["headdim"], dims["d_state"],
                                   dims["ngroups"])
    layers = [dfssm.Layer.from_host(l, dev) for l in m["layers"]]
    stack = dfssm.LayerStack(layers, dims, [to_dev(c, dev) for c in conv], [to_dev(s, dev) for s in ssm])
    W, sr, fw = to_dev(m["emb_w"], dev), to_dev(m["emb_s"], dev), to_dev(m["final_norm_w"], dev)
    V = m["emb_w"].shape[0]
    tokens = torch.zeros(n_tokens + 1, dtype=torch.int32, device=dev)
    tokens[0] = m["first_token"]
    taps = torch.zeros((n_tokens, dims["d_model"]), dtype=torch.float32, device=dev)
    last = torch.zeros(V, dtype=torch.float32, device=dev)
    gws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_GENERATE, V, dims["d_model"],
                                               dims["nheads"] * dims["headdim"]), dev)
    dfssm.generate(stack, W, sr, fw, tokens, hidden_taps=taps, logits=last, ws=gws)
    assert dfssm.device_status(gws) == 0
    gt = [int(t) for t in tokens.cpu().numpy()]
    taps = taps.cpu().numpy()
    olayers = []
    for l in m["layers"]:
        ol = dict(l)
        ol["in_proj"] = oracle.Linear.from_dict(l["in_proj"])
        ol["out_proj"] = oracle.Linear.from_dict(l["out_proj"])
        olayers.append(ol)
    _, hid, _ = oracle.generate(olayers, m["emb_w"], m["emb_s"], m["final_norm_w"], gt[0], n_tokens,
                                conv, ssm, forced_tokens=gt)
    mism = 0
    for t in range(n_tokens):
        mism += assert_tol(taps[t], hid[t], f"hidden after step {t}")
        rl, _ = oracle.final_head(m["emb_w"], m["emb_s"], taps[t], m["final_norm_w"])
        assert gt[t + 1] == oracle.greedy(rl), f"step {t}"
        if t == n_tokens - 1:
            assert np.array_equal(last.cpu().numpy(), rl)
    for l in range(n):
        mism += assert_tol(stack.ssm_states[l].cpu().numpy(), ssm[l], f"ssm state layer {l}")
    return gt, mism


def test_generate_full_48_layers(dev):
    """The 1.3B shape (fused 48-layer decode), the 50288-token tied matrix, 4 greedy steps."""
    m = inputs.generation_model(seed=5)
    gt, mism = _generate_compare(dev, m, FULL, 4)
    print(f"generated {gt}; {mism} fp32 values differ in the last bits")


def test_generate_small_chain(dev):
    """Small dims (the per-op kernel chain), 3 layers, vocabulary 300, 6 greedy steps."""
    m = inputs.generation_model(seed=62, n_layers=3, vocab=300, rank=4, **SMALL)
    gt, _ = _generate_compare(dev, m, SMALL, 6)
    assert len(set(gt)) > 1


def test_generate_in_a_cuda_graph_matches_eager(dev):
    """Captured once and replayed, generation gives the eager call's tokens."""
    from bit_quantized_mamba_b200 import dfssm
    m = inputs.generation_model(seed=63, n_layers=2, vocab=300, rank=4, **SMALL)
    W, sr, fw = to_dev(m["emb_w"], dev), to_dev(m["emb_s"], dev), to_dev(m["final_norm_w"], dev)
    layers = [dfssm.Layer.from_host(l, dev) for l in m["layers"]]

    def fresh():
        conv, ssm = inputs.zero_states(1, 2, 4, 16, 16, 1)
        return dfssm.LayerStack(layers, SMALL, [to_dev(c, dev) for c in conv],
                                [to_dev(s, dev) for s in ssm])

    eager = torch.zeros(9, dtype=torch.int32, device=dev)
    eager[0] = m["first_token"]
    dfssm.generate(fresh(), W, sr, fw, eager)
    stack = fresh()
    toks = torch.zeros(9, dtype=torch.int32, device=dev)
    toks[0] = m["first_token"]
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_GENERATE, 300, 64, 64), dev)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        dfssm.generate(stack, W, sr, fw, toks, ws=ws, stream=torch.cuda.current_stream())
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(toks, eager)
