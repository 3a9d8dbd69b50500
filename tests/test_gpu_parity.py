"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on the same seeded inputs.

Bar: integer intermediates (scaffold accumulators, LoRA-down accumulators, int8 codes) bit-exact; fp32
outputs and states within max|d| <= 1e-3 * (1 + |ref|).  The library evaluates every fp32 value that
feeds a quantizer exactly as the oracle defines it, so the fp32 results are also expected to be
bit-identical except for rare last-bit differences of fp64 reductions; the tests report that count.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_mamba_b200 import inputs

pytestmark = pytest.mark.gpu

RTOL = 1e-3


def assert_tol(gpu, ref, what):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, what
    bad = np.abs(gpu - ref) > RTOL * (1 + np.abs(ref))
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; max |d| = "
                           f"{np.abs(gpu - ref).max():.3e}")
    return int((gpu != ref).sum())


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


def run_linear(lin_host, x, dev):
    from bit_quantized_mamba_b200 import dfssm
    L = dfssm.Linear.from_host(lin_host, dev)
    B = x.shape[0]
    dbg = dict(acc=torch.zeros((B, L.d_out), dtype=torch.int32, device=dev),
               lora_t=torch.zeros((B, max(L.rank, 1)), dtype=torch.int32, device=dev),
               xq=torch.zeros((B, L.d_in), dtype=torch.int8, device=dev),
               xscale=torch.zeros(B, dtype=torch.float32, device=dev))
    y = dfssm.linear_decode(L, to_dev(x, dev), debug=dbg)
    torch.cuda.synchronize()
    out = {k: v.cpu().numpy() for k, v in dbg.items()}
    out["lora_t"] = out["lora_t"][:, :L.rank]
    out["y"] = y.cpu().numpy()
    return out


def compare_linear(g, r, what):
    assert np.array_equal(g["xq"], r["xq"]), f"{what}: int8 codes differ"
    assert np.array_equal(g["xscale"], r["xscale"]), f"{what}: scales differ"
    assert np.array_equal(g["acc"], r["acc"]), f"{what}: scaffold accumulators differ"
    assert np.array_equal(g["lora_t"], r["t"]), f"{what}: LoRA-down accumulators differ"
    return assert_tol(g["y"], r["y"], what)


def test_linear_tiny(dev):
    d = inputs.tiny_linear(0)
    g = run_linear(d["linear"], d["x"], dev)
    r = oracle.linear_decode(oracle.Linear.from_dict(d["linear"]), d["x"])
    assert compare_linear(g, r, "tiny") == 0


def _rand_linear(seed, d_out, d_in, rank):
    gen = np.random.default_rng(seed)
    return inputs.linear(gen, d_out, d_in, rank) if rank else dict(
        inputs.linear(gen, d_out, d_in, 1), lora_b=np.zeros((0, d_in), np.int8),
        lora_b_scale=np.zeros(0, np.float32), lora_a=np.zeros((d_out, 0), np.int8))


@pytest.mark.parametrize("d_out,d_in,rank,B", [
    (1, 32, 0, 1), (33, 64, 1, 2), (127, 96, 7, 3), (129, 160, 16, 5), (512, 256, 16, 16),
    (300, 384, 16, 4), (257, 1024, 16, 1), (1000, 8192, 16, 2), (8512, 2048, 16, 3),
    (2048, 4096, 16, 16), (77, 512, 16, 1), (1, 128, 0, 1), (640, 256, 5, 4), (8512, 2048, 16, 1),
    (2048, 4096, 16, 4), (1100, 1024, 1, 2), (8512, 2048, 16, 5), (1030, 1024, 3, 9),
    (8512, 2048, 16, 16), (4097, 4096, 16, 13), (300, 1024, 0, 16)])
def test_linear_shapes(dev, d_out, d_in, rank, B):
    lin = _rand_linear(d_out * 7 + d_in + rank + B, d_out, d_in, rank)
    gen = np.random.default_rng(B)
    x = inputs.normal(gen, (B, d_in)) * np.float32(2.5)
    if B > 1:
        x[1] = 0.0  # an all-zero token: s = 0, q = 0
    g = run_linear(lin, x, dev)
    r = oracle.linear_decode(oracle.Linear.from_dict(lin), x)
    assert compare_linear(g, r, f"{d_out}x{d_in} r{rank} B{B}") == 0


@pytest.mark.parametrize("d_out,d_in,B", [(700, 2048, 16), (300, 1024, 4), (130, 4096, 16)])
def test_linear_lora_sum_exactness_paths(dev, d_out, d_in, B):
    """The multi-token epilogue takes a block of eight tokens' LoRA sums on the fp64 tensor core only
    when every partial sum is exact (each token's nonzero tf within 18 binades), else the sequential
    chain.  W_B row 15 picks one input (t_15 = q[i0], sB_15 = 1e-5): tokens whose x[i0] quantizes to 127
    stay exact, tokens with a code of +-1 do not, and x[i0] = 0 gives tf_15 = 0 (exact)."""
    gen = np.random.default_rng(d_in + B)
    lin = inputs.linear(gen, d_out, d_in, 16)
    i0 = 5
    lin["lora_b"][15] = 0
    lin["lora_b"][15, i0] = 1
    lin["lora_b_scale"][15] = np.float32(1e-5)
    x = inputs.normal(gen, (B, d_in))
    for b in range(B):
        x[b, i0] = np.abs(x[b]).max() if b % 3 else 0.0
    x[B - 1, i0] = np.abs(x[B - 1]).max() / 127.0  # code +-1: its block takes the chain
    g = run_linear(lin, x, dev)
    r = oracle.linear_decode(oracle.Linear.from_dict(lin), x)
    assert compare_linear(g, r, f"exactness paths {d_out}x{d_in} B{B}") == 0
    assert np.array_equal(g["y"], r["y"])


def test_linear_lora_wide_scales(dev):
    """LoRA-down scales spread over 2^40: every block of the multi-token epilogue takes the sequential
    chain; outputs bit-identical."""
    gen = np.random.default_rng(65)
    lin = inputs.linear(gen, 900, 2048, 16)
    lin["lora_b_scale"] = (2.0 ** np.linspace(-30, 10, 16)).astype(np.float32)
    x = inputs.normal(gen, (16, 2048))
    g = run_linear(lin, x, dev)
    r = oracle.linear_decode(oracle.Linear.from_dict(lin), x)
    assert compare_linear(g, r, "wide LoRA scales") == 0
    assert np.array_equal(g["y"], r["y"])


@pytest.mark.parametrize("which", ["in_proj", "out_proj"])
def test_linear_full_stacks(dev, which):
    """The 48-copy in_proj / out_proj workloads at B = 1, 4, 16: every copy's codes checked, copies
    0 and 47 fully against the oracle, the others on 64 sampled rows."""
    from bit_quantized_mamba_b200 import dfssm
    data = inputs.in_proj_stack() if which == "in_proj" else inputs.out_proj_stack()
    lins = [dfssm.Linear.from_host(l, dev) for l in data["linears"]]
    gen = np.random.default_rng(99)
    for B in (1, 4, 16):
        x = data["x"][:B]
        xd = to_dev(x, dev)
        ys, accs, xqs = [], [], []
        for L in lins:
            dbg = dict(acc=torch.zeros((B, L.d_out), dtype=torch.int32, device=dev),
                       xq=torch.zeros((B, L.d_in), dtype=torch.int8, device=dev))
            ys.append(dfssm.linear_decode(L, xd, debug=dbg))
            accs.append(dbg["acc"])
            xqs.append(dbg["xq"])
        torch.cuda.synchronize()
        rq, rs = oracle.quantize(x)
        for c, host in enumerate(data["linears"]):
            assert np.array_equal(xqs[c].cpu().numpy(), rq)
            OL = oracle.Linear.from_dict(host)
            y = ys[c].cpu().numpy()
            acc = accs[c].cpu().numpy()
            if c in (0, len(lins) - 1):
                r = oracle.linear_decode(OL, x)
                assert np.array_equal(acc, r["acc"]), (which, B, c)
                assert assert_tol(y, r["y"], f"{which} B{B} copy{c}") == 0
            else:
                rows = np.sort(gen.choice(OL.d_out, 64, replace=False))
                for b in range(B):
                    _, rtf = oracle.lora_down(OL, rq[b], rs[b])
                    ry, racc = oracle.linear_rows(OL, rq[b], rs[b], rtf, rows)
                    assert np.array_equal(acc[b, rows], racc), (which, B, c, b)
                    assert assert_tol(y[b, rows], ry, f"{which} B{B} copy{c}") == 0


@pytest.mark.parametrize("which", ["in_proj", "out_proj"])
@pytest.mark.parametrize("B", [1, 4, 16])
def test_linear_multi_matches_per_call(dev, which, B):
    """dfssm_linear_decode_multi over the 48 in_proj (or out_proj) copies equals 48 dfssm_linear_decode
    calls bit for bit; copy 0 is checked in full and copy 47 on sampled rows against the oracle.  Each
    CTA of the multi launch runs through many tiles, so every ring stage is reused several times."""
    from bit_quantized_mamba_b200 import dfssm
    data = (inputs.in_proj_stack if which == "in_proj" else inputs.out_proj_stack)()
    lins = [dfssm.Linear.from_host(l, dev) for l in data["linears"]]
    x = data["x"][:B]
    xd = to_dev(x, dev)
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LINEAR_MULTI, 0, 0, 0), dev)
    ys = dfssm.linear_decode_multi(lins, xd, ws=ws)
    ref = [dfssm.linear_decode(L, xd) for L in lins]
    torch.cuda.synchronize()
    assert dfssm.device_status(ws) == 0  # no wait ran out of budget
    for c in range(len(lins)):
        assert torch.equal(ys[c], ref[c]), c
    r = oracle.linear_decode(oracle.Linear.from_dict(data["linears"][0]), x)
    assert assert_tol(ys[0].cpu().numpy(), r["y"], "multi copy 0") == 0
    OL = oracle.Linear.from_dict(data["linears"][47])
    rq, rs = oracle.quantize(x)
    rows = np.arange(0, OL.d_out, 97)
    y47 = ys[47].cpu().numpy()
    for b in range(B):
        _, rtf = oracle.lora_down(OL, rq[b], rs[b])
        ry, _ = oracle.linear_rows(OL, rq[b], rs[b], rtf, rows)
        assert assert_tol(y47[b, rows], ry, f"multi copy 47 token {b}") == 0


def test_linear_multi_mixed_shapes(dev):
    """Linears of different d_out (ragged tiles, rank 0 and rank < 16) sharing one input."""
    from bit_quantized_mamba_b200 import dfssm
    hosts = [_rand_linear(70 + j, d_out, 1024, rank) for j, (d_out, rank) in
             enumerate([(1, 16), (4353, 16), (129, 0), (300, 3), (2048, 16)])]
    lins = [dfssm.Linear.from_host(h, dev) for h in hosts]
    gen = np.random.default_rng(3)
    x = inputs.normal(gen, (3, 1024))
    x[2] = 0.0
    ys = dfssm.linear_decode_multi(lins, to_dev(x, dev))
    torch.cuda.synchronize()
    for j, h in enumerate(hosts):
        r = oracle.linear_decode(oracle.Linear.from_dict(h), x)
        assert assert_tol(ys[j].cpu().numpy(), r["y"], f"mixed linear {j}") == 0


@pytest.mark.parametrize("d_in,shapes", [
    (1024, [(12000, 16), (8000, 16), (129, 0), (300, 3)]),
    (8192, [(2000, 16), (1000, 5), (17, 16)])])
def test_linear_multi_large_tiles(dev, d_in, shapes):
    """Batch 1 with more 16 KB tiles than SMs: the launch streams 32 KB tiles (256 rows at d_in 1024, 32 at
    8192).  Every output equals the single call's (16 KB tiles) bit for bit and the oracle within
    tolerance."""
    from bit_quantized_mamba_b200 import dfssm
    hosts = [_rand_linear(90 + j, d_out, d_in, rank) for j, (d_out, rank) in enumerate(shapes)]
    lins = [dfssm.Linear.from_host(h, dev) for h in hosts]
    x = inputs.normal(np.random.default_rng(d_in), (1, d_in))
    xd = to_dev(x, dev)
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LINEAR_MULTI, 0, 0, 0), dev)
    ys = dfssm.linear_decode_multi(lins, xd, ws=ws)
    ref = [dfssm.linear_decode(L, xd) for L in lins]
    torch.cuda.synchronize()
    assert dfssm.device_status(ws) == 0
    for j, h in enumerate(hosts):
        assert torch.equal(ys[j], ref[j]), j
        r = oracle.linear_decode(oracle.Linear.from_dict(h), x)
        assert assert_tol(ys[j].cpu().numpy(), r["y"], f"large-tile linear {j}") == 0


def test_linear_multi_rejects_unsupported(dev):
    from bit_quantized_mamba_b200 import dfssm
    g = np.random.default_rng(8)
    lins = [dfssm.Linear.from_host(inputs.linear(g, 64, 384), dev)]
    with pytest.raises(dfssm.DfssmError) as e:
        dfssm.linear_decode_multi(lins, torch.zeros((1, 384), device=dev))
    assert e.value.status == -3  # d_in outside {1024, 2048, 4096, 8192}
    lins = [dfssm.Linear.from_host(inputs.linear(g, 64, 8192), dev)]
    with pytest.raises(dfssm.DfssmError) as e:
        dfssm.linear_decode_multi(lins, torch.zeros((5, 8192), device=dev))
    assert e.value.status == -3  # d_in 8192 takes at most 4 tokens


def test_conv_step(dev):
    from bit_quantized_mamba_b200 import dfssm
    gen = np.random.default_rng(5)
    B, Cn = 2, inputs.CONV_CH
    w = gen.normal(0, 0.1, (Cn, 4)).astype(np.float32)
    b = gen.normal(0, 0.1, Cn).astype(np.float32)
    st_ref = np.zeros((B, Cn, 3), np.float32)
    st = torch.zeros((B, Cn, 3), dtype=torch.float32, device=dev)
    wd, bd = to_dev(w, dev), to_dev(b, dev)
    mism = 0
    for t in range(6):
        x = inputs.normal(gen, (B, Cn)) * np.float32(3)
        out = dfssm.conv_step(st, wd, bd, to_dev(x, dev)).cpu().numpy()
        ref = oracle.conv_step(st_ref, w, b, x)
        mism += assert_tol(out, ref, f"conv step {t}")
        assert np.array_equal(st.cpu().numpy(), st_ref)
    assert mism <= 2


@pytest.mark.parametrize("B,H,P,N,G", [(2, 64, 64, 128, 1), (3, 8, 16, 32, 2), (1, 6, 5, 12, 3)])
def test_ssm_step(dev, B, H, P, N, G):
    from bit_quantized_mamba_b200 import dfssm
    gen = np.random.default_rng(H * N + G)
    A_log = gen.uniform(0, 2.7, H).astype(np.float32)
    dt_bias = gen.uniform(-4, -1, H).astype(np.float32)
    D = gen.uniform(0.5, 1.5, H).astype(np.float32)
    st_ref = (gen.standard_normal((B, H, P, N)) * 0.5).astype(np.float32)
    st = to_dev(st_ref, dev)
    pd = [to_dev(a, dev) for a in (A_log, dt_bias, D)]
    mism = 0
    for t in range(4):
        x = inputs.normal(gen, (B, H * P))
        dt_raw = (inputs.normal(gen, (B, H)) * np.float32(2)).astype(np.float32)
        Bm = inputs.normal(gen, (B, G, N))
        Cm = inputs.normal(gen, (B, G, N))
        y = dfssm.ssm_step(st, to_dev(x, dev), to_dev(dt_raw, dev), *pd, to_dev(Bm, dev),
                           to_dev(Cm, dev)).cpu().numpy()
        yr = oracle.ssm_step(st_ref, x, dt_raw, A_log, dt_bias, D, Bm, Cm)
        mism += assert_tol(y, yr, f"ssm y {t}")
        mism += assert_tol(st.cpu().numpy(), st_ref, f"ssm state {t}")
    assert mism <= 4


SMALL = dict(d_model=256, nheads=8, headdim=32, d_state=64, ngroups=1, rank=16)


def _stack(model, dims, B, dev):
    from bit_quantized_mamba_b200 import dfssm
    n = len(model["layers"])
    conv, ssm = inputs.zero_states(B, n, dims["nheads"], dims["headdim"], dims["d_state"],
                                   dims["ngroups"])
    layers = [dfssm.Layer.from_host(l, dev) for l in model["layers"]]
    conv_d = [to_dev(conv[i], dev) for i in range(n)]
    ssm_d = [to_dev(ssm[i], dev) for i in range(n)]
    stack = dfssm.LayerStack(layers, dims, conv_d, ssm_d)
    olayers = []
    for l in model["layers"]:
        ol = dict(l)
        ol["in_proj"] = oracle.Linear.from_dict(l["in_proj"])
        ol["out_proj"] = oracle.Linear.from_dict(l["out_proj"])
        olayers.append(ol)
    return stack, olayers, conv, ssm


def _decode_compare(dev, model, dims, B, n_tokens, final_only=False):
    from bit_quantized_mamba_b200 import dfssm
    stack, olayers, conv, ssm = _stack(model, dims, B, dev)
    n = len(olayers)
    mism = 0
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LAYER_DECODE, B, dims["d_model"],
                                              dims["nheads"] * dims["headdim"]), dev)
    for t in range(n_tokens):
        h_ref = np.ascontiguousarray(model["emb"][t][:B])
        h = to_dev(h_ref, dev)
        dfssm.layer_decode(stack, h, ws)
        for l in range(n):
            oracle.layer_decode(olayers[l], h_ref, conv[l], ssm[l])
        if not final_only or t == n_tokens - 1:
            torch.cuda.synchronize()
            mism += assert_tol(h.cpu().numpy(), h_ref, f"hidden after token {t}")
    for l in range(n):
        mism += assert_tol(stack.ssm_states[l].cpu().numpy(), ssm[l], f"ssm state layer {l}")
        mism += assert_tol(stack.conv_states[l].cpu().numpy(), conv[l], f"conv state layer {l}")
    return mism


def test_layer_decode_small_stack(dev):
    model = inputs.decode_model(seed=7, n_layers=4, n_tokens=6, batch=2, **SMALL)
    assert _decode_compare(dev, model, SMALL, 2, 6) <= 8


def test_layer_decode_full_48x64(dev):
    """The full 48-layer Mamba-2-1.3B-shaped stack, batch 1, 64 free-running decode steps."""
    model = inputs.decode_model(seed=3)
    dims = dict(d_model=2048, nheads=64, headdim=64, d_state=128, ngroups=1)
    mism = _decode_compare(dev, model, dims, 1, 64, final_only=True)
    print(f"48x64 decode: {mism} fp32 values differ in the last bits (all within tolerance)")


def test_lm_head(dev):
    from bit_quantized_mamba_b200 import dfssm
    p = inputs.prefill(seed=4, m=4)
    x = p["x_in"][-1]
    W = to_dev(p["lm_w"], dev)
    acc = torch.zeros(W.shape[0], dtype=torch.int32, device=dev)
    logits = dfssm.lm_head(W, to_dev(p["lm_s"], dev), to_dev(x, dev), acc=acc).cpu().numpy()
    rl, racc = oracle.lm_head(p["lm_w"], p["lm_s"], x)
    assert np.array_equal(acc.cpu().numpy(), racc)
    assert assert_tol(logits, rl, "lm head") == 0


@pytest.mark.parametrize("V,d,zero", [(1, 16, False), (37, 4096, False), (5003, 8192, False), (300, 2048, True),
                                       (70001, 512, False)])
def test_lm_head_shapes(dev, V, d, zero):
    """Other widths (the in-kernel quantizer's loop edges), row counts below and above one row pair per
    warp, and an all-zero token (s = 0, every code 0, logits 0)."""
    from bit_quantized_mamba_b200 import dfssm
    g = np.random.default_rng(V * 31 + d)
    W = g.integers(-127, 128, size=(V, d), dtype=np.int8)
    s_row = g.uniform(1e-4, 1e-3, size=V).astype(np.float32)
    x = np.zeros(d, np.float32) if zero else inputs.normal(g, (d,))
    acc = torch.zeros(V, dtype=torch.int32, device=dev)
    logits = dfssm.lm_head(to_dev(W, dev), to_dev(s_row, dev), to_dev(x, dev), acc=acc).cpu().numpy()
    rl, racc = oracle.lm_head(W, s_row, x)
    assert np.array_equal(acc.cpu().numpy(), racc)
    assert assert_tol(logits, rl, f"lm head {V}x{d}") == 0
    if zero:
        assert not logits.any()


FULL = dict(d_model=2048, nheads=64, headdim=64, d_state=128, ngroups=1)


def test_layer_decode_fused_few_layers(dev):
    """Batch 1 at the 1.3B shape runs the fused persistent kernel: 3 layers x 5 tokens."""
    model = inputs.decode_model(seed=12, n_layers=3, n_tokens=5)
    assert _decode_compare(dev, model, FULL, 1, 5) <= 4


def test_layer_decode_chain_full_dims_batch2(dev):
    """Batch 2 at the 1.3B shape runs the per-op kernel chain."""
    model = inputs.decode_model(seed=13, n_layers=2, n_tokens=3, batch=2)
    assert _decode_compare(dev, model, FULL, 2, 3) <= 4


def test_device_wait_timeout_is_reported(dev):
    """A device-side wait that can never complete runs out of its budget, records DFSSM_ETIMEOUT and
    returns; the status read clears it and the workspace is usable again."""
    from bit_quantized_mamba_b200 import dfssm
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LAYER_DECODE, 1, 2048, 4096), dev)
    assert dfssm.device_status(ws) == 0
    dfssm.selftest_timeout(ws)
    assert dfssm.device_status(ws) == -5
    assert dfssm.device_status(ws) == 0
    model = inputs.decode_model(seed=14, n_layers=1, n_tokens=1)
    stack, olayers, conv, ssm = _stack(model, FULL, 1, dev)
    h = to_dev(model["emb"][0], dev)
    dfssm.layer_decode(stack, h, ws)
    assert dfssm.device_status(ws) == 0
    h_ref = np.ascontiguousarray(model["emb"][0])
    oracle.layer_decode(olayers[0], h_ref, conv[0], ssm[0])
    assert_tol(h.cpu().numpy(), h_ref, "decode after a reported timeout")


def _prefill_compare(dev, lin_host, x, rows):
    """Prefill through the C ABI vs the oracle: int8 codes and scales of every token exact; scaffold
    accumulators, LoRA-down accumulators and outputs (the decode definition, fp64 epilogue) exact on the
    listed rows."""
    from bit_quantized_mamba_b200 import dfssm
    L = dfssm.Linear.from_host(lin_host, dev)
    M = x.shape[0]
    dbg = dict(acc=torch.zeros((M, L.d_out), dtype=torch.int32, device=dev),
               lora_t=torch.zeros((M, L.rank), dtype=torch.int32, device=dev),
               xq=torch.zeros((M, L.d_in), dtype=torch.int8, device=dev),
               xscale=torch.zeros(M, dtype=torch.float32, device=dev))
    y = dfssm.linear_prefill(L, to_dev(x, dev), debug=dbg)
    torch.cuda.synchronize()
    OL = oracle.Linear.from_dict(lin_host)
    rq, rs = oracle.quantize(x)
    assert np.array_equal(dbg["xq"].cpu().numpy(), rq), "prefill int8 codes differ"
    assert np.array_equal(dbg["xscale"].cpu().numpy(), rs), "prefill scales differ"
    yg, accg, tg = y.cpu().numpy(), dbg["acc"].cpu().numpy(), dbg["lora_t"].cpu().numpy()
    for m in rows:
        t, tf = oracle.lora_down(OL, rq[m], rs[m])
        assert np.array_equal(tg[m], t), f"prefill LoRA-down accumulators differ at row {m}"
        yr, accr = oracle.linear_core(OL, rq[m], rs[m], tf)
        assert np.array_equal(accg[m], accr), f"prefill scaffold accumulators differ at row {m}"
        assert_tol(yg[m], yr, f"prefill y row {m}")
        assert np.array_equal(yg[m], yr), f"prefill y row {m}: {(yg[m] != yr).sum()} values differ"


def test_prefill_ragged_small(dev):
    """M and d_out not multiples of the 128-row x 256-token tile; every row checked."""
    gen = np.random.default_rng(61)
    lin = inputs.linear(gen, 300, 256, 16)
    x = inputs.normal(gen, (200, 256)) * np.float32(2)
    x[7] = 0.0
    _prefill_compare(dev, lin, x, range(200))


def test_prefill_rank_below_16(dev):
    gen = np.random.default_rng(62)
    lin = inputs.linear(gen, 256, 384, 5)
    x = inputs.normal(gen, (130, 384))
    _prefill_compare(dev, lin, x, range(130))


def test_prefill_lora_sum_exactness_paths(dev):
    """The prefill epilogue takes a token block's LoRA sum on the fp64 tensor core only when every partial
    sum is exact (the token's nonzero tf span at most 18 binades), else the sequential chain.  W_B row 15
    picks one input, so t_15 = q[i0]: tokens whose x[i0] quantizes to +-1 get a tf_15 far below the
    others (sequential path for their block), tokens with x[i0] = 0 get tf_15 = 0 (still exact).  Every
    output is compared bit for bit."""
    gen = np.random.default_rng(63)
    lin = inputs.linear(gen, 300, 256, 16)
    i0 = 17
    lin["lora_b"][15] = 0
    lin["lora_b"][15, i0] = 1
    lin["lora_b_scale"][15] = np.float32(1e-5)
    x = inputs.normal(gen, (200, 256))
    x[::2, i0] = 0.0
    for m in range(1, 200, 2):
        x[m, i0] = np.abs(x[m]).max()  # code 127: tf_15 within 2^17 of the largest tf
    for m in (3, 41, 42, 100, 199):
        x[m, i0] = np.abs(x[m]).max() / 127.0  # code +-1: tf_15 about 2^-22 of the largest tf
    _prefill_compare(dev, lin, x, range(200))


def test_prefill_lora_wide_scales(dev):
    """LoRA-down scales spread over ~2^40: no token's sum is provably exact, every block takes the
    sequential chain."""
    gen = np.random.default_rng(64)
    lin = inputs.linear(gen, 260, 384, 16)
    lin["lora_b_scale"] = (2.0 ** np.linspace(-30, 10, 16)).astype(np.float32)
    x = inputs.normal(gen, (70, 384))
    _prefill_compare(dev, lin, x, range(70))


@pytest.mark.parametrize("which", ["in_proj", "out_proj"])
def test_prefill_full_size(dev, which):
    """The 2048-token prefill of the in_proj / out_proj-shaped linears: every token's codes, 12 sampled
    tokens across all output columns."""
    p = inputs.prefill(seed=4, m=2048, vocab=16)
    lin = p["in_proj"] if which == "in_proj" else p["out_proj"]
    x = p["x_in"] if which == "in_proj" else p["x_out"]
    rows = [0, 1, 127, 128, 129, 511, 1000, 1023, 1024, 1500, 2046, 2047]
    _prefill_compare(dev, lin, x, rows)
