"""GPU parity at the quantizer's rounding boundaries.

Random N(0,1) inputs essentially never land on a rounding tie of the per-token int8 quantizer, so the
kernels' tie handling (round half to even after an IEEE fp32 division, reached through a fast reciprocal
path that falls back to the division near a boundary) needs inputs built for it.  Each row below holds:
  * exact ties: values whose quotient fl32(v / s) is k + 1/2 exactly;
  * their fp32 neighbours one to three ulps away, whose quotients sit just off the tie;
  * ordinary values.
Scales are both powers of two (the quotient is exact) and arbitrary (the division rounds).  Rows that go
through an RMSNorm first are built so that the normalized values land on those boundaries: the squares
of the row sum exactly in fp64 in any order (every entry a multiple of 2^-12 below 16), and the norm
weights place fl32(fl32(h r) w) on the targets.  The expected codes, scales and outputs are the oracle's;
the construction only picks inputs (checked against the oracle's own codes: the ties are really there).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_mamba_b200 import inputs

pytestmark = pytest.mark.gpu

RTOL = 1e-3
f32 = np.float32


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


def _targets(s, rng, count):
    """fp32 values v with fl32(v / s) on (or one to three ulps around) a rounding tie k + 1/2, |k| <= 125."""
    out = []
    while len(out) < count:
        k = int(rng.integers(-126, 126))
        base = f32(np.float64(k + 0.5) * np.float64(s))
        for j in (0, -1, 1, -2, 2, -3, 3):
            v = base
            for _ in range(abs(j)):
                v = np.nextafter(v, f32(np.inf) if j > 0 else f32(-np.inf))
            out.append(v)
    return np.array(out[:count], f32)


def tie_rows(B, n, seed, pow2):
    """B rows of length n: row b has absmax amax_b (s = amax/127 a power of two when pow2), a third of
    its entries on or next to rounding ties, the rest ordinary values below the absmax."""
    rng = np.random.default_rng(seed)
    x = np.zeros((B, n), f32)
    for b in range(B):
        if pow2:
            s = f32(2.0 ** int(rng.integers(-8, 3)))
            amax = f32(127) * s
        else:
            amax = f32(rng.uniform(0.5, 40.0))
            s = f32(amax / f32(127))
        row = (rng.uniform(-1, 1, n) * 0.9 * float(amax)).astype(f32)
        idx = rng.permutation(n)
        nt = n // 3
        row[idx[:nt]] = _targets(s, rng, nt)
        row[idx[nt]] = amax if rng.integers(2) else -amax
        x[b] = row
    return x


def count_exact_ties(x):
    """Number of entries whose quotient by the row's quantizer scale (the oracle's) is exactly k + 1/2."""
    _, s = oracle.quantize(x)
    n = 0
    for b in range(x.shape[0]):
        if s[b] == 0:
            continue
        r = (x[b] / s[b]).astype(f32)
        n += int(np.sum(r - np.floor(r) == 0.5))
    return n


def normed_tie_row(n, seed, pow2):
    """(h, w): a row h and RMSNorm weights w such that u = fl32(fl32(h r) w) has ties and near-ties of its
    quantizer, r = fl32(1/sqrt(mean(h^2) + 1e-5)).  Entries of h are multiples of 2^-12 below 16, so their
    squares sum exactly in fp64 in any order and every implementation gets the same r."""
    rng = np.random.default_rng(seed)
    h = (np.round(rng.uniform(-4, 4, n) * 4096) / 4096).astype(f32)
    h[h == 0] = f32(1.0 / 4096)
    ss = float(np.sum(h.astype(np.float64) ** 2))
    r = f32(1.0 / np.sqrt(ss / n + 1e-5))
    t = (h * r).astype(f32)
    w = rng.uniform(0.5, 1.5, n).astype(f32)
    order = np.argsort(-np.abs(t))

    def place(i, target):
        """A weight w with fl32(t_i w) == target (searched among neighbours of target / t_i), or None."""
        c = f32(np.float64(target) / np.float64(t[i]))
        for j in range(-6, 7):
            v = c
            for _ in range(abs(j)):
                v = np.nextafter(v, f32(np.inf) if j > 0 else f32(-np.inf))
            if v > 0 and f32(t[i] * v) == target:
                return v
        return None

    # the absmax position: one of the largest |t|, with a weight that makes |u| = 127 2^k (pow2) or the
    # plain product with a weight of 1.2
    i0 = None
    for i in order[:64]:
        if pow2:
            s = f32(2.0 ** np.floor(np.log2(abs(float(t[i])) * 1.2 / 127)))
            amax = f32(127) * s
            wi = place(i, f32(np.sign(t[i]) * amax))
        else:
            wi = f32(1.2)
            amax = abs(f32(t[i] * wi))
        if wi is not None:
            i0 = i
            w[i] = wi
            break
    assert i0 is not None
    s = f32(amax / f32(127)) if not pow2 else s
    placed = 0
    for i in order:
        if i == i0:
            continue
        if placed >= n // 4:
            break
        # a target of t_i's sign whose magnitude is within 0.5 .. 1.5 times |t_i| and below the absmax
        k = int(np.clip(np.floor(abs(float(t[i])) / float(s)), 0, 125))
        base = f32(np.float64(k + 0.5) * np.float64(s))
        j = int(rng.integers(-2, 3))
        v = base
        for _ in range(abs(j)):
            v = np.nextafter(v, f32(np.inf) if j > 0 else f32(-np.inf))
        wi = place(i, f32(np.sign(t[i]) * v))
        if wi is not None and 0.25 < wi < 4:
            w[i] = wi
            placed += 1
    # keep every other |u| below the absmax
    u = (t * w).astype(f32)
    big = np.abs(u) >= amax
    big[i0] = False
    w[big] = f32(0.5) * w[big]
    return h, w


def normed_tie_count(h, w):
    q, s, u, _ = oracle.rmsnorm_quantize(h[None], w)
    r = (u[0] / s[0]).astype(f32)
    return int(np.sum(r - np.floor(r) == 0.5))


# ---------------------------------------------------------------------------------------- linears

def _linear(seed, d_out, d_in, rank=16):
    return inputs.linear(np.random.default_rng(seed), d_out, d_in, rank)


def _check_linear(dev, lin, x, what):
    from bit_quantized_mamba_b200 import dfssm
    L = dfssm.Linear.from_host(lin, dev)
    B = x.shape[0]
    dbg = dict(acc=torch.zeros((B, L.d_out), dtype=torch.int32, device=dev),
               lora_t=torch.zeros((B, L.rank), dtype=torch.int32, device=dev),
               xq=torch.zeros((B, L.d_in), dtype=torch.int8, device=dev),
               xscale=torch.zeros(B, dtype=torch.float32, device=dev))
    y = dfssm.linear_decode(L, to_dev(x, dev), debug=dbg).cpu().numpy()
    r = oracle.linear_decode(oracle.Linear.from_dict(lin), x)
    assert np.array_equal(dbg["xq"].cpu().numpy(), r["xq"]), f"{what}: int8 codes differ"
    assert np.array_equal(dbg["xscale"].cpu().numpy(), r["xscale"]), f"{what}: scales differ"
    assert np.array_equal(dbg["acc"].cpu().numpy(), r["acc"]), f"{what}: accumulators differ"
    assert np.array_equal(dbg["lora_t"].cpu().numpy(), r["t"]), f"{what}: LoRA-down differs"
    assert np.all(np.abs(y - r["y"]) <= RTOL * (1 + np.abs(r["y"]))), what


@pytest.mark.parametrize("d_in", [1024, 2048, 4096])
@pytest.mark.parametrize("B", [1, 4, 16])
@pytest.mark.parametrize("pow2", [True, False])
def test_ties_stream_linear(dev, d_in, B, pow2):
    """The streaming kernel (its in-CTA quantizer) at 1, 4 and 16 tokens."""
    x = tie_rows(B, d_in, seed=d_in + B + pow2, pow2=pow2)
    assert count_exact_ties(x) >= B * 10
    _check_linear(dev, _linear(d_in + B, 300, d_in), x, f"stream d_in {d_in} B {B} pow2 {pow2}")


@pytest.mark.parametrize("B", [1, 3])
def test_ties_quant_kernel_path(dev, B):
    """d_in 384 runs the separate quantize kernel and the fallback GEMV."""
    for pow2 in (True, False):
        x = tie_rows(B, 384, seed=40 + B + pow2, pow2=pow2)
        assert count_exact_ties(x) >= B * 10
        _check_linear(dev, _linear(41, 257, 384), x, f"d_in 384 B {B} pow2 {pow2}")


def test_ties_linear_multi(dev):
    from bit_quantized_mamba_b200 import dfssm
    hosts = [_linear(50 + j, d_out, 2048) for j, d_out in enumerate((700, 8512, 33))]
    lins = [dfssm.Linear.from_host(h, dev) for h in hosts]
    for B, pow2 in ((1, True), (4, False), (16, False)):
        x = tie_rows(B, 2048, seed=60 + B, pow2=pow2)
        ys = dfssm.linear_decode_multi(lins, to_dev(x, dev))
        torch.cuda.synchronize()
        for j, h in enumerate(hosts):
            r = oracle.linear_decode(oracle.Linear.from_dict(h), x)
            y = ys[j].cpu().numpy()
            assert np.array_equal(y, r["y"]), f"multi linear {j} B {B}: {(y != r['y']).sum()} differ"


@pytest.mark.parametrize("pow2", [True, False])
def test_ties_prefill(dev, pow2):
    from bit_quantized_mamba_b200 import dfssm
    M, d_in = 200, 1024
    x = tie_rows(M, d_in, seed=70 + pow2, pow2=pow2)
    lin = _linear(71, 384, d_in)
    L = dfssm.Linear.from_host(lin, dev)
    dbg = dict(acc=torch.zeros((M, L.d_out), dtype=torch.int32, device=dev),
               lora_t=torch.zeros((M, L.rank), dtype=torch.int32, device=dev),
               xq=torch.zeros((M, d_in), dtype=torch.int8, device=dev),
               xscale=torch.zeros(M, dtype=torch.float32, device=dev))
    y = dfssm.linear_prefill(L, to_dev(x, dev), debug=dbg).cpu().numpy()
    r = oracle.linear_decode(oracle.Linear.from_dict(lin), x)
    assert np.array_equal(dbg["xq"].cpu().numpy(), r["xq"]), "prefill codes differ"
    assert np.array_equal(dbg["xscale"].cpu().numpy(), r["xscale"]), "prefill scales differ"
    assert np.array_equal(dbg["acc"].cpu().numpy(), r["acc"]), "prefill accumulators differ"
    assert np.array_equal(y, r["y"]), "prefill outputs differ"


@pytest.mark.parametrize("pow2", [True, False])
def test_ties_lm_head(dev, pow2):
    from bit_quantized_mamba_b200 import dfssm
    g = np.random.default_rng(80)
    V, d = 3000, 2048
    W = g.integers(-127, 128, (V, d), dtype=np.int8)
    sr = g.uniform(1e-4, 1e-3, V).astype(f32)
    x = tie_rows(1, d, seed=81 + pow2, pow2=pow2)[0]
    acc = torch.zeros(V, dtype=torch.int32, device=dev)
    lg = dfssm.lm_head(to_dev(W, dev), to_dev(sr, dev), to_dev(x, dev), acc=acc).cpu().numpy()
    rl, racc = oracle.lm_head(W, sr, x)
    assert np.array_equal(acc.cpu().numpy(), racc) and np.array_equal(lg, rl)


@pytest.mark.parametrize("pow2", [True, False])
def test_ties_head_with_final_norm(dev, pow2):
    """The greedy head's in-CTA RMSNorm + quantizer on a row whose normalized values sit on ties."""
    from bit_quantized_mamba_b200 import dfssm
    g = np.random.default_rng(82)
    V, d = 3000, 2048
    W = g.integers(-127, 128, (V, d), dtype=np.int8)
    sr = g.uniform(1e-4, 1e-3, V).astype(f32)
    h, w = normed_tie_row(d, seed=83 + pow2, pow2=pow2)
    assert normed_tie_count(h, w) >= 20
    acc = torch.zeros(V, dtype=torch.int32, device=dev)
    tok, lg = dfssm.head_greedy(to_dev(W, dev), to_dev(sr, dev), to_dev(h, dev), norm_w=to_dev(w, dev),
                                acc=acc)
    rl, racc = oracle.final_head(W, sr, h, w)
    assert np.array_equal(acc.cpu().numpy(), racc)
    assert np.array_equal(lg.cpu().numpy(), rl)
    assert int(tok.cpu()[0]) == oracle.greedy(rl)


# --------------------------------------------------------------------------------- layer decode

FULL = dict(d_model=2048, nheads=64, headdim=64, d_state=128, ngroups=1)


@pytest.mark.parametrize("B", [1, 2])
def test_ties_layer_decode_pre_norm(dev, B):
    """The first layer's pre-norm quantizer on rows whose normalized values sit on ties: the fused
    persistent kernel (B = 1) and the per-op chain (B = 2).  A single differing code would move every
    in_proj output, so the residual stream after the layer must equal the oracle's bit for bit."""
    from bit_quantized_mamba_b200 import dfssm
    model = inputs.decode_model(seed=90 + B, n_layers=2, n_tokens=1, batch=B)
    # one norm weight per layer: row 0's ties are placed through it; a second row (B = 2) is another
    # exact-sum row through the same weights
    hs, ws = zip(*[normed_tie_row(2048, seed=91 + b, pow2=(b == 0)) for b in range(B)])
    model["layers"][0]["norm_w"] = ws[0]
    h0 = np.stack(hs).astype(f32)
    assert normed_tie_count(h0[0], ws[0]) >= 20
    n = 2
    conv, ssm = inputs.zero_states(B, n, 64, 64, 128, 1)
    layers = [dfssm.Layer.from_host(l, dev) for l in model["layers"]]
    stack = dfssm.LayerStack(layers, FULL, [to_dev(conv[i], dev) for i in range(n)],
                             [to_dev(ssm[i], dev) for i in range(n)])
    h = to_dev(h0, dev)
    dfssm.layer_decode(stack, h)
    h_ref = h0.copy()
    for i, l in enumerate(model["layers"]):
        ol = dict(l, in_proj=oracle.Linear.from_dict(l["in_proj"]),
                  out_proj=oracle.Linear.from_dict(l["out_proj"]))
        oracle.layer_decode(ol, h_ref, conv[i], ssm[i])
    got = h.cpu().numpy()
    assert np.array_equal(got, h_ref), f"{(got != h_ref).sum()} of {got.size} hidden values differ"
