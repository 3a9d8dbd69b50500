"""Pins for the CPU oracle: checks against what the pages and the mathematics fix, never against the
oracle's own formulas retyped.  CPU only.

Each test names the plausible mistake it would catch.
"""
import os

from decimal import Decimal, getcontext

import numpy as np
import pytest
from scipy.special import expit

import oracle
from bit_quantized_mamba_b200 import inputs


def unpack_pm1(bits: np.ndarray) -> np.ndarray:
    """Independent unpack: numpy's little-endian bit order over the little-endian words."""
    d_out, words = bits.shape
    b = np.unpackbits(bits.view(np.uint8).reshape(d_out, words * 4), axis=1, bitorder="little")
    return b.astype(np.int64) * 2 - 1


def pack_pm1(signs: np.ndarray) -> np.ndarray:
    """Independent pack of a +-1 matrix into LSB-first uint32 words."""
    d_out, d_in = signs.shape
    by = np.packbits((signs > 0).astype(np.uint8), axis=1, bitorder="little")
    return np.ascontiguousarray(by).view(np.uint32).reshape(d_out, d_in // 32)


# ------------------------------------------------------------------------------------- sign expansion

def test_sign_exhaustive_byte_patterns():
    """Every byte pattern in every byte lane: catches a wrong bit order (MSB-first), a wrong word index
    or an inverted sign convention."""
    rows = np.arange(256, dtype=np.uint32)
    bits = np.zeros((256, 2), np.uint32)
    for lane in range(4):
        bits[:, 0] |= rows << (8 * lane)
    bits[:, 1] = ~bits[:, 0]
    for o in range(256):
        for i in range(64):
            word, j = divmod(i, 32)
            byte_val = o if word == 0 else (255 - o)
            expected = 1 if (byte_val >> (j % 8)) & 1 else -1
            assert oracle.sign(bits, 64, o, i) == expected, (o, i)


def test_sign_random_round_trip():
    g = np.random.default_rng(11)
    signs = g.choice(np.array([-1, 1]), size=(24, 96))
    bits = pack_pm1(signs)
    for o in range(24):
        for i in range(96):
            assert oracle.sign(bits, 96, o, i) == signs[o, i]


# ------------------------------------------------------------------------------------------ quantizer

def test_quantize_absmax_and_error_bound():
    g = np.random.default_rng(5)
    x = g.standard_normal((6, 1000)).astype(np.float32) * np.float32(3.0)
    q, s = oracle.quantize(x)
    for b in range(6):
        k = np.argmax(np.abs(x[b]))
        assert abs(int(q[b, k])) == 127 and np.sign(q[b, k]) == np.sign(x[b, k])
        assert np.all(np.abs(q[b]) <= 127)
        err = np.abs(x[b].astype(np.float64) - float(s[b]) * q[b].astype(np.float64))
        assert err.max() <= float(s[b]) / 2 * (1 + 2.0 ** -18)
        # s is absmax/127 to fp32 precision
        assert abs(float(s[b]) * 127 - np.abs(x[b]).max()) <= 1e-6 * np.abs(x[b]).max()


def test_quantize_round_half_even_ties():
    """absmax 127 gives s == 1 exactly, so codes are rint(x): ties must go to even."""
    x = np.array([[127.0, 2.5, 3.5, -2.5, 0.5, -0.5, 1.5, 126.5]], np.float32)
    q, s = oracle.quantize(x)
    assert s[0] == 1.0
    assert q[0].tolist() == [127, 2, 4, -2, 0, 0, 2, 126]


def test_quantize_power_of_two_invariance():
    g = np.random.default_rng(6)
    x = g.standard_normal((3, 513)).astype(np.float32)
    q, s = oracle.quantize(x)
    for k in (-7, -1, 3, 10):
        q2, s2 = oracle.quantize(x * np.float32(2.0 ** k))
        assert np.array_equal(q, q2)
        assert np.array_equal(s2, s * np.float32(2.0 ** k))


def test_quantize_zero_row():
    q, s = oracle.quantize(np.zeros((2, 64), np.float32))
    assert np.all(q == 0) and np.all(s == 0)


def test_quantize_matches_ieee_fp32_division():
    """The fp64-then-round division equals numpy's IEEE fp32 division (no double-rounding slip)."""
    g = np.random.default_rng(7)
    x = g.standard_normal((50, 4096)).astype(np.float32)
    q, s = oracle.quantize(x)
    for b in range(50):
        m = np.abs(x[b]).max()
        s32 = np.float32(m) / np.float32(127.0)
        assert s32 == s[b]
        r = (x[b] / s32).astype(np.float32)
        assert np.array_equal(np.clip(np.rint(r), -127, 127).astype(np.int8), q[b])


# --------------------------------------------------------------------------------- scaffold GEMV

@pytest.fixture(scope="module")
def tiny():
    return inputs.tiny_linear(0)


def test_gemv_brute_force_tiny(tiny):
    """acc equals an explicit +-1 integer matmul (the brute-force tiny GEMV)."""
    L = oracle.Linear.from_dict(tiny["linear"])
    out = oracle.linear_decode(L, tiny["x"])
    S = unpack_pm1(L.bits)
    q = out["xq"][0].astype(np.int64)
    assert np.array_equal(out["acc"][0].astype(np.int64), S @ q)
    # identity acc = 2*sum_{bit=1} q - sum q
    ones = (S > 0).astype(np.int64)
    assert np.array_equal(out["acc"][0], 2 * (ones @ q) - q.sum())


def test_gemv_bit_flip_negates_and_all_ones(tiny):
    L = oracle.Linear.from_dict(tiny["linear"])
    base = oracle.linear_decode(L, tiny["x"])
    d = dict(tiny["linear"])
    d["bits"] = ~L.bits
    flipped = oracle.linear_decode(oracle.Linear.from_dict(d), tiny["x"])
    assert np.array_equal(flipped["acc"], -base["acc"])
    d["bits"] = np.full_like(L.bits, 0xFFFFFFFF)
    allones = oracle.linear_decode(oracle.Linear.from_dict(d), tiny["x"])
    assert np.all(allones["acc"][0] == base["xq"][0].astype(np.int64).sum())


def test_gemv_one_hot_input(tiny):
    L = oracle.Linear.from_dict(tiny["linear"])
    S = unpack_pm1(L.bits)
    for j in (0, 31, 32, 200, 255):
        x = np.zeros((1, 256), np.float32)
        x[0, j] = -2.0
        out = oracle.linear_decode(L, x)
        assert out["xq"][0, j] == -127
        assert np.array_equal(out["acc"][0], -127 * S[:, j])


# ------------------------------------------------------------------------------------------- LoRA

def test_lora_rank0_equals_scaffold_alone(tiny):
    """r = 0 gives the scaffold alone; W_A = 0 gives the same, bit for bit."""
    d = dict(tiny["linear"])
    full = oracle.linear_decode(oracle.Linear.from_dict(d), tiny["x"])
    r0 = dict(d, lora_b=np.zeros((0, 256), np.int8), lora_b_scale=np.zeros(0, np.float32),
              lora_a=np.zeros((512, 0), np.int8))
    out0 = oracle.linear_decode(oracle.Linear.from_dict(r0), tiny["x"])
    wa0 = dict(d, lora_a=np.zeros_like(d["lora_a"]))
    outa = oracle.linear_decode(oracle.Linear.from_dict(wa0), tiny["x"])
    assert np.array_equal(out0["y"], outa["y"])
    assert np.array_equal(out0["acc"], full["acc"])
    s = float(out0["xscale"][0])
    expect = (out0["acc"][0].astype(np.float64) * s * d["w_scale"].astype(np.float64))
    assert np.allclose(out0["y"][0], expect, rtol=2e-7, atol=0)
    assert not np.array_equal(full["y"], out0["y"])  # the LoRA term is not silently dropped


def test_lora_one_hot_down_rows(tiny):
    """A one-hot W_B row picks one activation code: t[r] = q_j exactly, tf[r] = fl32(q_j * sB[r] * s)."""
    d = dict(tiny["linear"])
    cols = [3, 17, 100, 255, 0, 64, 128, 129, 5, 6, 7, 8, 9, 10, 11, 12]
    lb = np.zeros((16, 256), np.int8)
    for r, c in enumerate(cols):
        lb[r, c] = 1
    out = oracle.linear_decode(oracle.Linear.from_dict(dict(d, lora_b=lb)), tiny["x"])
    q = out["xq"][0]
    assert np.array_equal(out["t"][0], q[cols].astype(np.int32))
    s = float(out["xscale"][0])
    t, tf = oracle.lora_down(oracle.Linear.from_dict(dict(d, lora_b=lb)), q, s)
    expect = q[cols].astype(np.float64) * d["lora_b_scale"].astype(np.float64) * s
    assert np.allclose(tf, expect, rtol=2 ** -24, atol=0)


def test_lora_down_brute_force_integer():
    """t = W_B q is the exact integer product (numpy int64 matmul) for random and extreme codes, and
    negating q negates t."""
    g = np.random.default_rng(12)
    for d_in in (32, 256, 4096):
        lb = g.integers(-127, 128, (16, d_in), dtype=np.int8)
        L = oracle.Linear(np.zeros((4, d_in // 32), np.uint32), np.ones(4, np.float32), lb,
                          np.ones(16, np.float32), np.zeros((4, 16), np.int8), np.ones(4, np.float32))
        for q in (g.integers(-127, 128, d_in, dtype=np.int8), np.full(d_in, 127, np.int8),
                  np.full(d_in, -127, np.int8)):
            t, _ = oracle.lora_down(L, q, 1.0)
            expect = lb.astype(np.int64) @ q.astype(np.int64)
            assert np.array_equal(t.astype(np.int64), expect)
            tn, _ = oracle.lora_down(L, (-q.astype(np.int16)).astype(np.int8), 1.0)
            assert np.array_equal(tn, -t)


def test_lora_epilogue_real_number_formula(tiny):
    """y = acc*s*sW + sA * W_A @ ((W_B @ q) * sB * s) to fp32 accuracy: catches a transposed W_A or W_B,
    a missing scale or a wrong-sign term."""
    d = tiny["linear"]
    L = oracle.Linear.from_dict(d)
    out = oracle.linear_decode(L, tiny["x"])
    s = float(out["xscale"][0])
    t = d["lora_b"].astype(np.int64) @ out["xq"][0].astype(np.int64)
    assert np.array_equal(out["t"][0].astype(np.int64), t)
    tf = t * d["lora_b_scale"].astype(np.float64) * s
    y = (out["acc"][0] * s * d["w_scale"].astype(np.float64)
         + d["lora_a_scale"].astype(np.float64) * (d["lora_a"].astype(np.float64) @ tf))
    assert np.allclose(out["y"][0], y, rtol=1e-6, atol=1e-7)


def test_lora_power_of_two_input_scaling(tiny):
    """Scaling x by 2^k leaves the codes and t unchanged and scales tf and y by exactly 2^k (the LoRA
    intermediate carries the input's quantizer scale s)."""
    L = oracle.Linear.from_dict(tiny["linear"])
    a = oracle.linear_decode(L, tiny["x"])
    for k in (-3, 5):
        b = oracle.linear_decode(L, tiny["x"] * np.float32(2.0 ** k))
        assert np.array_equal(a["xq"], b["xq"]) and np.array_equal(a["t"], b["t"])
        assert np.array_equal(b["xscale"], (a["xscale"] * np.float32(2.0 ** k)).astype(np.float32))
        _, tfa = oracle.lora_down(L, a["xq"][0], float(a["xscale"][0]))
        _, tfb = oracle.lora_down(L, b["xq"][0], float(b["xscale"][0]))
        assert np.array_equal(tfb, (tfa * np.float32(2.0 ** k)).astype(np.float32))
        assert np.array_equal(b["y"], (a["y"] * np.float32(2.0 ** k)).astype(np.float32))


# ------------------------------------------------------------------------------------------- conv

def silu(v):
    return v * expit(v)


def test_conv_stepped_equals_textbook_convolution():
    g = np.random.default_rng(9)
    T, Cn = 11, 8
    x = g.standard_normal((T, Cn)).astype(np.float32)
    w = g.normal(0, 0.5, (Cn, 4)).astype(np.float32)
    b = g.normal(0, 0.1, Cn).astype(np.float32)
    state = np.zeros((1, Cn, 3), np.float32)
    outs = np.stack([oracle.conv_step(state, w, b, x[t:t + 1])[0] for t in range(T)])
    for c in range(Cn):
        # causal conv: out[t] = sum_k w[c,k] * x[t-3+k]  (numpy full convolution with reversed taps)
        pre = np.convolve(x[:, c].astype(np.float64), w[c, ::-1].astype(np.float64))[:T] + b[c]
        assert np.allclose(outs[:, c], silu(pre), rtol=1e-6, atol=1e-7)
    assert np.array_equal(state[0], x[-3:].T)


def test_conv_impulse_reproduces_taps():
    Cn = 5
    w = np.arange(20, dtype=np.float32).reshape(Cn, 4) / 10 - 1
    b = np.zeros(Cn, np.float32)
    state = np.zeros((1, Cn, 3), np.float32)
    for t in range(6):
        x = np.ones((1, Cn), np.float32) if t == 0 else np.zeros((1, Cn), np.float32)
        out = oracle.conv_step(state, w, b, x)[0]
        expect = silu(w[:, 3 - t].astype(np.float64)) if t < 4 else np.zeros(Cn)
        assert np.allclose(out, expect, rtol=1e-6, atol=1e-8)


# -------------------------------------------------------------------------------------------- SSM

def softplus(v):
    return np.logaddexp(0.0, v)


def ssd_dual_form(x, dt_raw, A_log, dt_bias, D, Bm, Cm, G):
    """Quadratic (attention-like) form of the selective SSM over a whole sequence, fp64:
    y_t = sum_{s<=t} (prod_{k=s+1..t} a_k) * dt_s * (C_t . B_s) * x_s + D * x_t."""
    T, H, P = x.shape
    N = Bm.shape[-1]
    dt = softplus(dt_raw.astype(np.float64) + dt_bias.astype(np.float64))  # [T,H]
    a = np.exp(dt * -np.exp(A_log.astype(np.float64)))                     # [T,H]
    y = np.zeros((T, H, P))
    for h in range(H):
        g = h // (H // G)
        for t in range(T):
            for s in range(t + 1):
                decay = np.prod(a[s + 1:t + 1, h])
                cb = float(Cm[t, g].astype(np.float64) @ Bm[s, g].astype(np.float64))
                y[t, h] += decay * dt[s, h] * cb * x[s, h].astype(np.float64)
            y[t, h] += D[h] * x[t, h]
    return y


@pytest.mark.parametrize("H,G", [(2, 1), (4, 2)])
def test_ssm_stepped_equals_dual_form(H, G):
    g = np.random.default_rng(13 + H)
    T, P, N = 12, 3, 5
    x = g.standard_normal((T, H, P)).astype(np.float32)
    dt_raw = g.standard_normal((T, H)).astype(np.float32)
    A_log = g.uniform(0, 1.5, H).astype(np.float32)
    dt_bias = g.uniform(-2, 0, H).astype(np.float32)
    D = g.uniform(0.5, 1.5, H).astype(np.float32)
    Bm = g.standard_normal((T, G, N)).astype(np.float32)
    Cm = g.standard_normal((T, G, N)).astype(np.float32)
    state = np.zeros((1, H, P, N), np.float32)
    ys = np.stack([oracle.ssm_step(state, x[t].reshape(1, -1), dt_raw[t:t + 1], A_log, dt_bias, D,
                                   Bm[t:t + 1], Cm[t:t + 1]).reshape(H, P) for t in range(T)])
    ref = ssd_dual_form(x, dt_raw, A_log, dt_bias, D, Bm, Cm, G)
    assert np.allclose(ys, ref, rtol=1e-5, atol=1e-5)


def test_ssm_constant_input_geometric_closed_form():
    H, P, N, T = 1, 2, 3, 9
    x = np.array([[0.7, -1.3]], np.float32)
    Bv = np.array([[[0.5, -0.25, 1.0]]], np.float32)
    Cv = np.array([[[1.5, 2.0, -0.5]]], np.float32)
    dt_raw = np.array([[0.3]], np.float32)
    A_log = np.array([0.2], np.float32)
    dt_bias = np.array([-1.0], np.float32)
    D = np.array([0.9], np.float32)
    state = np.zeros((1, H, P, N), np.float32)
    for _ in range(T):
        y = oracle.ssm_step(state, x, dt_raw, A_log, dt_bias, D, Bv, Cv)
    dt = softplus(-0.7)
    a = np.exp(dt * -np.exp(0.2))
    S = dt * x[0][:, None].astype(np.float64) * Bv[0, 0][None, :] * (1 - a ** T) / (1 - a)
    assert np.allclose(state[0, 0], S, rtol=1e-5)
    assert np.allclose(y[0], S @ Cv[0, 0] + 0.9 * x[0], rtol=1e-5)


def test_ssm_dt_to_zero_freezes_state():
    g = np.random.default_rng(21)
    H, P, N = 2, 4, 8
    state = g.standard_normal((1, H, P, N)).astype(np.float32)
    before = state.copy()
    x = g.standard_normal((1, H * P)).astype(np.float32)
    Bv = g.standard_normal((1, 1, N)).astype(np.float32)
    Cv = g.standard_normal((1, 1, N)).astype(np.float32)
    D = np.array([0.5, 1.25], np.float32)
    y = oracle.ssm_step(state, x, np.zeros((1, H), np.float32), np.zeros(H, np.float32),
                        np.full(H, -60.0, np.float32), D, Bv, Cv)
    assert np.array_equal(state, before)
    ref = before[0] @ Cv[0, 0].astype(np.float64) + (np.repeat(D, P) * x[0]).reshape(H, P)
    assert np.allclose(y[0].reshape(H, P), ref, rtol=1e-6, atol=1e-6)


def test_ssm_dA_to_zero_is_memoryless():
    g = np.random.default_rng(22)
    H, P, N = 2, 3, 4
    state = g.standard_normal((1, H, P, N)).astype(np.float32) * 100
    x = g.standard_normal((1, H * P)).astype(np.float32)
    Bv = g.standard_normal((1, 1, N)).astype(np.float32)
    Cv = g.standard_normal((1, 1, N)).astype(np.float32)
    D = np.zeros(H, np.float32)
    y = oracle.ssm_step(state, x, np.zeros((1, H), np.float32), np.full(H, 6.0, np.float32),
                        np.full(H, 2.0, np.float32), D, Bv, Cv)
    dt = softplus(2.0)
    S = dt * x[0].reshape(H, P, 1).astype(np.float64) * Bv[0, 0].astype(np.float64)
    assert np.allclose(state[0], S, rtol=1e-6)
    assert np.allclose(y[0].reshape(H, P), S @ Cv[0, 0].astype(np.float64), rtol=1e-5, atol=1e-6)


# --------------------------------------------------------------------------------- norms and gate

def _f32_correctly_rounded(d: Decimal):
    """The fp32 value nearest the exact decimal d, and the relative distance of d from the nearest fp32
    rounding boundary (a midpoint between two fp32 neighbours)."""
    f = np.float32(float(d))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    best = min(cands, key=lambda c: abs(Decimal(float(c)) - d))
    lo, hi = np.nextafter(best, np.float32(-np.inf)), np.nextafter(best, np.float32(np.inf))
    mids = [(Decimal(float(best)) + Decimal(float(lo))) / 2, (Decimal(float(best)) + Decimal(float(hi))) / 2]
    margin = min(abs(d - m) for m in mids) / abs(d)
    return best, margin


def test_rmsnorm_factor_is_the_correctly_rounded_real_number():
    """r = 1/sqrt(mean(h^2) + eps), evaluated exactly in 60-digit decimal arithmetic from the fp32 inputs
    and rounded once to fp32.  Catches a wrong epsilon, n - 1 for n, a missing square root, or the sum
    of |h| instead of h^2.  Rows near a rounding boundary (relative margin below 2^-45, where the fp64
    evaluation may legitimately round the other way) are skipped and counted."""
    getcontext().prec = 60
    g = np.random.default_rng(33)
    rows = [g.standard_normal(256) * 3, g.standard_normal(2048), g.standard_normal(64) * 1e-3,
            np.full(32, 2.0 ** -9), g.uniform(-1, 1, 4096) * 50, np.zeros(128)]
    checked = 0
    for h in rows:
        h = h.astype(np.float32)
        w = np.ones(h.size, np.float32)
        _, _, _, r = oracle.rmsnorm_quantize(h[None], w)
        ss = sum(Decimal(float(v)) ** 2 for v in h)
        exact = 1 / (ss / h.size + Decimal(1e-5)).sqrt()
        want, margin = _f32_correctly_rounded(exact)
        if margin < Decimal(2) ** -45:
            continue
        assert r[0] == want, (h.size, r[0], want)
        checked += 1
    assert checked >= 5


def test_rmsnorm_normalized_row_and_codes():
    """u = h w / sqrt(mean(h^2) + eps) to fp32 accuracy (two fp32 roundings and r's), and the codes and
    scale are exactly those of the pinned quantizer applied to u: catches a missing weight, a quantizer
    that runs before the norm, or the RMS factor applied to the scale instead of the values."""
    g = np.random.default_rng(31)
    h = (g.standard_normal((8, 2048)) * 3).astype(np.float32)
    w = g.uniform(0.5, 1.5, 2048).astype(np.float32)
    q, s, u, r = oracle.rmsnorm_quantize(h, w)
    h64 = h.astype(np.float64)
    exact = h64 / np.sqrt(np.mean(h64 ** 2, axis=1, keepdims=True) + 1e-5) * w
    assert np.all(np.abs(u - exact) <= 4 * 2.0 ** -24 * np.abs(exact))
    q2, s2 = oracle.quantize(u)
    assert np.array_equal(q, q2) and np.array_equal(s, s2)


def test_rmsnorm_constant_row_closed_form():
    """h = c everywhere: mean(h^2) = c^2, so u_i = w_i sign(c) / sqrt(1 + eps/c^2), and the largest
    weight's code is 127 sign(c)."""
    g = np.random.default_rng(30)
    w = g.uniform(0.5, 1.5, 256).astype(np.float32)
    for c in (-3.0, 0.25, 40.0, 1e-3):
        q, s, u, r = oracle.rmsnorm_quantize(np.full((1, 256), c, np.float32), w)
        want = np.sign(c) * w.astype(np.float64) / np.sqrt(1 + 1e-5 / c ** 2)
        assert np.all(np.abs(u[0] - want) <= 3 * 2.0 ** -24 * np.abs(want))
        assert q[0, np.argmax(w)] == 127 * np.sign(c)
        assert np.all(np.abs(s[0] * q[0] - want) <= s[0] / 2 * 1.0001)


def test_rmsnorm_zero_weight_and_zero_row():
    """A zero weight zeroes its code (the weight multiplies before the quantizer); an all-zero row gives
    r = fl32(1/sqrt(eps)), u = 0, s = 0 and all codes 0."""
    g = np.random.default_rng(34)
    h = g.standard_normal((1, 64)).astype(np.float32)
    w = np.ones(64, np.float32)
    w[::2] = 0
    q, s, u, _ = oracle.rmsnorm_quantize(h, w)
    assert np.all(q[0, ::2] == 0) and np.all(u[0, ::2] == 0)
    assert np.any(q[0, 1::2] != 0)
    q, s, u, r = oracle.rmsnorm_quantize(np.zeros((1, 64), np.float32), np.ones(64, np.float32))
    assert r[0] == np.float32(1 / np.sqrt(1e-5))
    assert np.all(u == 0) and np.all(q == 0) and s[0] == 0


def test_gate_silu_against_logistic():
    g = np.random.default_rng(32)
    y = g.standard_normal(1000).astype(np.float32)
    z = (g.standard_normal(1000) * 4).astype(np.float32)
    out = oracle.gate(y, z)
    assert np.allclose(out, y * (z * expit(z.astype(np.float64))), rtol=1e-6, atol=1e-9)


# ------------------------------------------------------------------------------------ layer wiring

SMALL = dict(d_model=64, nheads=4, headdim=16, d_state=16, ngroups=1, rank=4)


def _oracle_layer(ld):
    lay = dict(ld)
    lay["in_proj"] = oracle.Linear.from_dict(ld["in_proj"])
    lay["out_proj"] = oracle.Linear.from_dict(ld["out_proj"])
    return lay


def test_layer_zero_out_proj_keeps_residual():
    m = inputs.decode_model(seed=40, n_layers=1, n_tokens=2, **SMALL)
    ld = m["layers"][0]
    ld["out_proj"]["w_scale"][:] = 0
    ld["out_proj"]["lora_a_scale"][:] = 0
    lay = _oracle_layer(ld)
    conv, ssm = inputs.zero_states(1, 1, 4, 16, 16, 1)
    h = m["emb"][0].copy()
    h0 = h.copy()
    taps = oracle.layer_decode(lay, h, conv[0], ssm[0], taps=True)
    assert np.array_equal(h, h0)
    assert np.any(ssm[0] != 0) and np.any(taps["y"] != 0)


def _hand_layer(P, h, conv, S):
    """One decode step of a Mamba-2 layer with one head, d_state 1 and ngroups 1, written out from the
    definitions in float64 numpy (no oracle call): RMSNorm, per-token absmax int8 codes, the +-1
    scaffold and the int8 LoRA on the codes, the split z | x | B | C | dt, the width-4 causal conv with
    SiLU, softplus dt, the scalar-state recurrence S <- exp(dt A) S + dt x B, y = S C + D x, the gate
    y SiLU(z), the gated RMSNorm, out_proj and the residual.  conv [C][3] and S [E] are updated in
    place; returns the new h and the codes' distances from a rounding tie (to check the margin)."""
    silu = lambda v: v / (1 + np.exp(-v))

    def norm_codes(v, w):
        u = v / np.sqrt(np.mean(v * v) + 1e-5) * w
        s = np.abs(u).max() / 127
        t = u / s
        return np.rint(t), s, np.abs(np.abs(t - np.floor(t)) - 0.5)

    def linear(L, q, s):
        sign = unpack_pm1(L["bits"]).astype(np.float64)
        t = L["lora_b"].astype(np.float64) @ q
        tf = t * L["lora_b_scale"] * s
        return (sign @ q) * s * L["w_scale"] + L["lora_a_scale"] * (L["lora_a"].astype(np.float64) @ tf)

    E = P["gnorm_w"].size
    q, s, gap1 = norm_codes(h, P["norm_w"])
    zx = linear(P["in_proj"], q, s)
    z, xbc, dt_raw = zx[:E], zx[E:2 * E + 2], zx[2 * E + 2]
    w = P["conv_w"].astype(np.float64)
    pre = P["conv_b"] + w[:, 0] * conv[:, 0] + w[:, 1] * conv[:, 1] + w[:, 2] * conv[:, 2] + w[:, 3] * xbc
    conv[:, :2] = conv[:, 1:]
    conv[:, 2] = xbc
    xc = silu(pre)
    x, Bv, Cv = xc[:E], xc[E], xc[E + 1]
    dt = np.log1p(np.exp(dt_raw + P["dt_bias"][0]))
    a = np.exp(dt * -np.exp(float(P["A_log"][0])))
    S[:] = a * S + dt * x * Bv
    y = S * Cv + P["D"][0] * x
    g = y * silu(z)
    q2, s2, gap2 = norm_codes(g, P["gnorm_w"])
    return h + linear(P["out_proj"], q2, s2), min(gap1.min(), gap2.min())


WIRE = dict(d_model=32, nheads=1, headdim=32, d_state=1, ngroups=1, rank=3)


def test_layer_wiring_against_hand_computed_closed_form():
    """The oracle's layer decode over four tokens equals the whole step written out in float64 from the
    definitions (one head of 32 channels, d_state 1, rank 3): catches a wrong split order, the gate after
    the norm, a missing D skip or residual, a conv state shifted the wrong way, or dt from the wrong row.
    The test's own codes stay at least 1e-3 away from a rounding tie, so both sides pick the same codes
    and agree to fp32 rounding."""
    m = inputs.decode_model(seed=43, n_layers=1, n_tokens=4, **WIRE)
    P = m["layers"][0]
    lay = _oracle_layer(P)
    conv, ssm = inputs.zero_states(1, 1, 1, 32, 1, 1)
    conv_h = np.zeros((34, 3))
    S_h = np.zeros(32)
    for t in range(4):
        h = m["emb"][t].copy()
        oracle.layer_decode(lay, h, conv[0], ssm[0])
        want, gap = _hand_layer(P, m["emb"][t][0].astype(np.float64), conv_h, S_h)
        assert gap > 1e-3
        assert np.allclose(h[0], want, rtol=2e-6, atol=1e-6), t
        assert np.allclose(ssm[0, 0, 0, :, 0], S_h, rtol=2e-6, atol=1e-7)
        assert np.allclose(conv[0, 0], conv_h, rtol=1e-6, atol=1e-7)


def test_layer_prefill_against_hand_computed_closed_form():
    """A 5-token prompt through two such layers: the oracle's layer-major prefill equals the hand-written
    step applied token by token through both layers, and so does the token-major decode."""
    m = inputs.decode_model(seed=44, n_layers=2, n_tokens=5, **WIRE)
    layers = [_oracle_layer(ld) for ld in m["layers"]]
    conv, ssm = inputs.zero_states(1, 2, 1, 32, 1, 1)
    prompt = np.ascontiguousarray(m["emb"][:, 0, :])
    h = oracle.layer_prefill(layers, prompt.copy(), conv, ssm)
    conv_h = [np.zeros((34, 3)) for _ in range(2)]
    S_h = [np.zeros(32) for _ in range(2)]
    for t in range(5):
        v = prompt[t].astype(np.float64)
        for l in range(2):
            v, gap = _hand_layer(m["layers"][l], v, conv_h[l], S_h[l])
            assert gap > 1e-3
        assert np.allclose(h[t], v, rtol=5e-6, atol=2e-6), t
    for l in range(2):
        assert np.allclose(ssm[l, 0, 0, :, 0], S_h[l], rtol=5e-6, atol=1e-7)


# ------------------------------------------------------------------------------------------ LM head

def test_lm_head_brute_force():
    g = np.random.default_rng(50)
    W = g.integers(-127, 128, (300, 128), dtype=np.int8)
    sr = g.uniform(1e-4, 1e-3, 300).astype(np.float32)
    x = g.standard_normal(128).astype(np.float32)
    logits, acc = oracle.lm_head(W, sr, x)
    q, s = oracle.quantize(x[None])
    assert np.array_equal(acc, W.astype(np.int64) @ q[0].astype(np.int64))
    assert np.allclose(logits, acc.astype(np.float64) * float(s[0]) * sr, rtol=2e-7)
    rows = np.array([299, 0, 17])
    l2, a2 = oracle.lm_head(W, sr, x, rows)
    assert np.array_equal(a2, acc[rows]) and np.array_equal(l2, logits[rows])


def test_prefill_layer_major_equals_token_major():
    """A prompt through the stack layer after layer (each layer over the whole prompt) equals feeding the
    tokens one at a time through every layer: the same recurrence, states carried per layer."""
    m = inputs.decode_model(seed=42, n_layers=3, n_tokens=5, **SMALL)
    layers = [_oracle_layer(ld) for ld in m["layers"]]
    conv_a, ssm_a = inputs.zero_states(1, 3, 4, 16, 16, 1)
    conv_b, ssm_b = conv_a.copy(), ssm_a.copy()
    prompt = np.ascontiguousarray(m["emb"][:, 0, :])
    h_a = oracle.layer_prefill(layers, prompt.copy(), conv_a, ssm_a)
    for t in range(5):
        h_t = np.ascontiguousarray(m["emb"][t])
        for l in range(3):
            oracle.layer_decode(layers[l], h_t, conv_b[l], ssm_b[l])
        assert np.array_equal(h_a[t], h_t[0])
    assert np.array_equal(ssm_a, ssm_b) and np.array_equal(conv_a, conv_b)


# --------------------------------------------------------------------- embedding, final head, greedy

def test_embed_power_of_two_scales_are_exact():
    """Row scales 2^-k make every dequantized value exact: catches a wrong row, a dropped scale or a
    transposed matrix."""
    g = np.random.default_rng(51)
    W = g.integers(-127, 128, (40, 96), dtype=np.int8)
    k = g.integers(4, 16, 40)
    sr = np.ldexp(1.0, -k).astype(np.float32)
    for tok in (0, 17, 39):
        e = oracle.embed(W, sr, tok)
        assert np.array_equal(e.astype(np.float64), W[tok].astype(np.float64) * 2.0 ** -int(k[tok]))


def test_embed_matches_ieee_fp32_multiply_and_rejects_bad_tokens():
    g = np.random.default_rng(52)
    W = g.integers(-127, 128, (50, 64), dtype=np.int8)
    sr = g.uniform(1e-4, 1e-3, 50).astype(np.float32)
    for tok in (0, 1, 49):
        assert np.array_equal(oracle.embed(W, sr, tok), W[tok].astype(np.float32) * sr[tok])
    for bad in (-1, 50):
        with pytest.raises(IndexError):
            oracle.embed(W, sr, bad)


def test_final_head_constant_row_closed_form():
    """h = c (all equal), unit norm weight: every code is 127 sign(c), so
    logits[v] = sign(c) * sum_i W[v,i] * s_row[v] / sqrt(1 + eps / c^2).  Catches a missing RMS factor,
    a wrong epsilon, a sign error or the norm weight left out."""
    g = np.random.default_rng(53)
    W = g.integers(-127, 128, (64, 128), dtype=np.int8)
    sr = g.uniform(1e-4, 1e-3, 64).astype(np.float32)
    ones = np.ones(128, np.float32)
    for c in (-2.5, 0.01, 7.0):
        logits, acc = oracle.final_head(W, sr, np.full(128, c, np.float32), ones)
        rowsum = W.astype(np.int64).sum(axis=1)
        assert np.array_equal(acc, 127 * int(np.sign(c)) * rowsum)
        want = np.sign(c) * rowsum * sr.astype(np.float64) / np.sqrt(1 + 1e-5 / c ** 2)
        assert np.allclose(logits, want, rtol=1e-6, atol=0)


def test_final_head_norm_weight_enters_the_codes():
    """A norm weight that is zero on half the inputs zeroes their codes (the weight multiplies before
    the quantizer, not after)."""
    g = np.random.default_rng(54)
    W = g.integers(-127, 128, (32, 64), dtype=np.int8)
    sr = g.uniform(1e-4, 1e-3, 32).astype(np.float32)
    h = g.standard_normal(64).astype(np.float32)
    w = np.ones(64, np.float32)
    w[32:] = 0
    _, acc = oracle.final_head(W, sr, h, w)
    _, acc_half = oracle.final_head(W[:, :32].copy(), sr, h[:32].copy(), w[:32].copy())
    assert np.array_equal(acc, acc_half)


def test_final_head_is_the_lm_head_of_the_normalized_row():
    """The final head equals the plain LM head applied to the pinned normalized row u (same integer sums,
    same logits), and its integer sums are the brute-force product with the codes of u."""
    g = np.random.default_rng(55)
    V, d = 500, 256
    W = g.integers(-127, 128, (V, d), dtype=np.int8)
    sr = g.uniform(1e-4, 1e-3, V).astype(np.float32)
    h = (g.standard_normal(d) * 2).astype(np.float32)
    w = g.uniform(0.5, 1.5, d).astype(np.float32)
    logits, acc = oracle.final_head(W, sr, h, w)
    q, s, u, _ = oracle.rmsnorm_quantize(h[None], w)
    assert np.array_equal(acc, W.astype(np.int64) @ q[0].astype(np.int64))
    l2, a2 = oracle.lm_head(W, sr, u[0])
    assert np.array_equal(a2, acc) and np.array_equal(l2, logits)
    # the plain head is the final head without a norm
    l3, a3 = oracle.final_head(W, sr, h)
    l4, a4 = oracle.lm_head(W, sr, h)
    assert np.array_equal(l3, l4) and np.array_equal(a3, a4)
    rows = np.array([499, 3, 250])
    l5, a5 = oracle.final_head(W, sr, h, w, rows)
    assert np.array_equal(l5, logits[rows]) and np.array_equal(a5, acc[rows])


def test_greedy_takes_first_index_on_ties():
    assert oracle.greedy(np.array([0.5, 2.0, -1.0, 2.0], np.float32)) == 1
    assert oracle.greedy(np.array([-3.0, -3.0], np.float32)) == 0


def test_generate_with_identity_layers_follows_the_head():
    """With every out_proj scaled to zero the layers leave the residual stream unchanged, so each
    step's hidden state is the embedding itself and the next token is the greedy choice of the head
    on it, computed here by brute force from the pinned quantizer codes."""
    dims = dict(SMALL)
    m = inputs.generation_model(seed=56, n_layers=2, vocab=300, **dims)
    for ld in m["layers"]:
        ld["out_proj"]["w_scale"][:] = 0
        ld["out_proj"]["lora_a_scale"][:] = 0
    layers = [_oracle_layer(ld) for ld in m["layers"]]
    conv, ssm = inputs.zero_states(1, 2, 4, 16, 16, 1)
    W, sr, fw = m["emb_w"], m["emb_s"], m["final_norm_w"]
    toks, hid, _ = oracle.generate(layers, W, sr, fw, m["first_token"], 5, conv, ssm)
    assert toks[0] == m["first_token"] and len(toks) == 6
    assert np.any(ssm != 0)
    for t in range(5):
        e = W[toks[t]].astype(np.float32) * sr[toks[t]]
        assert np.array_equal(hid[t], e)
        q, s, _, _ = oracle.rmsnorm_quantize(e[None], fw)
        acc = W.astype(np.int64) @ q[0].astype(np.int64)
        logits = (acc.astype(np.float64) * float(s[0]) * sr.astype(np.float64)).astype(np.float32)
        assert toks[t + 1] == int(np.argmax(logits))


# ------------------------------------------------------------------------------------- shape pins

def _golden(name):
    vals = {}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split()
                vals[k] = float(v)
    return vals


def test_model_size_and_composition_pin():
    """The 1.3B shapes reproduce the printed sizes (tests/golden/model_size.txt): the split of the 278 MB
    model (scaffold, embedding/LM head, LoRA, other), the 2.7 GB FP16 teacher (every weight in fp16) and
    its 9.7x reduction, and 1 bit per scaffold weight (8x less than int8)."""
    g = _golden("model_size.txt")
    total = g["compressed_model_mb"] * 1e6
    L, Dm, E, Nst, H = inputs.N_LAYERS, inputs.D_MODEL, inputs.D_INNER, inputs.D_STATE, inputs.N_HEADS
    d_ip = inputs.D_IN_PROJ
    assert d_ip == 2 * E + 2 * Nst + H == 8512
    scaffold_weights = L * (d_ip * Dm + Dm * E)
    scaffold_bytes = scaffold_weights / 8
    lm_bytes = inputs.VOCAB * Dm
    lora_bytes = L * (inputs.RANK * Dm + d_ip * inputs.RANK + inputs.RANK * E + Dm * inputs.RANK)
    assert round(100 * scaffold_bytes / total) == g["share_scaffold_pct"]
    assert round(100 * lm_bytes / total) == g["share_embedding_lm_head_pct"]
    assert g["share_lora_pct"] <= 100 * lora_bytes / total < g["share_lora_pct"] + 1
    other = total - scaffold_bytes - lm_bytes - lora_bytes
    assert abs(100 * other / total - g["share_other_pct"]) < 1
    assert scaffold_weights / scaffold_bytes == g["scaffold_memory_reduction_x"]
    # the FP16 teacher: the scaffold's weights and the embedding/LM-head matrix at 2 bytes each
    teacher_bytes = 2 * (scaffold_weights + inputs.VOCAB * Dm)
    assert round(teacher_bytes / 1e9, 1) == g["fp16_teacher_gb"]
    assert round(g["fp16_teacher_gb"] * 1e9 / total, 1) == g["reduction_x"]
