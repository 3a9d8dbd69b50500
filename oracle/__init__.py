"""DF-SSM CPU oracle — TEST INFRASTRUCTURE ONLY.

A numpy-facing wrapper over the plain C++ oracle in ``dfssm_oracle.cpp``.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import this package; the
product path (``bit_quantized_mamba_b200``) never does, and this package imports nothing from it.

Every function here is argument marshalling around one C function whose header comment cites the
passage it follows and says what pins it.  All arrays are numpy, C-contiguous, host memory.
"""
from __future__ import annotations

import ctypes as C
import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(_build.build())
        _declare(_lib)
    return _lib


_P = C.c_void_p
_I = C.c_int


def _declare(L):
    L.oracle_abi_version.restype = _I
    L.oracle_set_threads.argtypes = [_I]
    L.oracle_set_threads.restype = _I
    L.oracle_sign.argtypes = [_P, _I, _I, _I]
    L.oracle_sign.restype = _I
    L.oracle_quantize.argtypes = [_P, _I, _I, _P, _P]
    L.oracle_linear_decode.argtypes = [_I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P]
    L.oracle_lora_down.argtypes = [_I, _I, _P, _P, _P, C.c_float, _P, _P]
    L.oracle_linear_core.argtypes = [_I, _I, _I, _P, _P, _P, _P, _P, C.c_float, _P, _P, _P]
    L.oracle_linear_rows.argtypes = [_I, _I, _I, _P, _P, _P, _P, _P, C.c_float, _P, _P, _I, _P, _P]
    L.oracle_conv_step.argtypes = [_P, _P, _P, _P, _P, _I, _I]
    L.oracle_ssm_step.argtypes = [_P] * 9 + [_I] * 5
    L.oracle_rmsnorm_quantize.argtypes = [_P, _P, _I, _I, _P, _P, _P, _P]
    L.oracle_gate.argtypes = [_P, _P, _P, _I]
    L.oracle_layer_decode.argtypes = [_I] * 7 + [_P] * 12 + [_P] * 7 + [_P] * 3 + [_P, _P]
    L.oracle_lm_head.argtypes = [_P, _P, _I, _I, _P, _P, _I, _P, _P]
    L.oracle_embed.argtypes = [_P, _P, _I, _I, _I, _P]
    L.oracle_embed.restype = _I
    L.oracle_final_head.argtypes = [_P, _P, _I, _I, _P, _P, _P, _I, _P, _P]
    L.oracle_field_encode.argtypes = [_P, _I, _I, _P, _P]
    L.oracle_field_decode.argtypes = [_P, _P, _I, _I, _P]


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def set_threads(n: int) -> int:
    """Host threads of the oracle's OpenMP loops (for the CPU-baseline timing); returns the previous
    maximum.  n <= 0 leaves it unchanged."""
    return lib().oracle_set_threads(int(n))


def sign(bits: np.ndarray, d_in: int, o: int, i: int) -> int:
    bits = _c(bits, np.uint32)
    return lib().oracle_sign(_p(bits), d_in, o, i)


def quantize(x: np.ndarray):
    """Per-token absmax int8 quantization of each row of x -> (q int8, s fp32[rows])."""
    x = _c(np.atleast_2d(x), np.float32)
    B, n = x.shape
    q = np.zeros((B, n), np.int8)
    s = np.zeros(B, np.float32)
    lib().oracle_quantize(_p(x), B, n, _p(q), _p(s))
    return q, s


class Linear:
    """Host copy of one scaffold+LoRA linear: bits [d_out][d_in/32] u32 (LSB-first), w_scale [d_out],
    lora_b [rank][d_in] i8, lora_b_scale [rank], lora_a [d_out][rank] i8, lora_a_scale [d_out]."""

    def __init__(self, bits, w_scale, lora_b, lora_b_scale, lora_a, lora_a_scale):
        self.bits = _c(bits, np.uint32)
        self.d_out = self.bits.shape[0]
        self.d_in = self.bits.shape[1] * 32
        self.w_scale = _c(w_scale, np.float32)
        self.lora_b = _c(lora_b, np.int8).reshape(-1, self.d_in)
        self.rank = self.lora_b.shape[0]
        self.lora_b_scale = _c(lora_b_scale, np.float32).reshape(self.rank)
        self.lora_a = _c(lora_a, np.int8).reshape(self.d_out, self.rank)
        self.lora_a_scale = _c(lora_a_scale, np.float32).reshape(self.d_out)

    @classmethod
    def from_dict(cls, d):
        return cls(d["bits"], d["w_scale"], d["lora_b"], d["lora_b_scale"], d["lora_a"],
                   d["lora_a_scale"])

    def _args(self):
        rb = self.lora_b if self.rank else np.zeros((1, self.d_in), np.int8)
        ra = self.lora_a if self.rank else np.zeros((self.d_out, 1), np.int8)
        rbs = self.lora_b_scale if self.rank else np.zeros(1, np.float32)
        self._keep = (rb, ra, rbs)
        return (self.d_out, self.d_in, self.rank, _p(self.bits), _p(self.w_scale), _p(rb), _p(rbs),
                _p(ra), _p(self.lora_a_scale))


def linear_decode(L: Linear, x: np.ndarray):
    """Quantize each row of x and apply the linear. Returns dict(y, acc, t, xq, xscale)."""
    x = _c(np.atleast_2d(x), np.float32)
    B = x.shape[0]
    assert x.shape[1] == L.d_in
    y = np.zeros((B, L.d_out), np.float32)
    acc = np.zeros((B, L.d_out), np.int32)
    t = np.zeros((B, max(L.rank, 1)), np.int32)
    xq = np.zeros((B, L.d_in), np.int8)
    xs = np.zeros(B, np.float32)
    lib().oracle_linear_decode(*L._args(), _p(x), B, _p(y), _p(acc), _p(t), _p(xq), _p(xs))
    return dict(y=y, acc=acc, t=t.reshape(-1)[:B * L.rank].reshape(B, L.rank), xq=xq, xscale=xs)


def lora_down(L: Linear, q: np.ndarray, s: float):
    """LoRA down-projection of one row of codes q (int8) with scale s:
    t[r] = sum_i W_B[r,i] q_i (int32) and tf[r] = fl32(t[r] * sB[r] * s). Returns (t, tf)."""
    q = _c(q, np.int8).reshape(L.d_in)
    t = np.zeros(max(L.rank, 1), np.int32)
    tf = np.zeros(max(L.rank, 1), np.float32)
    a = L._args()
    lib().oracle_lora_down(L.d_in, L.rank, a[5], a[6], _p(q), C.c_float(float(s)), _p(t), _p(tf))
    return t[:L.rank], tf[:L.rank]


def linear_core(L: Linear, q: np.ndarray, s: float, tf: np.ndarray):
    """The linear on one pre-quantized row q (int8) with scale s and LoRA intermediate tf.
    Returns (y, acc)."""
    q = _c(q, np.int8).reshape(L.d_in)
    tf = _c(tf, np.float32).reshape(-1) if L.rank else np.zeros(1, np.float32)
    y = np.zeros(L.d_out, np.float32)
    acc = np.zeros(L.d_out, np.int32)
    a = L._args()
    lib().oracle_linear_core(L.d_out, L.d_in, L.rank, a[3], a[4], a[7], a[8], _p(q),
                             C.c_float(float(s)), _p(tf), _p(acc), _p(y))
    return y, acc


def linear_rows(L: Linear, q: np.ndarray, s: float, tf: np.ndarray, rows):
    """Only the listed output rows of the linear on pre-quantized q. Returns (y, acc)."""
    q = _c(q, np.int8).reshape(L.d_in)
    tf = _c(tf, np.float32).reshape(-1) if L.rank else np.zeros(1, np.float32)
    rows = _c(rows, np.int32)
    y = np.zeros(len(rows), np.float32)
    acc = np.zeros(len(rows), np.int32)
    a = L._args()
    lib().oracle_linear_rows(L.d_out, L.d_in, L.rank, a[3], a[4], a[7], a[8], _p(q),
                             C.c_float(float(s)), _p(tf), _p(rows), len(rows), _p(acc), _p(y))
    return y, acc


def conv_step(conv_state, w, b, x_in):
    """One shift-register conv step. conv_state [B][C][3] is updated in place; returns x_out [B][C]."""
    assert conv_state.dtype == np.float32 and conv_state.flags["C_CONTIGUOUS"]
    x_in = _c(np.atleast_2d(x_in), np.float32)
    B, Cn = x_in.shape
    w = _c(w, np.float32)
    b = _c(b, np.float32)
    out = np.zeros((B, Cn), np.float32)
    lib().oracle_conv_step(_p(conv_state), _p(w), _p(b), _p(x_in), _p(out), B, Cn)
    return out


def ssm_step(ssm_state, x, dt_raw, A_log, dt_bias, D, Bm, Cm):
    """One SSM step. ssm_state [B][H][P][N] updated in place; x [B][H*P], dt_raw [B][H],
    Bm/Cm [B][G][N]. Returns y [B][H*P]."""
    assert ssm_state.dtype == np.float32 and ssm_state.flags["C_CONTIGUOUS"]
    B, H, P, N = ssm_state.shape
    Bm = _c(Bm, np.float32).reshape(B, -1, N)
    G = Bm.shape[1]
    Cm = _c(Cm, np.float32).reshape(B, G, N)
    x = _c(x, np.float32).reshape(B, H * P)
    dt_raw = _c(dt_raw, np.float32).reshape(B, H)
    A_log, dt_bias, D = (_c(a, np.float32) for a in (A_log, dt_bias, D))
    y = np.zeros((B, H * P), np.float32)
    lib().oracle_ssm_step(_p(ssm_state), _p(x), _p(dt_raw), _p(A_log), _p(dt_bias), _p(D), _p(Bm),
                          _p(Cm), _p(y), B, H, P, N, G)
    return y


def rmsnorm_quantize(h, w):
    """RMSNorm then the per-token quantizer. Returns (q [B][n], s [B], u [B][n], r [B]): u the normalized
    rows fl32(fl32(h r) w), r = fl32(1 / sqrt(mean(h^2) + 1e-5))."""
    h = _c(np.atleast_2d(h), np.float32)
    B, n = h.shape
    w = _c(w, np.float32)
    q = np.zeros((B, n), np.int8)
    s = np.zeros(B, np.float32)
    u = np.zeros((B, n), np.float32)
    r = np.zeros(B, np.float32)
    lib().oracle_rmsnorm_quantize(_p(h), _p(w), B, n, _p(q), _p(s), _p(u), _p(r))
    return q, s, u, r


def gate(y, z):
    y = _c(y, np.float32).ravel()
    z = _c(z, np.float32).ravel()
    g = np.zeros_like(y)
    lib().oracle_gate(_p(y), _p(z), _p(g), y.size)
    return g


def layer_decode(layer: dict, h, conv_state, ssm_state, taps: bool = False):
    """One Mamba-2 layer decode step; h [B][D], conv_state [B][C][3], ssm_state [B][H][P][N] are all
    updated in place.  `layer` holds in_proj / out_proj (Linear), conv_w, conv_b, A_log, dt_bias, D,
    norm_w, gnorm_w.  With taps=True returns dict(zxbcdt, y) of this step."""
    for a in (h, conv_state, ssm_state):
        assert a.dtype == np.float32 and a.flags["C_CONTIGUOUS"]
    B, H, P, N = ssm_state.shape
    Dm = h.shape[1]
    ip, op = layer["in_proj"], layer["out_proj"]
    E = H * P
    Cn = conv_state.shape[1]
    G = (Cn - E) // (2 * N)
    d_ip = ip.d_out
    tz = np.zeros((B, d_ip), np.float32) if taps else None
    ty = np.zeros((B, E), np.float32) if taps else None
    ia = ip._args()[3:]
    oa = op._args()[3:]
    vec = [_c(layer[k], np.float32) for k in ("conv_w", "conv_b", "A_log", "dt_bias", "D", "norm_w",
                                              "gnorm_w")]
    lib().oracle_layer_decode(B, Dm, H, P, N, G, ip.rank, *ia, *oa, *[_p(v) for v in vec], _p(h),
                              _p(conv_state), _p(ssm_state), _p(tz), _p(ty))
    if taps:
        return dict(zxbcdt=tz, y=ty)
    return None


def lm_head(W, s_row, x, rows=None):
    """Int8 LM head on one token x [d]. Returns (logits, acc) for all rows or the listed rows."""
    W = _c(W, np.int8)
    V, d = W.shape
    s_row = _c(s_row, np.float32)
    x = _c(x, np.float32).reshape(d)
    if rows is None:
        n = V
        rp = None
    else:
        rows = _c(rows, np.int32)
        n = len(rows)
        rp = rows
    logits = np.zeros(n, np.float32)
    acc = np.zeros(n, np.int32)
    lib().oracle_lm_head(_p(W), _p(s_row), V, d, _p(x), _p(rp), n, _p(logits), _p(acc))
    return logits, acc


def embed(W, s_row, token: int):
    """Row `token` of the tied int8 embedding, dequantized: fl32(W[token] * s_row[token])."""
    W = _c(W, np.int8)
    V, d = W.shape
    s_row = _c(s_row, np.float32)
    e = np.zeros(d, np.float32)
    if lib().oracle_embed(_p(W), _p(s_row), V, d, int(token), _p(e)) != 0:
        raise IndexError(f"token {token} outside [0, {V})")
    return e


def final_head(W, s_row, h, norm_w=None, rows=None):
    """Final RMSNorm (then the quantizer; None: no norm) + int8 LM head on one token h [d].
    Returns (logits, acc) for all rows or the listed rows."""
    W = _c(W, np.int8)
    V, d = W.shape
    s_row = _c(s_row, np.float32)
    h = _c(h, np.float32).reshape(d)
    nw = None if norm_w is None else _c(norm_w, np.float32).reshape(d)
    rp = None if rows is None else _c(rows, np.int32)
    n = V if rows is None else len(rp)
    logits = np.zeros(n, np.float32)
    acc = np.zeros(n, np.int32)
    lib().oracle_final_head(_p(W), _p(s_row), V, d, _p(h), _p(nw), _p(rp), n, _p(logits), _p(acc))
    return logits, acc


def greedy(logits) -> int:
    """Greedy choice: the index of the largest logit, the smallest such index on ties."""
    return int(np.argmax(np.asarray(logits)))


def generate(layers, W, s_row, final_norm_w, first_token: int, n_tokens: int, conv_states,
             ssm_states, forced_tokens=None):
    """Greedy generation, batch 1: each step embeds the current token, runs every layer (states
    updated in place), applies the final head and takes the greedy choice as the next token.
    forced_tokens (optional, length n_tokens + 1) feeds those tokens instead of the oracle's own
    choices (teacher forcing).  Returns (tokens [n_tokens + 1], hidden [n_tokens][d] after the last
    layer, logits [n_tokens][V])."""
    tokens = [int(first_token)]
    hid, lg = [], []
    for t in range(n_tokens):
        cur = tokens[-1] if forced_tokens is None else int(forced_tokens[t])
        h = embed(W, s_row, cur)[None, :].copy()
        for L, cs, ss in zip(layers, conv_states, ssm_states):
            layer_decode(L, h, cs, ss)
        hid.append(h[0].copy())
        logits, _ = final_head(W, s_row, h[0], final_norm_w)
        lg.append(logits)
        tokens.append(greedy(logits))
    return tokens, np.stack(hid), np.stack(lg)


def layer_prefill(layers, h, conv_states, ssm_states):
    """Prefill of a prompt h [M][d_model] (batch 1) through the layers, layer after layer: each layer
    runs its decode step on tokens 0 .. M-1 in order (the definition of the recurrent model on a
    sequence), h and the per-layer states conv_states[l] [1][C][3], ssm_states[l] [1][H][P][N] are
    updated in place.  Pinned by a hand-written float64 layer applied token by token through two layers
    (one head, d_state 1)."""
    assert h.dtype == np.float32 and h.flags["C_CONTIGUOUS"]
    for L, cs, ss in zip(layers, conv_states, ssm_states):
        for t in range(h.shape[0]):
            layer_decode(L, h[t:t + 1], cs, ss)
    return h


def field_encode(state):
    """Density-field encoding of state rows [..., N] (N % 8 == 0): returns (field uint32 [rows, N/8],
    scale float32 [rows]) with rows = the product of the leading dimensions."""
    S = _c(state, np.float32)
    N = S.shape[-1]
    assert N % 8 == 0 and N > 0
    S = S.reshape(-1, N)
    rows = S.shape[0]
    field = np.zeros((rows, N // 8), np.uint32)
    scale = np.zeros(rows, np.float32)
    lib().oracle_field_encode(_p(S), rows, N, _p(field), _p(scale))
    return field, scale


def field_decode(field, scale, N: int):
    """Popcount readout of density fields [rows, N/8] with their scales [rows] -> state rows [rows, N]."""
    F = _c(field, np.uint32).reshape(-1, N // 8)
    sc = _c(scale, np.float32).reshape(-1)
    rows = F.shape[0]
    assert sc.shape[0] == rows
    out = np.zeros((rows, N), np.float32)
    lib().oracle_field_decode(_p(F), _p(sc), rows, N, _p(out))
    return out
