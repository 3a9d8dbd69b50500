"""Thin ctypes binding of libdfssm (include/dfssm.h): argument marshalling only.

Every compute step runs in the CUDA library; this module only turns torch tensors (device memory,
allocated by the caller) into pointers, picks the current torch stream and raises on a negative status.
There is no fallback: if the library or a CUDA device is missing, the calls raise.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np
import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdfssm.so")

OP_LINEAR_DECODE = 1
OP_LINEAR_PREFILL = 2
OP_LAYER_DECODE = 3
OP_LM_HEAD = 4
OP_HEAD_GREEDY = 5
OP_GENERATE = 6
OP_LAYER_PREFILL = 7
OP_LINEAR_MULTI = 8
OP_EMBED = 9
MAX_RANK = 16
MAX_BATCH = 16
MAX_LAYERS = 64

STATUS = {0: "DFSSM_OK", -1: "DFSSM_EINVAL", -2: "DFSSM_EALIGN", -3: "DFSSM_EUNSUPPORTED",
          -4: "DFSSM_ECUDA", -5: "DFSSM_ETIMEOUT", -6: "DFSSM_EDEVICE", -7: "DFSSM_EWORKSPACE"}


class DfssmError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = f"{fn} returned {STATUS.get(status, status)}"
        if status == -4:
            msg += f" ({lib().dfssm_last_cuda_error().decode()})"
        super().__init__(msg)
        self.status = status


class LinearT(C.Structure):
    _fields_ = [("d_out", C.c_int32), ("d_in", C.c_int32), ("rank", C.c_int32),
                ("bits", C.c_void_p), ("w_scale", C.c_void_p), ("lora_b", C.c_void_p),
                ("lora_b_scale", C.c_void_p), ("lora_a", C.c_void_p), ("lora_a_scale", C.c_void_p)]


class DebugT(C.Structure):
    _fields_ = [("acc", C.c_void_p), ("lora_t", C.c_void_p), ("xq", C.c_void_p),
                ("xscale", C.c_void_p)]


class DimsT(C.Structure):
    _fields_ = [("d_model", C.c_int32), ("nheads", C.c_int32), ("headdim", C.c_int32),
                ("d_state", C.c_int32), ("ngroups", C.c_int32)]


class LayerT(C.Structure):
    _fields_ = [("in_proj", LinearT), ("out_proj", LinearT), ("conv_w", C.c_void_p),
                ("conv_b", C.c_void_p), ("A_log", C.c_void_p), ("dt_bias", C.c_void_p),
                ("D", C.c_void_p), ("norm_w", C.c_void_p), ("gnorm_w", C.c_void_p)]


_lib = None

# name -> (restype, argtypes); every function that include/dfssm.h declares.
_P, _I, _Z = C.c_void_p, C.c_int, C.c_size_t
SIGNATURES = {
    "dfssm_workspace_size": (_Z, [_I, _I, _I, _I]),
    "dfssm_linear_decode": (_I, [_P, _P, _I, _P, _P, _Z, _P, _P]),
    "dfssm_linear_prefill": (_I, [_P, _P, _I, _P, _P, _Z, _P, _P]),
    "dfssm_linear_decode_noalloc": (_I, [_P, _P, _I, _P, _P, _P]),
    "dfssm_linear_decode_multi": (_I, [_P, _I, _P, _I, _P, _P, C.c_size_t, _P]),
    "dfssm_conv_step": (_I, [_P, _P, _P, _P, _P, _I, _I, _P]),
    "dfssm_ssm_step": (_I, [_P] * 9 + [_I] * 5 + [_P]),
    "dfssm_layer_decode": (_I, [_P, _I, _P, _P, _P, _P, _I, _P, _Z, _P]),
    "dfssm_lm_head": (_I, [_P, _P, _I, _I, _P, _P, _P, _P, _Z, _P]),
    "dfssm_layer_prefill": (_I, [_P, _I, _P, _P, _P, _P, _I, _P, _Z, _P]),
    "dfssm_embed": (_I, [_P, _P, _I, _I, _P, _P, _P, C.c_size_t, _P]),
    "dfssm_head_greedy": (_I, [_P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _Z, _P]),
    "dfssm_generate": (_I, [_P, _I, _P, _P, _P, _I, _P, _P, _I, _P, _P, _P, _P, _P, _Z, _P]),
    "dfssm_state_field_encode": (_I, [_P, _I, _I, _P, _P, _P]),
    "dfssm_state_field_decode": (_I, [_P, _P, _I, _I, _P, _P]),
    "dfssm_state_field_roundtrip": (_I, [_P, _I, _I, _P, _P, _P]),
    "dfssm_pack_signs": (_I, [_P, _I, _I, _P]),
    "dfssm_device_status": (_I, [_P, _P]),
    "dfssm_selftest_timeout": (_I, [_P, _Z, _P]),
    "dfssm_status_string": (C.c_char_p, [_I]),
    "dfssm_last_cuda_error": (C.c_char_p, []),
    "dfssm_abi_version": (_I, []),
}


def lib():
    """Load libdfssm.so (built in-tree by bit_quantized_mamba_b200.build); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdfssm.so not built ({LIB_PATH}); run __graft_entry__.build()")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(fn: str, status: int):
    if status != 0:
        raise DfssmError(fn, status)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _hptr(t):
    """Host pointer of a contiguous CPU tensor (the host-CPU engine's arguments)."""
    if t is None:
        return None
    if t.device.type != "cpu":
        raise ValueError("expected a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _aptr(t, host: bool):
    return _hptr(t) if host else _ptr(t)


def _side(obj, host: bool):
    if obj.host != host:
        raise ValueError(f"{type(obj).__name__} lives in {'host' if obj.host else 'device'} memory; "
                         f"{'the cpu_* calls' if obj.host else 'the CUDA calls'} take it")


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def workspace_size(op: int, a: int, b: int, c: int) -> int:
    return int(lib().dfssm_workspace_size(op, a, b, c))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Caller-owned scratch, zero-filled (torch allocations are 512-byte aligned)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


class Linear:
    """Device copy of one scaffold+LoRA linear (see dfssm_linear_t)."""

    def __init__(self, bits, w_scale, lora_b, lora_b_scale, lora_a, lora_a_scale):
        self.bits, self.w_scale = bits, w_scale
        self.lora_b, self.lora_b_scale = lora_b, lora_b_scale
        self.lora_a, self.lora_a_scale = lora_a, lora_a_scale
        self.d_out = bits.shape[0]
        self.d_in = bits.shape[1] * 32
        self.rank = lora_b.shape[0] if lora_b is not None else 0
        self.host = bits.device.type == "cpu"
        P = lambda t: _aptr(t, self.host)  # noqa: E731
        self._c = LinearT(self.d_out, self.d_in, self.rank, P(bits), P(w_scale),
                          P(lora_b) if self.rank else None, P(lora_b_scale) if self.rank else None,
                          P(lora_a) if self.rank else None, P(lora_a_scale) if self.rank else None)

    @classmethod
    def from_host(cls, d: dict, device="cuda"):
        t = {k: torch.from_numpy(np.ascontiguousarray(v)).to(device) for k, v in d.items()
             if k != "bits"}
        # the sign words travel as int32 (same bytes); only their address reaches the library
        bits = torch.from_numpy(np.ascontiguousarray(d["bits"]).view(np.int32)).to(device)
        return cls(bits, t["w_scale"], t["lora_b"], t["lora_b_scale"], t["lora_a"], t["lora_a_scale"])

    def cstruct(self, host: bool = False) -> LinearT:
        _side(self, host)
        return self._c


def linear_decode(lin: Linear, x: torch.Tensor, y: torch.Tensor | None = None, ws=None,
                  debug: dict | None = None, stream=None) -> torch.Tensor:
    B = x.shape[0]
    if y is None:
        y = torch.empty((B, lin.d_out), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace(workspace_size(OP_LINEAR_DECODE, B, lin.d_in, lin.d_out), x.device)
    dbg = None
    if debug is not None:
        dbg = DebugT(*(_ptr(debug.get(k)) for k in ("acc", "lora_t", "xq", "xscale")))
    _check("dfssm_linear_decode", lib().dfssm_linear_decode(
        C.byref(lin.cstruct()), _ptr(x), B, _ptr(y), _ptr(ws), ws.numel(),
        C.byref(dbg) if dbg is not None else None, _stream(stream)))
    return y


def linear_decode_noalloc(lin: Linear, x: torch.Tensor, y: torch.Tensor | None = None,
                          debug: dict | None = None, stream=None) -> torch.Tensor:
    """dfssm_linear_decode without a workspace (the library keeps a fixed scratch array per device)."""
    B = x.shape[0]
    if y is None:
        y = torch.empty((B, lin.d_out), dtype=torch.float32, device=x.device)
    dbg = None
    if debug is not None:
        dbg = DebugT(*(_ptr(debug.get(k)) for k in ("acc", "lora_t", "xq", "xscale")))
    _check("dfssm_linear_decode_noalloc", lib().dfssm_linear_decode_noalloc(
        C.byref(lin.cstruct()), _ptr(x), B, _ptr(y), C.byref(dbg) if dbg is not None else None,
        _stream(stream)))
    return y


def linear_decode_multi(lins, x: torch.Tensor, ys=None, ws=None, stream=None):
    """n linears that share x in one launch (dfssm_linear_decode_multi); returns the list of outputs.
    ws (optional) holds the call's status word."""
    B = x.shape[0]
    if ys is None:
        ys = [torch.empty((B, L.d_out), dtype=torch.float32, device=x.device) for L in lins]
    if ws is None:
        ws = workspace(workspace_size(OP_LINEAR_MULTI, 0, 0, 0), x.device)
    arr = (LinearT * len(lins))(*[L.cstruct() for L in lins])
    ptrs = (C.c_void_p * len(lins))(*[_ptr(y) for y in ys])
    _check("dfssm_linear_decode_multi", lib().dfssm_linear_decode_multi(
        arr, len(lins), _ptr(x), B, ptrs, _ptr(ws), ws.numel(), _stream(stream)))
    return ys


def linear_prefill(lin: Linear, x: torch.Tensor, y: torch.Tensor | None = None, ws=None,
                   debug: dict | None = None, stream=None) -> torch.Tensor:
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, lin.d_out), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace(workspace_size(OP_LINEAR_PREFILL, M, lin.d_in, lin.d_out), x.device)
    dbg = None
    if debug is not None:
        dbg = DebugT(*(_ptr(debug.get(k)) for k in ("acc", "lora_t", "xq", "xscale")))
    _check("dfssm_linear_prefill", lib().dfssm_linear_prefill(
        C.byref(lin.cstruct()), _ptr(x), M, _ptr(y), _ptr(ws), ws.numel(),
        C.byref(dbg) if dbg is not None else None, _stream(stream)))
    return y


def conv_step(conv_state, w, b, x_in, x_out=None, stream=None):
    B, Cn = x_in.shape
    if x_out is None:
        x_out = torch.empty_like(x_in)
    _check("dfssm_conv_step", lib().dfssm_conv_step(_ptr(conv_state), _ptr(w), _ptr(b), _ptr(x_in),
                                                    _ptr(x_out), B, Cn, _stream(stream)))
    return x_out


def ssm_step(ssm_state, x, dt_raw, A_log, dt_bias, D, Bm, Cm, y=None, stream=None):
    B, H, P, N = ssm_state.shape
    G = Bm.numel() // (B * N)
    if y is None:
        y = torch.empty((B, H * P), dtype=torch.float32, device=x.device)
    _check("dfssm_ssm_step", lib().dfssm_ssm_step(
        _ptr(ssm_state), _ptr(x), _ptr(dt_raw), _ptr(A_log), _ptr(dt_bias), _ptr(D), _ptr(Bm),
        _ptr(Cm), _ptr(y), B, H, P, N, G, _stream(stream)))
    return y


def _field_rows(state):
    N = state.shape[-1]
    return state.numel() // N if N else 0, N


def _field_dtypes(state=None, field=None, scale=None):
    """The density-field calls take f32 rows and scales and 32-bit field words (int32 or uint32)."""
    if state is not None and state.dtype != torch.float32:
        raise ValueError(f"state rows must be float32, not {state.dtype}")
    if field is not None and field.dtype not in (torch.int32, getattr(torch, "uint32", torch.int32)):
        raise ValueError(f"field words must be int32 or uint32, not {field.dtype}")
    if scale is not None and scale.dtype != torch.float32:
        raise ValueError(f"scales must be float32, not {scale.dtype}")


def state_field_encode(state, field=None, scale=None, stream=None):
    """Density-field encoding of the state rows [..., N] (dfssm_state_field_encode): returns (field int32
    [rows, N/8] holding the u32 words, scale float32 [rows])."""
    _field_dtypes(state, field, scale)
    rows, N = _field_rows(state)
    if field is None:
        field = torch.empty((rows, N // 8), dtype=torch.int32, device=state.device)
    if scale is None:
        scale = torch.empty(rows, dtype=torch.float32, device=state.device)
    _check("dfssm_state_field_encode", lib().dfssm_state_field_encode(
        _ptr(state), rows, N, _ptr(field), _ptr(scale), _stream(stream)))
    return field, scale


def state_field_decode(field, scale, N: int, out=None, stream=None):
    """Popcount readout of density fields [rows, N/8] (dfssm_state_field_decode) into rows [rows, N]."""
    _field_dtypes(out, field, scale)
    rows = scale.numel()
    if out is None:
        out = torch.empty((rows, N), dtype=torch.float32, device=scale.device)
    _check("dfssm_state_field_decode", lib().dfssm_state_field_decode(
        _ptr(field), _ptr(scale), rows, N, _ptr(out), _stream(stream)))
    return out


def state_field_roundtrip(state, field=None, scale=None, stream=None):
    """state <- readout(encode(state)) in place (dfssm_state_field_roundtrip); field and scale, when
    given, receive the encoding too."""
    _field_dtypes(state, field, scale)
    rows, N = _field_rows(state)
    _check("dfssm_state_field_roundtrip", lib().dfssm_state_field_roundtrip(
        _ptr(state), rows, N, _ptr(field), _ptr(scale), _stream(stream)))
    return state


class Layer:
    """Device copy of one DF-SSM Mamba-2 layer (see dfssm_layer_t)."""

    VEC = ("conv_w", "conv_b", "A_log", "dt_bias", "D", "norm_w", "gnorm_w")

    def __init__(self, in_proj: Linear, out_proj: Linear, **vec):
        self.in_proj, self.out_proj = in_proj, out_proj
        for k in self.VEC:
            setattr(self, k, vec[k])
        self.host = in_proj.host
        self._c = LayerT(in_proj.cstruct(self.host), out_proj.cstruct(self.host),
                         *(_aptr(vec[k], self.host) for k in self.VEC))

    @classmethod
    def from_host(cls, d: dict, device="cuda"):
        vec = {k: torch.from_numpy(np.ascontiguousarray(d[k])).to(device) for k in cls.VEC}
        return cls(Linear.from_host(d["in_proj"], device), Linear.from_host(d["out_proj"], device),
                   **vec)

    def cstruct(self, host: bool = False) -> LayerT:
        _side(self, host)
        return self._c


class LayerStack:
    """Layers plus their per-layer conv/SSM state tensors, marshalled once for repeated decode calls."""

    def __init__(self, layers: list[Layer], dims: dict, conv_states: list, ssm_states: list):
        n = len(layers)
        self.layers, self.conv_states, self.ssm_states = layers, conv_states, ssm_states
        self.dims = DimsT(dims["d_model"], dims["nheads"], dims["headdim"], dims["d_state"],
                          dims["ngroups"])
        self.d_model = dims["d_model"]
        self.d_inner = dims["nheads"] * dims["headdim"]
        self.host = layers[0].host
        self._layers = (LayerT * n)(*(L.cstruct(self.host) for L in layers))
        self._conv = (C.c_void_p * n)(*(_aptr(t, self.host) for t in conv_states))
        self._ssm = (C.c_void_p * n)(*(_aptr(t, self.host) for t in ssm_states))
        self.n = n

    def c(self, host: bool = False):
        """(layers, conv state pointers, SSM state pointers) for a call on that side of the bus."""
        _side(self, host)
        return self._layers, self._conv, self._ssm


def layer_decode(stack: LayerStack, hidden: torch.Tensor, ws=None, stream=None) -> torch.Tensor:
    """One decode step of every layer of the stack; hidden [B][d_model] is updated in place."""
    B = hidden.shape[0]
    if ws is None:
        ws = workspace(workspace_size(OP_LAYER_DECODE, B, stack.d_model, stack.d_inner),
                       hidden.device)
    _check("dfssm_layer_decode", lib().dfssm_layer_decode(
        *stack.c()[:1], stack.n, C.byref(stack.dims), _ptr(hidden), *stack.c()[1:], B,
        _ptr(ws), ws.numel(), _stream(stream)))
    return hidden


def layer_prefill(stack: LayerStack, hidden: torch.Tensor, ws=None, stream=None) -> torch.Tensor:
    """Prefill of an M-token prompt (hidden [M][d_model], batch 1) through every layer of the stack;
    hidden is updated in place and the stack's states advance by M tokens."""
    M = hidden.shape[0]
    if ws is None:
        ws = workspace(workspace_size(OP_LAYER_PREFILL, M, stack.d_model, stack.d_inner), hidden.device)
    _check("dfssm_layer_prefill", lib().dfssm_layer_prefill(
        *stack.c()[:1], stack.n, C.byref(stack.dims), _ptr(hidden), *stack.c()[1:], M,
        _ptr(ws), ws.numel(), _stream(stream)))
    return hidden


def device_status(ws=None, stream=None) -> int:
    """Synchronise the stream, read and clear the status word at the start of the workspace (None: the
    no-alloc entry point's module word): 0 (DFSSM_OK), -5 (DFSSM_ETIMEOUT) or -1 (DFSSM_EINVAL: a bad
    token id)."""
    return int(lib().dfssm_device_status(_ptr(ws), _stream(stream)))


def selftest_timeout(ws, stream=None) -> None:
    _check("dfssm_selftest_timeout", lib().dfssm_selftest_timeout(_ptr(ws), ws.numel(),
                                                                  _stream(stream)))


def lm_head(W, s_row, x, logits=None, acc=None, ws=None, stream=None):
    V, d = W.shape
    if logits is None:
        logits = torch.empty(V, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace(workspace_size(OP_LM_HEAD, 1, d, V), x.device)
    _check("dfssm_lm_head", lib().dfssm_lm_head(_ptr(W), _ptr(s_row), V, d, _ptr(x), _ptr(logits),
                                                _ptr(acc), _ptr(ws), ws.numel(), _stream(stream)))
    return logits


def embed(W, s_row, token, h=None, ws=None, stream=None):
    """Row token[0] of the tied int8 embedding, dequantized (token: device int32 [1]).  ws (optional)
    holds the call's status word (an out-of-range id is reported there)."""
    V, d = W.shape
    if h is None:
        h = torch.empty(d, dtype=torch.float32, device=W.device)
    if ws is None:
        ws = workspace(workspace_size(OP_EMBED, 0, 0, 0), W.device)
    _check("dfssm_embed", lib().dfssm_embed(_ptr(W), _ptr(s_row), V, d, _ptr(token), _ptr(h), _ptr(ws),
                                            ws.numel(), _stream(stream)))
    return h


def head_greedy(W, s_row, h, norm_w=None, logits=None, acc=None, token=None, ws=None, stream=None):
    """Final RMSNorm (norm_w; None = no norm) + int8 LM head + greedy choice on one token.
    Returns (token device int32 [1], logits)."""
    V, d = W.shape
    if logits is None:
        logits = torch.empty(V, dtype=torch.float32, device=h.device)
    if token is None:
        token = torch.empty(1, dtype=torch.int32, device=h.device)
    if ws is None:
        ws = workspace(workspace_size(OP_HEAD_GREEDY, 1, d, V), h.device)
    _check("dfssm_head_greedy", lib().dfssm_head_greedy(
        _ptr(W), _ptr(s_row), V, d, _ptr(h), _ptr(norm_w), _ptr(logits), _ptr(acc), _ptr(token),
        _ptr(ws), ws.numel(), _stream(stream)))
    return token, logits


def generate(stack: "LayerStack", W, s_row, final_norm_w, tokens, hidden_taps=None, logits=None,
             ws=None, stream=None):
    """Greedy generation at batch 1: tokens (device int32 [n + 1]) holds the first token in [0];
    entries 1..n are written.  The stack's states advance by n steps."""
    V, d = W.shape
    n = tokens.numel() - 1
    if ws is None:
        ws = workspace(workspace_size(OP_GENERATE, V, stack.d_model, stack.d_inner), W.device)
    _check("dfssm_generate", lib().dfssm_generate(
        stack.c()[0], stack.n, C.byref(stack.dims), _ptr(W), _ptr(s_row), V, _ptr(final_norm_w),
        _ptr(tokens), n, stack.c()[1], stack.c()[2], _ptr(hidden_taps), _ptr(logits), _ptr(ws),
        ws.numel(), _stream(stream)))
    return tokens


def pack_signs(signs: np.ndarray) -> np.ndarray:
    """Host: +-1 int8 [d_out][d_in] -> LSB-first uint32 words [d_out][d_in/32]."""
    signs = np.ascontiguousarray(signs, dtype=np.int8)
    d_out, d_in = signs.shape
    bits = np.zeros((d_out, d_in // 32), np.uint32)
    _check("dfssm_pack_signs", lib().dfssm_pack_signs(signs.ctypes.data, d_out, d_in,
                                                      bits.ctypes.data))
    return bits


# ------------------------------------------------------------------ host-CPU engine (include/dfssm_cpu.h)

CPU_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdfssm_cpu.so")
_cpu_lib = None


def cpu_lib():
    """Load libdfssm_cpu.so (built in-tree by bit_quantized_mamba_b200.build.build_cpu); raise if missing."""
    global _cpu_lib
    if _cpu_lib is None:
        if not os.path.exists(CPU_LIB_PATH):
            raise RuntimeError(f"libdfssm_cpu.so not built ({CPU_LIB_PATH}); run __graft_entry__.build()")
        L = C.CDLL(CPU_LIB_PATH)
        L.dfssm_cpu_abi_version.restype = C.c_int
        L.dfssm_cpu_available.restype = C.c_int
        L.dfssm_cpu_set_threads.restype = C.c_int
        L.dfssm_cpu_set_threads.argtypes = [C.c_int]
        L.dfssm_cpu_linear_decode.restype = C.c_int
        L.dfssm_cpu_linear_decode.argtypes = [C.POINTER(LinearT), C.c_void_p, C.c_int, C.c_void_p,
                                              C.POINTER(DebugT)]
        L.dfssm_cpu_layer_decode.restype = C.c_int
        L.dfssm_cpu_layer_decode.argtypes = [C.POINTER(LayerT), C.c_int, C.POINTER(DimsT), C.c_void_p,
                                             C.POINTER(C.c_void_p), C.POINTER(C.c_void_p), C.c_int]
        L.dfssm_cpu_state_field_encode.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p]
        L.dfssm_cpu_state_field_decode.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_void_p]
        L.dfssm_cpu_state_field_roundtrip.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p]
        _cpu_lib = L
    return _cpu_lib


def cpu_available() -> bool:
    """True when the host CPU runs the VNNI engine (AVX-512 F/BW and VNNI)."""
    return bool(cpu_lib().dfssm_cpu_available())


def cpu_set_threads(n: int = 0) -> int:
    return int(cpu_lib().dfssm_cpu_set_threads(n))


def cpu_linear_decode(lin: Linear, x: torch.Tensor, y: torch.Tensor | None = None,
                      debug: dict | None = None) -> torch.Tensor:
    """dfssm_cpu_linear_decode: lin built with host tensors (Linear.from_host(d, "cpu")), x host f32."""
    B = x.shape[0]
    if y is None:
        y = torch.empty((B, lin.d_out), dtype=torch.float32)
    dbg = None
    if debug is not None:
        dbg = DebugT(*(_hptr(debug.get(k)) for k in ("acc", "lora_t", "xq", "xscale")))
    _check("dfssm_cpu_linear_decode", cpu_lib().dfssm_cpu_linear_decode(
        C.byref(lin.cstruct(host=True)), _hptr(x), B, _hptr(y), C.byref(dbg) if dbg is not None else None))
    return y


def cpu_layer_decode(stack: LayerStack, hidden: torch.Tensor) -> torch.Tensor:
    """dfssm_cpu_layer_decode over a LayerStack of host tensors; hidden [B][d_model] updated in place."""
    _check("dfssm_cpu_layer_decode", cpu_lib().dfssm_cpu_layer_decode(
        *stack.c(host=True)[:1], stack.n, C.byref(stack.dims), _hptr(hidden), *stack.c(host=True)[1:],
        hidden.shape[0]))
    return hidden


def cpu_state_field_encode(state: torch.Tensor, field=None, scale=None):
    """dfssm_cpu_state_field_encode on host rows [..., N]: returns (field int32 [rows, N/8] holding the u32
    words, scale float32 [rows])."""
    _field_dtypes(state, field, scale)
    rows, N = _field_rows(state)
    if field is None:
        field = torch.empty((rows, N // 8), dtype=torch.int32)
    if scale is None:
        scale = torch.empty(rows, dtype=torch.float32)
    _check("dfssm_cpu_state_field_encode", cpu_lib().dfssm_cpu_state_field_encode(
        _hptr(state), rows, N, _hptr(field), _hptr(scale)))
    return field, scale


def cpu_state_field_decode(field: torch.Tensor, scale: torch.Tensor, N: int, out=None):
    """dfssm_cpu_state_field_decode: the popcount readout of host fields into rows [rows, N]."""
    _field_dtypes(out, field, scale)
    rows = scale.numel()
    if out is None:
        out = torch.empty((rows, N), dtype=torch.float32)
    _check("dfssm_cpu_state_field_decode", cpu_lib().dfssm_cpu_state_field_decode(
        _hptr(field), _hptr(scale), rows, N, _hptr(out)))
    return out


def cpu_state_field_roundtrip(state: torch.Tensor, field=None, scale=None):
    """dfssm_cpu_state_field_roundtrip: host rows replaced in place by the readout of their encoding."""
    _field_dtypes(state, field, scale)
    rows, N = _field_rows(state)
    _check("dfssm_cpu_state_field_roundtrip", cpu_lib().dfssm_cpu_state_field_roundtrip(
        _hptr(state), rows, N, _hptr(field), _hptr(scale)))
    return state
