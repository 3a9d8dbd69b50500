"""Seeded synthetic inputs for the DF-SSM decode/prefill workloads.

This module only draws random numbers with the distributions of the published workload shapes; it
holds none of the method's arithmetic.  Both the CPU oracle and the CUDA library are fed from it.

Generator: numpy ``default_rng(seed)`` (PCG64).  Draw order inside each builder is fixed as written.

Distributions (the workload descriptions of the DF-SSM 1.3B shape; starred items are readings where
no distribution is given):
  activations / embeddings       N(0, 1)
  scaffold sign bits             Bernoulli(0.5), packed 32 per uint32 word, least significant bit first
  per-output-channel scale sW    LogNormal(-3, 0.3)
  LoRA W_B, W_A                  int8 uniform on [-127, 127]
  LoRA per-row scales            U(1e-4, 1e-3)
  conv weights                   N(0, 0.1);   conv bias* N(0, 0.1)
  A_log                          U(0, 2.7);   dt_bias U(-4, -1)
  D skip*                        U(0.5, 1.5); RMSNorm weights* U(0.5, 1.5)
  LM head W                      int8 uniform on [-127, 127];  row scales* U(1e-4, 1e-3)
  tied embedding / LM head*      one int8 matrix as the LM head;  final RMSNorm weight* U(0.5, 1.5)
  first token of a generation*   uniform on [0, vocab)
  SSM state rows (density field)* N(0, 1) times a per-row magnitude 10^U(-3, 1); every 64th row all
                                 zero, every 64th (offset 32) one nonzero value (a spike)
"""
from __future__ import annotations

import numpy as np

# Mamba-2 1.3B shape.
D_MODEL = 2048
D_INNER = 4096
N_HEADS = 64
HEADDIM = 64
D_STATE = 128
N_GROUPS = 1
D_CONV = 4
RANK = 16
N_LAYERS = 48
VOCAB = 50288
CONV_CH = D_INNER + 2 * N_GROUPS * D_STATE            # 4352
D_IN_PROJ = 2 * D_INNER + 2 * N_GROUPS * D_STATE + N_HEADS  # 8512


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def linear(g: np.random.Generator, d_out: int, d_in: int, rank: int = RANK) -> dict:
    """One scaffold+LoRA linear (host arrays)."""
    assert d_in % 32 == 0
    return dict(
        bits=g.integers(0, 2**32, size=(d_out, d_in // 32), dtype=np.uint32),
        w_scale=g.lognormal(-3.0, 0.3, size=d_out).astype(np.float32),
        lora_b=g.integers(-127, 128, size=(rank, d_in), dtype=np.int8),
        lora_b_scale=g.uniform(1e-4, 1e-3, size=rank).astype(np.float32),
        lora_a=g.integers(-127, 128, size=(d_out, rank), dtype=np.int8),
        lora_a_scale=g.uniform(1e-4, 1e-3, size=d_out).astype(np.float32),
    )


def layer(g: np.random.Generator, d_model: int = D_MODEL, nheads: int = N_HEADS,
          headdim: int = HEADDIM, d_state: int = D_STATE, ngroups: int = N_GROUPS,
          rank: int = RANK) -> dict:
    """Parameters of one DF-SSM Mamba-2 layer (host arrays)."""
    e = nheads * headdim
    c = e + 2 * ngroups * d_state
    d_ip = 2 * e + 2 * ngroups * d_state + nheads
    return dict(
        in_proj=linear(g, d_ip, d_model, rank),
        out_proj=linear(g, d_model, e, rank),
        conv_w=g.normal(0.0, 0.1, size=(c, D_CONV)).astype(np.float32),
        conv_b=g.normal(0.0, 0.1, size=c).astype(np.float32),
        A_log=g.uniform(0.0, 2.7, size=nheads).astype(np.float32),
        dt_bias=g.uniform(-4.0, -1.0, size=nheads).astype(np.float32),
        D=g.uniform(0.5, 1.5, size=nheads).astype(np.float32),
        norm_w=g.uniform(0.5, 1.5, size=d_model).astype(np.float32),
        gnorm_w=g.uniform(0.5, 1.5, size=e).astype(np.float32),
    )


def normal(g: np.random.Generator, shape) -> np.ndarray:
    return g.standard_normal(size=shape, dtype=np.float64).astype(np.float32)


# ---------------------------------------------------------------- the five published workloads

def tiny_linear(seed: int = 0) -> dict:
    """Tiny linear 1x256 -> 512, rank 16, batch 1."""
    g = rng(seed)
    lin = linear(g, 512, 256, RANK)
    return dict(linear=lin, x=normal(g, (1, 256)))


def in_proj_stack(seed: int = 1, copies: int = N_LAYERS, batch: int = 16) -> dict:
    """48 independent in_proj-shaped linears [8512 x 2048] and x [batch x 2048]; a batch-b run uses
    the first b rows of x."""
    g = rng(seed)
    lins = [linear(g, D_IN_PROJ, D_MODEL, RANK) for _ in range(copies)]
    return dict(linears=lins, x=normal(g, (batch, D_MODEL)))


def out_proj_stack(seed: int = 2, copies: int = N_LAYERS, batch: int = 16) -> dict:
    """48 independent out_proj-shaped linears [2048 x 4096] and x [batch x 4096]."""
    g = rng(seed)
    lins = [linear(g, D_MODEL, D_INNER, RANK) for _ in range(copies)]
    return dict(linears=lins, x=normal(g, (batch, D_INNER)))


def decode_model(seed: int = 3, n_layers: int = N_LAYERS, n_tokens: int = 64, batch: int = 1,
                 **dims) -> dict:
    """A stack of DF-SSM Mamba-2 layers plus random-token embeddings [n_tokens][batch][d_model].
    Default dims are the 1.3B shape; smaller dims (d_model, nheads, headdim, d_state, ngroups, rank)
    give scaled-down stacks for fast tests."""
    g = rng(seed)
    layers = [layer(g, **dims) for _ in range(n_layers)]
    d_model = dims.get("d_model", D_MODEL)
    emb = normal(g, (n_tokens, batch, d_model))
    return dict(layers=layers, emb=emb)


def prefill(seed: int = 4, m: int = 2048, vocab: int = VOCAB) -> dict:
    """Prefill: x_in [m x 2048] and x_out [m x 4096] prompts through in_proj/out_proj-shaped linears,
    plus an int8 LM head [vocab x 2048] applied to the last row of x_in."""
    g = rng(seed)
    x_in = normal(g, (m, D_MODEL))
    x_out = normal(g, (m, D_INNER))
    in_proj = linear(g, D_IN_PROJ, D_MODEL, RANK)
    out_proj = linear(g, D_MODEL, D_INNER, RANK)
    lm_w = g.integers(-127, 128, size=(vocab, D_MODEL), dtype=np.int8)
    lm_s = g.uniform(1e-4, 1e-3, size=vocab).astype(np.float32)
    return dict(x_in=x_in, x_out=x_out, in_proj=in_proj, out_proj=out_proj, lm_w=lm_w, lm_s=lm_s)


def generation_model(seed: int = 5, n_layers: int = N_LAYERS, vocab: int = VOCAB, **dims) -> dict:
    """A stack of layers plus the tied int8 embedding / LM head [vocab x d_model] with its row scales,
    the final RMSNorm weight and a first token, for greedy generation."""
    g = rng(seed)
    layers = [layer(g, **dims) for _ in range(n_layers)]
    d_model = dims.get("d_model", D_MODEL)
    emb_w = g.integers(-127, 128, size=(vocab, d_model), dtype=np.int8)
    emb_s = g.uniform(1e-4, 1e-3, size=vocab).astype(np.float32)
    final_norm_w = g.uniform(0.5, 1.5, size=d_model).astype(np.float32)
    first_token = int(g.integers(0, vocab))
    return dict(layers=layers, emb_w=emb_w, emb_s=emb_s, final_norm_w=final_norm_w,
                first_token=first_token)


def zero_states(batch: int = 1, n_layers: int = N_LAYERS, nheads: int = N_HEADS,
                headdim: int = HEADDIM, d_state: int = D_STATE, ngroups: int = N_GROUPS):
    """Reading (x): initial conv and SSM states are zero."""
    c = nheads * headdim + 2 * ngroups * d_state
    conv = np.zeros((n_layers, batch, c, D_CONV - 1), np.float32)
    ssm = np.zeros((n_layers, batch, nheads, headdim, d_state), np.float32)
    return conv, ssm


def ssm_state_rows(seed: int, rows: int, d_state: int = D_STATE) -> np.ndarray:
    """State rows [rows][d_state] for the density-field encoding: per-row magnitudes spread over four
    decades, with all-zero rows and single-spike rows mixed in (fixed positions)."""
    g = rng(seed)
    mag = (10.0 ** g.uniform(-3.0, 1.0, size=(rows, 1))).astype(np.float32)
    S = (g.standard_normal((rows, d_state), dtype=np.float32) * mag).astype(np.float32)
    S[0::64] = 0.0
    spikes = np.arange(32, rows, 64)
    if len(spikes):
        pos = g.integers(0, d_state, size=len(spikes))
        val = g.standard_normal(len(spikes), dtype=np.float32)
        S[spikes] = 0.0
        S[spikes, pos] = val
    return S
