"""Host-side checks of the C ABI (no GPU): the library builds, loads, exports every function that
include/dfssm.h declares, and validates arguments before touching a device."""
import ctypes as C
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dfssm.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dfssm_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from bit_quantized_mamba_b200 import build, dfssm
    build.build()
    return dfssm.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("dfssm_linear_decode", "dfssm_linear_prefill", "dfssm_conv_step",
                     "dfssm_ssm_step", "dfssm_layer_decode"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    from bit_quantized_mamba_b200 import dfssm
    names = declared_functions()
    for n in names:
        assert hasattr(L, n), f"{n} declared in dfssm.h but not exported"
    assert set(names) == set(dfssm.SIGNATURES), "binding and header disagree"
    assert L.dfssm_abi_version() == 5


def test_cpu_engine_exports_every_declared_symbol():
    """libdfssm_cpu.so (the host-CPU engine) exports every function include/dfssm_cpu.h declares and
    validates its arguments before computing (no AVX-512 needed for these calls)."""
    from bit_quantized_mamba_b200 import build, dfssm
    build.build_cpu()
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "dfssm_cpu.h")).read(), flags=re.S)
    names = sorted(set(re.findall(r"\b(dfssm_cpu_[a-z0-9_]+)\s*\(", text)))
    assert len(names) >= 5
    Lc = dfssm.cpu_lib()
    for n in names:
        assert hasattr(Lc, n), f"{n} declared in dfssm_cpu.h but not exported"
    assert Lc.dfssm_cpu_abi_version() == 2
    assert Lc.dfssm_cpu_available() in (0, 1)
    assert Lc.dfssm_cpu_linear_decode(None, None, 1, None, None) == -1
    assert Lc.dfssm_cpu_layer_decode(None, 0, None, None, None, None, 1) == -1
    assert Lc.dfssm_cpu_state_field_encode(None, 4, 12, None, None) == -1      # N % 8
    assert Lc.dfssm_cpu_state_field_encode(None, 4, 264, None, None) == -3     # N > 256
    assert Lc.dfssm_cpu_state_field_encode(None, 4, 128, None, None) == -1     # NULL rows
    assert Lc.dfssm_cpu_state_field_decode(None, None, 0, 128, None) == 0      # no rows
    assert Lc.dfssm_cpu_state_field_roundtrip(None, -1, 128, None, None) == -1


def test_status_strings(L):
    assert L.dfssm_status_string(0) == b"ok"
    assert L.dfssm_status_string(-7).startswith(b"workspace")


def test_workspace_sizes(L):
    from bit_quantized_mamba_b200 import dfssm
    assert dfssm.workspace_size(dfssm.OP_LINEAR_DECODE, 1, 2048, 8512) >= 2048 + 16 * 16 * 4
    assert dfssm.workspace_size(dfssm.OP_LINEAR_DECODE, 17, 2048, 8512) == 0
    assert dfssm.workspace_size(dfssm.OP_LINEAR_DECODE, 1, 100, 8512) == 0
    assert dfssm.workspace_size(dfssm.OP_LAYER_DECODE, 1, 2048, 4096) > 8512 * 4
    assert dfssm.workspace_size(dfssm.OP_LM_HEAD, 1, 2048, 50288) >= 2048
    assert dfssm.workspace_size(dfssm.OP_HEAD_GREEDY, 1, 2048, 50288) >= 16
    gen = dfssm.workspace_size(dfssm.OP_GENERATE, 50288, 2048, 4096)
    assert gen >= dfssm.workspace_size(dfssm.OP_LAYER_DECODE, 1, 2048, 4096) + 4 * (2048 + 50288) + 16
    assert dfssm.workspace_size(dfssm.OP_GENERATE, 0, 2048, 4096) == 0
    # the status word every workspace starts with
    assert dfssm.workspace_size(dfssm.OP_LINEAR_MULTI, 0, 0, 0) == 256
    assert dfssm.workspace_size(dfssm.OP_EMBED, 0, 0, 0) == 256
    assert (dfssm.workspace_size(dfssm.OP_LINEAR_DECODE, 1, 2048, 8512)
            >= 256 + 2048 + 16 * 16 * 4)


def test_argument_validation_precedes_device_use(L):
    """Invalid arguments are rejected on the host (these calls would fault if they reached a device)."""
    from bit_quantized_mamba_b200 import dfssm
    lin = dfssm.LinearT(512, 100, 16, 16, 16, 16, 16, 16, 16)  # d_in not a multiple of 32
    assert L.dfssm_linear_decode(C.byref(lin), 16, 1, 16, 256, 1 << 20, None, None) == -1
    lin = dfssm.LinearT(512, 256, 17, 16, 16, 16, 16, 16, 16)  # rank > 16
    assert L.dfssm_linear_decode(C.byref(lin), 16, 1, 16, 256, 1 << 20, None, None) == -1
    lin = dfssm.LinearT(512, 256, 16, 8, 16, 16, 16, 16, 16)   # bits misaligned
    assert L.dfssm_linear_decode(C.byref(lin), 16, 1, 16, 256, 1 << 20, None, None) == -2
    lin = dfssm.LinearT(512, 256, 16, 16, 16, 16, 16, 16, 16)
    assert L.dfssm_linear_decode(C.byref(lin), 16, 17, 16, 256, 1 << 20, None, None) == -3
    assert L.dfssm_linear_decode(C.byref(lin), 16, 1, 16, None, 1 << 20, None, None) == -7
    assert L.dfssm_linear_decode(C.byref(lin), 16, 1, 16, 256, 10, None, None) == -7
    assert L.dfssm_linear_decode(None, 16, 1, 16, 256, 1 << 20, None, None) == -1
    assert L.dfssm_ssm_step(16, 16, 16, 16, 16, 16, 16, 16, 16, 1, 3, 4, 8, 2, None) == -1  # H % G
    assert L.dfssm_ssm_step(16, 16, 16, 16, 16, 16, 16, 16, 16, 1, 4, 4, 6, 1, None) == -3  # N % 4
    assert L.dfssm_conv_step(None, 16, 16, 16, 16, 1, 8, None) == -1
    assert L.dfssm_lm_head(16, 16, 10, 24, 16, 16, None, 256, 1 << 20, None) == -1  # d % 16
    assert L.dfssm_embed(16, 16, 10, 24, 16, 16, 256, 256, None) == -1              # d % 16
    assert L.dfssm_embed(16, 16, 10, 32, 16, 8, 256, 256, None) == -2               # h misaligned
    assert L.dfssm_embed(16, 16, 10, 32, None, 16, 256, 256, None) == -1            # no token
    assert L.dfssm_embed(16, 16, 10, 32, 16, 16, None, 256, None) == -7             # no workspace
    assert L.dfssm_embed(16, 16, 10, 32, 16, 16, 256, 64, None) == -7               # workspace too small
    assert L.dfssm_head_greedy(16, 16, 10, 32, 16, None, 16, None, 16, None, 256, None) == -7
    assert L.dfssm_head_greedy(16, 16, 10, 32, 16, None, None, None, 16, 256, 256, None) == -1
    assert L.dfssm_head_greedy(16, 16, 10, 16384, 16, None, 16, None, 16, 256, 256, None) == -3
    dims = dfssm.DimsT(2048, 64, 64, 128, 1)
    assert L.dfssm_generate(None, 48, C.byref(dims), 16, 16, 10, 16, 16, 0, None, None, None, None,
                            256, 1 << 30, None) == -1                                 # n_tokens 0
    assert L.dfssm_generate(None, 48, C.byref(dims), 16, 16, 10, 16, 16, 4, None, None, None, None,
                            256, 1024, None) == -7                                    # workspace
    assert L.dfssm_generate(None, 48, C.byref(dims), 16, 16, 10, 16, 16, 4, None, None, None, None,
                            256, 1 << 30, None) == -1                                 # no layers


def test_state_field_validation_precedes_device_use(L):
    """The density-field calls reject bad sizes, pointers and alignment on the host."""
    for enc in (lambda st, r, n, f, s: L.dfssm_state_field_encode(st, r, n, f, s, None),
                lambda st, r, n, f, s: L.dfssm_state_field_decode(f, s, r, n, st, None)):
        assert enc(None, 4, 128, 256, 256) == -1      # no state
        assert enc(256, 4, 128, None, 256) == -1      # no field
        assert enc(256, 4, 128, 256, None) == -1      # no scale
        assert enc(256, -1, 128, 256, 256) == -1      # rows < 0
        assert enc(256, 4, 12, 256, 256) == -1        # N % 8
        assert enc(256, 4, 0, 256, 256) == -1         # N < 8
        assert enc(256, 4, 264, 256, 256) == -3       # N > 256
        assert enc(8, 4, 128, 256, 256) == -2         # state not 16-byte aligned
        assert enc(256, 4, 128, 2, 256) == -2         # field misaligned
    assert L.dfssm_state_field_roundtrip(256, 4, 128, 256, None, None) == -1  # field without scale
    assert L.dfssm_state_field_roundtrip(256, 4, 128, None, 256, None) == -1  # scale without field
    assert L.dfssm_state_field_roundtrip(None, 4, 128, None, None, None) == -1
    assert L.dfssm_state_field_roundtrip(8, 4, 128, None, None, None) == -2
    assert L.dfssm_state_field_roundtrip(256, 4, 304, None, None, None) == -3
    # no rows: nothing to read, NULL pointers accepted, no device touched
    assert L.dfssm_state_field_encode(None, 0, 128, None, None, None) == 0
    assert L.dfssm_state_field_decode(None, None, 0, 128, None, None) == 0
    assert L.dfssm_state_field_roundtrip(None, 0, 128, None, None, None) == 0
    assert L.dfssm_state_field_encode(None, 0, 12, None, None, None) == -1


def _linears(dfssm, *descs):
    arr = (dfssm.LinearT * len(descs))(*descs)
    return arr


def test_multi_and_noalloc_validate_like_the_single_call(L):
    """dfssm_linear_decode_multi and dfssm_linear_decode_noalloc reject the same malformed descriptors as
    dfssm_linear_decode (one shared check), and their own size limits, before touching a device."""
    from bit_quantized_mamba_b200 import dfssm
    ys = (C.c_void_p * 2)(16, 16)
    good = dfssm.LinearT(512, 2048, 16, 16, 16, 16, 16, 16, 16)
    cases = [
        (dfssm.LinearT(512, 100, 16, 16, 16, 16, 16, 16, 16), -1),   # d_in not a multiple of 32
        (dfssm.LinearT(512, 256, 17, 16, 16, 16, 16, 16, 16), -1),   # rank > 16
        (dfssm.LinearT(512, 256, 16, 8, 16, 16, 16, 16, 16), -2),    # bits misaligned
        (dfssm.LinearT(512, 256, 16, 16, 16, 16, 16, 8, 16), -2),    # W_A misaligned at rank 16
        (dfssm.LinearT(512, 256, 16, None, 16, 16, 16, 16, 16), -1), # no bits
        (dfssm.LinearT(512, 8224, 16, 16, 16, 16, 16, 16, 16), -3),  # d_in above 8192
    ]
    for desc, want in cases:
        assert L.dfssm_linear_decode(C.byref(desc), 16, 1, 16, 256, 1 << 20, None, None) == want
        assert L.dfssm_linear_decode_noalloc(C.byref(desc), 16, 1, 16, None, None) == want
        arr = _linears(dfssm, good, desc)
        assert L.dfssm_linear_decode_multi(arr, 2, 16, 1, ys, 256, 256, None) == want
    assert L.dfssm_linear_decode_noalloc(None, 16, 1, 16, None, None) == -1
    assert L.dfssm_linear_decode_noalloc(C.byref(good), 16, 17, 16, None, None) == -3   # B > 16
    assert L.dfssm_linear_decode_noalloc(C.byref(good), 8, 1, 16, None, None) == -2     # x misaligned
    assert L.dfssm_linear_decode_noalloc(C.byref(good), None, 1, 16, None, None) == -1  # no x
    arr = _linears(dfssm, good, good)
    assert L.dfssm_linear_decode_multi(arr, 2, 16, 1, ys, None, 256, None) == -7        # no workspace
    assert L.dfssm_linear_decode_multi(arr, 2, 16, 1, ys, 256, 16, None) == -7          # too small
    odd = dfssm.LinearT(512, 384, 16, 16, 16, 16, 16, 16, 16)
    arr = _linears(dfssm, odd, odd)
    assert L.dfssm_linear_decode_multi(arr, 2, 16, 1, ys, 256, 256, None) == -3         # d_in 384


def test_pack_signs_matches_oracle_bit_layout(L):
    """The host packer writes the documented layout (checked against the oracle's independent unpack)."""
    import oracle
    from bit_quantized_mamba_b200 import dfssm
    g = np.random.default_rng(3)
    signs = g.choice(np.array([-1, 1], np.int8), size=(7, 96))
    bits = dfssm.pack_signs(signs)
    for o in range(7):
        for i in range(96):
            assert oracle.sign(bits, 96, o, i) == signs[o, i]
