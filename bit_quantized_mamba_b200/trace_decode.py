"""Per-phase timeline of the fused 48-layer decode kernel (one token per launch, batch 1).

Builds libdfssm_trace.so (the library with the kernel's phase stamps compiled in: thread 0 of CTA 0 and of
CTA 74 reads the global timer at twelve points of every layer), decodes a few tokens of the Mamba-2-1.3B
shape through it, and prints the mean time of each phase over layers 2..47 of the last token, for both
CTAs.  Usage on a B200:  python -m bit_quantized_mamba_b200.trace_decode
"""
from __future__ import annotations

import ctypes as C

import numpy as np

POINTS = [
    "layer start",
    "h received (poll)",
    "pre-norm + quantize",
    "GEMV pass 0 + LoRA-down",
    "B/C/dt producers, pass 1",
    "B/C/dt received (poll) + state copy",
    "SSM update + g published",
    "g received (poll)",
    "gated norm + quantize",
    "out_proj GEMV + LoRA-down",
    "out_proj epilogue + h published",
    "next layer's copies issued",
]


def main(n_tokens: int = 4) -> None:
    import torch

    from bit_quantized_mamba_b200 import build, dfssm, inputs

    path = build.build_trace()
    L = C.CDLL(path)
    for name, (res, args) in dfssm.SIGNATURES.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    L.dfssm_decode_trace_ptr.restype = C.c_void_p
    dfssm._lib = L
    dev = torch.device("cuda", 0)
    dims = dict(d_model=2048, nheads=64, headdim=64, d_state=128, ngroups=1)
    nl = 48
    m = inputs.decode_model(seed=3, n_layers=nl, n_tokens=n_tokens)
    conv, ssm = inputs.zero_states(1, nl)
    layers = [dfssm.Layer.from_host(x, dev) for x in m["layers"]]
    stack = dfssm.LayerStack(layers, dims, [torch.from_numpy(conv[i]).to(dev) for i in range(nl)],
                             [torch.from_numpy(ssm[i]).to(dev) for i in range(nl)])
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LAYER_DECODE, 1, 2048, 4096), dev)
    for t in range(n_tokens):
        h = torch.from_numpy(np.ascontiguousarray(m["emb"][t])).to(dev)
        dfssm.layer_decode(stack, h, ws)
    torch.cuda.synchronize()
    if dfssm.device_status(ws) != 0:
        raise RuntimeError("the traced decode reported a device-side timeout")
    n = 2 * 64 * len(POINTS)
    buf = torch.empty(n, dtype=torch.int64, device=dev)
    cudart = C.CDLL("libcudart.so.12")
    cudart.cudaMemcpy(C.c_void_p(buf.data_ptr()), C.c_void_p(L.dfssm_decode_trace_ptr()), C.c_size_t(8 * n), 3)
    T = buf.cpu().numpy().reshape(2, 64, len(POINTS)).astype(np.float64)[:, :nl]
    lay = T[:, 2:nl]
    print("phase (mean over layers 2..47, us)      CTA 0    CTA 74")
    for k in range(1, len(POINTS)):
        d = (lay[:, :, k] - lay[:, :, k - 1]).mean(axis=1) / 1e3
        print(f"{POINTS[k]:<38s} {d[0]:7.2f}  {d[1]:7.2f}")
    per_layer = np.diff(T[:, 1:nl, 0], axis=1).mean(axis=1) / 1e3
    print(f"{'layer (start to start)':<38s} {per_layer[0]:7.2f}  {per_layer[1]:7.2f}")
    skew = (T[1, 2:nl, 0] - T[0, 2:nl, 0]).mean() / 1e3
    print(f"layer-start skew, CTA 74 - CTA 0: {skew:.2f} us")


if __name__ == "__main__":
    main()
