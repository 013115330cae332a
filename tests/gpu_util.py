"""Helpers shared by the GPU parity tests: host <-> device transfer of the
synthetic layers and the error bounds the outputs are held to."""
import numpy as np
import torch

import oracle
from synth import LayerSpec, make_layer

DEV = "cuda:0"


def to_dev(layer):
    """numpy layer dict -> torch tensors on the GPU (codes keep their bit patterns)."""
    out = {}
    codes = layer["codes"]
    out["codes"] = torch.from_numpy(np.ascontiguousarray(codes)).to(DEV)
    out["codebooks"] = torch.from_numpy(layer["codebooks"]).to(DEV)
    out["scales"] = torch.from_numpy(layer["scales"]).to(DEV)
    if layer.get("x") is not None:
        x = layer["x"]
        if x.dtype == np.uint16:   # bf16 bit patterns
            out["x"] = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
        else:
            out["x"] = torch.from_numpy(x).to(DEV)
    return out


def bf16_to_np_bits(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def stated_tolerance_bound(W, x64):
    """Per-token bound 2e-3 * ||x_tau||_2 * max_i ||(s . W)_i||_2 (norms in double)."""
    row = np.sqrt((W * W).sum(axis=1)).max()
    return 2e-3 * np.sqrt((x64 * x64).sum(axis=1)) * row          # [T]


def check_fp_output(y_gpu, y_ref, W, x64, out_rel, acc_rel):
    """Hold y_gpu [T, d_out] to both bounds:
    - the stated tolerance, max|y - y_ref| <= 2e-3 ||x|| max_i ||row_i||, per token;
    - a tight one from the arithmetic: out_rel * |y_ref| (one output rounding)
      plus acc_rel * sum_k |W_ik x_k| (fp32 accumulation) plus a subnormal floor."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    err = np.abs(y_gpu - y_ref)
    bound = stated_tolerance_bound(W, x64)
    worst = err.max(axis=1)
    assert np.all(worst <= bound), f"stated tolerance exceeded: {worst} > {bound}"
    absdot = x64.__abs__() @ np.abs(W).T                            # [T, d_out]
    tight = out_rel * np.abs(y_ref) + acc_rel * absdot + 1e-7
    bad = err > tight
    assert not bad.any(), (f"{bad.sum()} outputs outside the arithmetic bound; first at "
                           f"{np.argwhere(bad)[:3].tolist()}: got {y_gpu[bad][:3]}, want {y_ref[bad][:3]}")
    return float(worst.max()), float(bound.min())


def layer(d_out, d_in, M, B, seed=0, tokens=1, x_dtype="fp16"):
    return make_layer(LayerSpec(d_out, d_in, M, B), seed=seed, tokens=tokens, x_dtype=x_dtype)


def oracle_W(L, spec):
    return oracle.dequant_f64(L["codes"], L["codebooks"], L["scales"], spec.d_out, spec.d_in, 8, spec.M, spec.B)
