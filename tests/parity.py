"""Shared helpers for the GPU parity tests: tolerances and comparisons against the oracle."""
import json
import os

import torch

# Tolerances on O and LSE against the fp64 oracle, as stated for this library's target:
# max |dO| <= 2e-2, mean |dO| <= 2e-3, max |dLSE| <= 1e-3 (absolute).
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3


def compare(o_gpu: torch.Tensor, lse_gpu: torch.Tensor, o_ref: torch.Tensor, lse_ref: torch.Tensor,
            what: str = ""):
    """Element-by-element comparison; returns a dict of the errors and asserts the bar."""
    o = o_gpu.detach().cpu().double()
    l = lse_gpu.detach().cpu().double()
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert l.shape == lse_ref.shape, (l.shape, lse_ref.shape)
    assert torch.isfinite(o).all(), f"{what}: non-finite O"
    err = (o - o_ref).abs()
    fin = torch.isfinite(lse_ref)
    assert torch.equal(torch.isfinite(l), fin), f"{what}: LSE finiteness differs"
    assert torch.equal(l[~fin], lse_ref[~fin]), f"{what}: infinite LSE entries differ"
    lerr = (l[fin] - lse_ref[fin]).abs()
    res = {
        "o_max_abs": err.max().item() if err.numel() else 0.0,
        "o_mean_abs": err.mean().item() if err.numel() else 0.0,
        "lse_max_abs": lerr.max().item() if lerr.numel() else 0.0,
        # floor set by rounding the exact result to bf16 (shows pure-rounding failures)
        "bf16_floor": (o_ref.to(torch.bfloat16).double() - o_ref).abs().max().item() if o_ref.numel() else 0.0,
    }
    log = os.environ.get("FA_PARITY_LOG")
    if log:  # optional record of the margins, one JSON object per comparison
        with open(log, "a") as f:
            f.write(json.dumps({"case": what, "test": os.environ.get("PYTEST_CURRENT_TEST", ""), **res}) + "\n")
    assert res["o_max_abs"] <= O_MAX_ABS, f"{what}: {res}"
    assert res["o_mean_abs"] <= O_MEAN_ABS, f"{what}: {res}"
    assert res["lse_max_abs"] <= LSE_MAX_ABS, f"{what}: {res}"
    return res


def guarded(shape, dtype, device, fill=float("nan"), guard=4096):
    """A tensor that is a view into a larger buffer whose guard bands hold `fill`."""
    n = 1
    for s in shape:
        n *= s
    buf = torch.full((guard + n + guard,), fill, dtype=dtype, device=device)
    return buf, buf[guard:guard + n].view(shape)


def guards_intact(buf, guard=4096, fill_is_nan=True):
    head, tail = buf[:guard], buf[-guard:]
    if fill_is_nan:
        return bool(torch.isnan(head.float()).all() and torch.isnan(tail.float()).all())
    return True
