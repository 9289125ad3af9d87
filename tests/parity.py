"""Shared helpers of the GPU parity tests (tolerances, device tensors)."""
import numpy as np
import pytest
import torch

# Tolerances for floating point outputs: max-abs 1e-2 and mean-abs 1e-3 on O and
# the gradients, 1e-3 absolute on LSE.  For bf16 outputs the tolerance is applied
# on top of the output format's own rounding: half the bf16 spacing at the exact
# value (2^-9 relative), since a perfectly rounded bf16 value of magnitude >= 4
# already differs from the exact one by up to 2^-6.
MAX_ABS = 1e-2
MEAN_ABS = 1e-3
LSE_ABS = 1e-3


def bf16_half_spacing(ref):
    a = np.maximum(np.abs(ref), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 8)


# One record per checked output: the error as written (no slack), how many
# entries exceed the stated max-abs bound as written, and how many of those sit
# where |oracle| >= 2 (where a perfectly rounded bf16 value may already miss).
# conftest.py prints them at the end of the session and, when PARITY_REPORT
# names a file, appends them to it as JSON lines.
REPORT = []


def _case():
    import os
    return os.environ.get("PYTEST_CURRENT_TEST", "?").split(" (")[0].split("::")[-1]


def record(what, got, ref, bf16_output):
    err = np.abs(got - ref)
    over = err > MAX_ABS
    REPORT.append({"case": _case(), "what": what, "n": int(err.size), "bf16": bool(bf16_output),
                   "max_abs": float(err.max(initial=0.0)), "mean_abs": float(err.mean()) if err.size else 0.0,
                   "over_1e-2": int(over.sum()), "over_1e-2_at_abs_ref_ge_2": int((over & (np.abs(ref) >= 2)).sum()),
                   "max_abs_ref": float(np.abs(ref).max(initial=0.0))})


def check_close(got, ref, bf16_output, what="output", max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    record(what, got, ref, bf16_output)
    err = np.abs(got - ref)
    slack = bf16_half_spacing(ref) if bf16_output else np.zeros_like(ref)
    worst = np.argmax(err - slack)
    assert np.all(err <= max_abs + slack), \
        f"{what}: max err {err.flat[worst]:.3e} at {np.unravel_index(worst, err.shape)} (ref {ref.flat[worst]:.4f})"
    assert err.mean() <= mean_abs + slack.mean(), f"{what}: mean err {err.mean():.3e}"


def check_lse(got, ref, what="lse"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    inf_ref = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), inf_ref), f"{what}: -inf pattern differs"
    if (~inf_ref).any():
        err = np.abs(got[~inf_ref] - ref[~inf_ref])
        REPORT.append({"case": _case(), "what": what, "n": int(err.size), "bf16": False, "max_abs": float(err.max()),
                       "mean_abs": float(err.mean()), "over_1e-3": int((err > LSE_ABS).sum())})
        assert err.max() <= LSE_ABS, f"{what}: max err {err.max():.3e}"


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    major, minor = torch.cuda.get_device_capability()
    if (major, minor) != (10, 0):
        pytest.skip(f"needs sm_100 (B200), found sm_{major}{minor}")
    from exact_tiled_attention_46_b200 import build
    build.build()


def f64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


# e4m3 rounding of the probabilities in the FP8 forward.  The kernel stores
# y_i = 2^(x_i - m + 8) with m within 0.75 (log2) below the row's running max,
# rounded to e4m3: |y~ - y| <= 2^-4 y where y is a normal e4m3 value and
# <= 2^-10 below (subnormal spacing 2^-9), i.e. <= 2^-18 of the row's largest
# probability.  With O normalised by the sum of the rounded values,
#     O_gpu - O = sum_i (p~_i - p_i) (v_i - O) / sum_i p~_i
# exactly, so per output element
#     |O_gpu - O| <= (2^-4 sum_i w_i |v_i - O| + 2^-18 sum_i |v_i - O|) / (1 - 2^-4 - n 2^-18)
# (w the exact softmax weights, i over the n allowed keys).  Everything else
# (fp32 accumulation, the hardware exp2) stays far below FP8_SLACK.
FP8_P_REL = 2.0 ** -4
FP8_P_ABS = 2.0 ** -18
FP8_SLACK = 1e-3


def fp8_o_bound(w, allowed, v, o, rows_per_block=64):
    """Per-element bound [Lq, D] for one (batch, head): w [Lq, Lk] exact softmax
    weights, allowed [Lq, Lk] bool, v [Lk, D] (dequantized), o [Lq, D] oracle O."""
    Lq, D = o.shape
    out = np.zeros((Lq, D))
    for r0 in range(0, Lq, rows_per_block):
        r1 = min(Lq, r0 + rows_per_block)
        dev = np.abs(v[None, :, :] - o[r0:r1, None, :])                 # [rows, Lk, D]
        a = allowed[r0:r1, :, None]
        s_w = np.einsum("rk,rkd->rd", w[r0:r1], dev)
        s_abs = np.where(a, dev, 0.0).sum(axis=1)
        n = allowed[r0:r1].sum(axis=1)[:, None]
        out[r0:r1] = (FP8_P_REL * s_w + FP8_P_ABS * s_abs) / (1.0 - FP8_P_REL - n * FP8_P_ABS)
    return out


def check_fp8_o(got, ref, bound, bf16_output, what="O fp8"):
    """|got - ref| <= bound + FP8_SLACK (+ half a bf16 spacing for bf16 outputs)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape == bound.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    record(what, got, ref, bf16_output)
    err = np.abs(got - ref)
    lim = bound + FP8_SLACK + (bf16_half_spacing(ref) if bf16_output else 0.0)
    worst = np.argmax(err - lim)
    assert np.all(err <= lim), (f"{what}: err {err.flat[worst]:.3e} > bound {lim.flat[worst]:.3e} at "
                                f"{np.unravel_index(worst, err.shape)}")
    REPORT[-1]["fp8_bound_max"] = float(bound.max(initial=0.0))
    REPORT[-1]["err_over_bound_max"] = float(np.max(err / lim, initial=0.0))
