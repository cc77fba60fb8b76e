"""Tolerances and comparison helpers shared by the GPU parity tests.

Bars (from the operator's accuracy targets):
* fp32 inputs: max |out_gpu - out_oracle| <= 1e-4 (absolute).
* bf16 inputs: max |out_gpu - out_oracle| / RMS(out_oracle) <= 2e-2 over the
  checked rows of a configuration.
* lse: |lse_gpu - lse_oracle| <= 1e-5 * max(1, |lse|) for fp32 inputs and
  <= 1e-3 for bf16 inputs.
The oracle always sees the exact values the GPU saw (bf16 upcast exactly).

A bf16 OUTPUT is itself rounded to 8 significant bits: |x - bf16(x)| <= 2^-8 |x|.
On the named workloads (long contexts) max|out| is a few times RMS(out) and
this rounding is far inside the bar.  Edge-case shapes with a handful of keys
can have max|out| near 20 x RMS, where rounding alone would exceed 2e-2 RMS;
those tests pass ``output_rounding=True``, which adds the format's own bound
2^-8 |ref| per element to the bar.
"""
import numpy as np

FP32_ATOL = 1e-4
BF16_REL_RMS = 2e-2
LSE_FP32_REL = 1e-5
LSE_BF16_ABS = 1e-3


def to_np(t):
    import torch
    t = t.detach().to("cpu")
    if t.dtype in (torch.bfloat16, torch.float16):
        t = t.float()
    return t.numpy().astype(np.float64)


def check_out(gpu, ref, bf16: bool, what: str = "", output_rounding: bool = False):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, f"{what}: shape {gpu.shape} vs {ref.shape}"
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    err = np.max(np.abs(gpu - ref)) if gpu.size else 0.0
    if bf16:
        rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 1.0
        diff = np.abs(gpu - ref)
        if output_rounding and gpu.size:
            diff = np.maximum(diff - 2.0 ** -8 * np.abs(ref), 0.0)
        err = float(diff.max()) if gpu.size else 0.0
        rel = err / max(rms, 1e-30)
        where = np.unravel_index(int(np.argmax(diff)), diff.shape) if gpu.size else ()
        assert rel <= BF16_REL_RMS, (f"{what}: max err {err:.3e} / rms {rms:.3e} = {rel:.3e} "
                                     f"at {where} (gpu {gpu[where]:.5f}, ref {ref[where]:.5f})")
        return rel
    assert err <= FP32_ATOL, f"{what}: max abs err {err:.3e} > {FP32_ATOL}"
    return err


def check_lse(gpu, ref, bf16: bool, what: str = ""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(gpu), fin), f"{what}: lse finiteness differs"
    if not fin.any():
        return 0.0
    d = np.abs(gpu[fin] - ref[fin])
    if bf16:
        err = float(d.max())
        assert err <= LSE_BF16_ABS, f"{what}: lse err {err:.3e}"
    else:
        err = float((d / np.maximum(1.0, np.abs(ref[fin]))).max())
        assert err <= LSE_FP32_REL, f"{what}: lse rel err {err:.3e}"
    return err
