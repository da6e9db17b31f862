"""Error metrics and tolerances for comparing the CUDA path with the oracle.

Tolerances (bf16 inputs, fp32 accumulation, bf16 output), applied to O and
LSE over the compared set:
  O   : max |O - O*| <= 2e-2 and sqrt(sum (O - O*)^2 / sum O*^2) <= 5e-3
  LSE : max |LSE - LSE*| <= 1e-3 (natural-log units)
"""
import numpy as np

O_MAX_ABS = 2e-2
O_REL_RMS = 5e-3
LSE_MAX_ABS = 1e-3


def errors(o, lse, o_ref, lse_ref):
    o = np.asarray(o, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    diff = o - o_ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float((o_ref ** 2).sum())
    rel_rms = float(np.sqrt((diff ** 2).sum() / denom)) if denom > 0 else float(np.sqrt((diff ** 2).sum()))
    lse_err = float(np.abs(lse - lse_ref).max()) if lse.size else 0.0
    return {"o_max_abs": max_abs, "o_rel_rms": rel_rms, "lse_max_abs": lse_err,
            "finite": bool(np.isfinite(o).all() and np.isfinite(lse).all())}


def assert_close(o, lse, o_ref, lse_ref, what=""):
    e = errors(o, lse, o_ref, lse_ref)
    assert e["finite"], f"{what}: non-finite output"
    assert e["o_max_abs"] <= O_MAX_ABS, f"{what}: {e}"
    assert e["o_rel_rms"] <= O_REL_RMS, f"{what}: {e}"
    assert e["lse_max_abs"] <= LSE_MAX_ABS, f"{what}: {e}"
    return e
