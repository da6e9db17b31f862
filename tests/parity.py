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


# Backward pass (dQ, dK, dV), per gradient tensor over the compared set:
#   max |G - G*| <= 2e-2 * max |G*|  and  sqrt(sum (G - G*)^2 / sum G*^2) <= 1e-2
# Derived from the arithmetic: P and dS are rounded to bf16 (relative
# 2^-9 = 1.95e-3 per element) before their products, the outputs are rounded
# to bf16 once more, and delta_i = dO_i . O_i uses the bf16 O of the forward
# pass. A CPU model of exactly these roundings on the test inputs gives
# relative RMS 2.2e-3 to 4e-3 and max-abs 2.2e-3 to 5.7e-3 times max |G*|;
# the bounds leave a factor 2.5 to 3.5 for the tensor-core accumulation
# order and the fp32 atomic sum of dQ.
# A gradient that is exactly zero in exact arithmetic (one allowed key, w = 0)
# comes out as fp32 rounding noise (dO.v from the tensor cores minus dO.O
# from the fp32 row sum, about 1e-7): an absolute floor of 1e-5 covers it and
# is far below the bf16 resolution of any nonzero gradient compared here.
G_MAX_ABS_REL = 2e-2
G_REL_RMS = 1e-2
G_ABS_FLOOR = 1e-5


def grad_errors(g, g_ref):
    g = np.asarray(g, dtype=np.float64)
    g_ref = np.asarray(g_ref, dtype=np.float64)
    diff = g - g_ref
    scale = float(np.abs(g_ref).max()) if g_ref.size else 0.0
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float((g_ref ** 2).sum())
    rel_rms = float(np.sqrt((diff ** 2).sum() / denom)) if denom > 0 else float(np.sqrt((diff ** 2).sum()))
    return {"max_abs": max_abs, "max_ref": scale, "rel_rms": rel_rms, "finite": bool(np.isfinite(g).all())}


def assert_grads_close(grads, refs, what=""):
    out = {}
    for name, g, r in zip(("dq", "dk", "dv"), grads, refs):
        e = grad_errors(g, r)
        assert e["finite"], f"{what} {name}: non-finite"
        assert e["max_abs"] <= G_MAX_ABS_REL * e["max_ref"] + G_ABS_FLOOR, f"{what} {name}: {e}"
        if e["max_ref"] > 0:
            assert e["rel_rms"] <= G_REL_RMS, f"{what} {name}: {e}"
        out[name] = e
    return out
