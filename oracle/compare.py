"""Parity rules between a computed EM step and the oracle's (TEST INFRASTRUCTURE ONLY).

The pages state no tolerances; these are the stated definitions used by the
tests and the benchmark (relative 1e-3 on weights, means and variances, 1e-4
relative on the total log-likelihood, top-m indices exact except where the
oracle's responsibility gap is below 1e-5):

  weights    |dpi|  <= 1e-3 pi_ref + 1e-9
  means      |dmu|  <= 1e-3 max(|mu_ref|, sqrt(var_ref))   (a mean near 0 has no
                                                           relative scale)
  variances  |dvar| <= 1e-3 var_ref
  LL         |dLL|  <= 1e-4 |LL_ref|
Means and variances are gated only for components with N_k_ref >= 10 points
(the rest are reported).  Comparisons are teacher-forced: both sides start the
step from the same stored parameters.  The report also carries the weight
ratio under the looser reading 1e-3 max(pi_ref, 10/N) ("w_floor10") for
comparison with earlier records.
"""
import numpy as np

REL = 1e-3
LL_REL = 1e-4
MIN_NK = 10.0
TOPM_GAP = 1e-5
W_ABS = 1e-9


def compare_step(ref, got, Nk_ref, N=None):
    """ref/got = (w, mu, var, ll).  Returns a dict of worst ratios (<= 1 passes) and 'ok'.

    N (the number of points) defaults to sum(Nk_ref)."""
    w_r, mu_r, var_r, ll_r = (np.asarray(a, dtype=np.float64) for a in ref)
    w_g, mu_g, var_g, ll_g = (np.asarray(a, dtype=np.float64) for a in got)
    Nk_ref = np.asarray(Nk_ref, dtype=np.float64)
    gate = Nk_ref >= MIN_NK
    N = float(Nk_ref.sum()) if N is None else float(N)
    rw = np.abs(w_g - w_r) / (REL * w_r + W_ABS)
    rw_floor10 = np.abs(w_g - w_r) / (REL * np.maximum(w_r, MIN_NK / max(N, 1.0)))
    scale_mu = REL * np.maximum(np.abs(mu_r), np.sqrt(var_r))
    rmu = np.abs(mu_g - mu_r) / scale_mu
    rvar = np.abs(var_g - var_r) / (REL * var_r)
    rll = abs(float(ll_g) - float(ll_r)) / (LL_REL * abs(float(ll_r)))
    out = {
        "w": float(rw.max()),
        "w_worst_k": int(np.argmax(rw)),
        "w_floor10": float(rw_floor10.max()),
        "mu": float(rmu[gate].max()) if gate.any() else 0.0,
        "var": float(rvar[gate].max()) if gate.any() else 0.0,
        "ll": rll,
        "mu_ungated": float(rmu[~gate].max()) if (~gate).any() else 0.0,
        "var_ungated": float(rvar[~gate].max()) if (~gate).any() else 0.0,
        "gated_components": int(gate.sum()),
    }
    out["ok"] = bool(np.isfinite([out["w"], out["mu"], out["var"], out["ll"]]).all()
                     and max(out["w"], out["mu"], out["var"], out["ll"]) <= 1.0)
    return out


def compare_topm(idx_ref, resp_ref, idx_got, resp_got, R_sorted_ref=None):
    """Top-m check.  A mismatch at rank j is excused iff the oracle's
    r_(j) - r_(j+1) < 1e-5 (the two candidates are within the gap), where
    R_sorted_ref holds the oracle's m+1 largest responsibilities per row.
    Responsibilities are compared at 1e-3 relative where >= 1e-6 and the
    indices agree.
    Returns (n_unexcused_index_mismatches, worst_resp_ratio)."""
    idx_ref = np.asarray(idx_ref)
    idx_got = np.asarray(idx_got)
    resp_ref = np.asarray(resp_ref, dtype=np.float64)
    resp_got = np.asarray(resp_got, dtype=np.float64)
    same = idx_ref == idx_got
    mism = ~same
    if R_sorted_ref is not None:
        gaps = np.abs(np.diff(np.asarray(R_sorted_ref, dtype=np.float64), axis=1))
        m = idx_ref.shape[1]
        # rank j may swap with j+1 (gap j) or with j-1 (gap j-1)
        near = gaps[:, :m] < TOPM_GAP
        near_prev = np.zeros_like(near)
        near_prev[:, 1:] = gaps[:, :m - 1] < TOPM_GAP
        mism = mism & ~(near | near_prev)
    big = (resp_ref >= 1e-6) & same
    ratio = np.zeros_like(resp_ref)
    ratio[big] = np.abs(resp_got[big] - resp_ref[big]) / (REL * resp_ref[big])
    return int(mism.sum()), float(ratio.max()) if ratio.size else 0.0
