"""Comparators for GPU-vs-oracle parity (test helpers; no method arithmetic).

Tolerances:
* CSR masks: identical, except kv-blocks whose oracle p lies within 1e-5 of the
  row's threshold p (the p of the last block the rule keeps).  In mass mode a
  row whose cumulative mass at the cut, or one block before it, lies within
  1e-5 of tau is exempt from equality; its block set must still be valid
  (ascending, in range, forced blocks present, size within the cap) and be the
  forced blocks plus a prefix of the (p desc, j asc) order one block shorter,
  as long or one longer than the oracle's (capped), ties within 1e-5 swapped.
* O: max |O_gpu - O_ref| <= 2e-2 and rms(O_gpu - O_ref) / rms(O_ref) <= 1e-2.
* LSE: max |LSE_gpu - LSE_ref| <= 1e-3 where finite; -inf exactly where the
  oracle's is -inf (empty rows), and O exactly 0 there.
"""
from __future__ import annotations

import numpy as np

MASK_BAND = 1e-5
O_MAX_ABS = 2e-2
O_REL_RMS = 1e-2
LSE_ABS = 1e-3


def csr_rows(row_ptr, col_idx):
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    col_idx = np.asarray(col_idx)
    return [col_idx[row_ptr[r]:row_ptr[r + 1]].tolist() for r in range(len(row_ptr) - 1)]


def check_csr_valid(row_ptr, col_idx, nb):
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    assert row_ptr[0] == 0 and np.all(np.diff(row_ptr) >= 0)
    assert row_ptr[-1] == len(col_idx)
    for cols in csr_rows(row_ptr, col_idx):
        assert all(0 <= c < nb for c in cols)
        assert all(a < b for a, b in zip(cols, cols[1:]))


def _is_near_prefix(g, p, m, cap, forced):
    """True if the row g is F ∪ (the first L blocks in (p desc, j asc) order) for
    some L in {m-1, m, m+1} (each capped), up to swaps among blocks whose p lies
    within MASK_BAND of the p at that cut: the rows a mass cut within MASK_BAND
    of tau may validly give."""
    order = np.lexsort((np.arange(len(p)), -p))
    g = set(g)
    if not forced <= g:
        return False
    for L in {m - 1, m, m + 1}:
        if cap is not None:
            L = min(L, cap)
        if L < 1 or L > len(p):
            continue
        want = set(int(j) for j in order[:L]) | forced
        p_cut = p[order[L - 1]]
        if all(abs(p[j] - p_cut) <= MASK_BAND for j in (g ^ want) - forced):
            return True
    return False


def compare_masks(gpu_rp, gpu_ci, info, nb, mode, mass_tau=0.0, cap=None, forced=None):
    """Returns (n_rows, n_identical, n_band, n_exempt); asserts the band rule."""
    check_csr_valid(gpu_rp, gpu_ci, nb)
    g_rows = csr_rows(gpu_rp, gpu_ci)
    o_rows = csr_rows(info.row_ptr, info.col_idx)
    assert len(g_rows) == len(o_rows)
    probs = info.probs.reshape(-1, nb)
    ident = band = exempt = 0
    for r, (g, o) in enumerate(zip(g_rows, o_rows)):
        if g == o:
            ident += 1
            continue
        if forced is not None:
            assert set(forced(r)) <= set(g), f"row {r}: forced blocks missing"
        if mode == 1 and (abs(info.mass_at_cut[r] - mass_tau) <= MASK_BAND or
                          abs(info.mass_before_cut[r] - mass_tau) <= MASK_BAND):
            if cap is not None:
                assert len(g) <= cap + len(set(forced(r)) if forced else 0)
            assert _is_near_prefix(g, probs[r], int(info.n_prefix[r]), cap,
                                   set(forced(r)) if forced else set()), \
                f"row {r}: not a prefix of the (p desc, j asc) order one block either side of the cut"
            exempt += 1
            continue
        diff = set(g) ^ set(o)
        p = probs[r]
        bad = [j for j in diff if abs(p[j] - info.p_thr[r]) > MASK_BAND]
        assert not bad, (f"row {r}: blocks {sorted(bad)} differ outside the band "
                         f"(p={[float(p[j]) for j in sorted(bad)]}, p_thr={info.p_thr[r]})")
        if mode == 0:
            assert len(g) == len(o), f"row {r}: top-k size differs"
        band += 1
    return len(g_rows), ident, band, exempt


def compare_attention(o_gpu, lse_gpu, o_ref, lse_ref, rows_mask=None):
    """o_*: [..., d] float arrays over the same token set; lse_*: [...]."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), empty), "empty-row pattern of LSE differs"
    assert np.all(o_gpu[empty] == 0.0), "empty rows must give O == 0"
    err = np.abs(o_gpu - o_ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.sqrt(np.mean(o_ref ** 2))) if o_ref.size else 0.0
    rel_rms = float(np.sqrt(np.mean(err ** 2)) / denom) if denom > 0 else float(np.sqrt(np.mean(err ** 2)))
    fin = ~empty
    lse_err = float(np.abs(lse_gpu[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    assert np.all(np.isfinite(o_gpu)), "non-finite O"
    assert max_abs <= O_MAX_ABS, f"O max-abs {max_abs:.3e} > {O_MAX_ABS}"
    assert rel_rms <= O_REL_RMS, f"O rel-RMS {rel_rms:.3e} > {O_REL_RMS}"
    assert lse_err <= LSE_ABS, f"LSE max-abs {lse_err:.3e} > {LSE_ABS}"
    return max_abs, rel_rms, lse_err


# ---- gradients -----------------------------------------------------------------
# dQ, dK, dV: rel-RMS <= 1e-2 and max|err| <= 2e-2 * max|ref| per gradient.  dQ
# gets one more term: the kernel takes D_t = dO_t . Ô_t from the bf16 Ô the
# forward returned, and an error dD_t in D moves dQ_t by scale * dD_t * k̄_t
# (k̄_t = sum_u P_tu k_u, the attention of q over the keys with V := K).
# Rounding O to bf16 has relative error at most u = 2^-8, independently per
# element, so dD_t is within three standard deviations of a sum of uniform
# terms: |dD_t| <= sqrt(3) * u * ||dO_t ∘ Ô_t||_2.  The dQ bounds add the RMS
# (and the max) of scale * that * |k̄_t| to the base ones.
GRAD_REL_RMS = 1e-2
GRAD_MAX_REL = 2e-2
BF16_U = 2.0 ** -8


def d_term(do, o_hat, kbar, scale):
    """Per-element size of the dQ error that D's rounding allows."""
    do = np.asarray(do, dtype=np.float64)
    o_hat = np.asarray(o_hat, dtype=np.float64)
    dd = np.sqrt(3.0) * BF16_U * np.sqrt(np.sum((do * o_hat) ** 2, axis=-1))
    return scale * dd[..., None] * np.abs(np.asarray(kbar, dtype=np.float64))


# Where the exact gradient is zero everywhere (every query row has a single live
# key, e.g. a one-token sequence), dS = P (dP - D) vanishes exactly because
# O_t = v_u, so dP_tu = dO_t . v_u = dO_t . O_t = D_t.  The kernels form dP on the
# tensor core and D in a separate pass, each an fp32 sum of d products in its own
# order, so their difference is rounding, not zero:
# * each sum is within 2 d 2^-23 sum_i |dO_ti x_i| of exact.  Products of bf16
#   values are exact in fp32; a tensor-core step adds 16 products and the
#   accumulator after aligning them, losing under 2^-23 of the largest addend
#   per addend (chopped, not rounded), i.e. at most (18 d / 16) 2^-23 sum|terms|
#   over d/16 steps; the separate pass rounds to nearest and is well inside it;
# * D is formed from the returned bf16 Ô; its exact effect, dO_t . (Ô_t - O_t),
#   is added as it is (zero when Ô = O, as for a single key);
# * dS = P (dP - D) is rounded to bf16, and dQ_t = scale sum_u dS_tu k_u,
#   dK_u = scale sum_t dS_tu q_t are fp32 sums rounded to bf16: a factor
#   (1 + 2^-6) covers those roundings and the few ulp of the recomputed P.
# dV needs no bound: it is zero only for keys no row reaches, which the kernels
# never touch.
FP32_CHOP = 2.0 ** -23


def zero_gradient_bounds(q, k, v, do, o_hat, o_ref, probs, scale):
    """Per-element bounds (dQ, dK, None) on the kernels' gradients where the exact
    ones are zero.  q, k, v, do, o_hat, o_ref: [B, H, N, d]; probs: the oracle's
    attention weights [B, H, N, N]."""
    q, k, v, do, o_hat, o_ref, probs = (np.asarray(x, dtype=np.float64)
                                        for x in (q, k, v, do, o_hat, o_ref, probs))
    d = q.shape[-1]
    gamma = 2.0 * d * FP32_CHOP
    s_dp = np.abs(do) @ np.swapaxes(np.abs(v), -1, -2)           # sum_i |dO_ti v_ui|
    s_d = np.sum(np.abs(do * o_hat), axis=-1)[..., None]          # sum_i |dO_ti Ô_ti|
    d_round = np.abs(np.sum(do * (o_hat - o_ref), axis=-1))[..., None]
    e = probs * (gamma * (s_dp + s_d) + d_round)                  # bound on |dS_tu|
    f = scale * (1.0 + 2.0 ** -6)
    return f * (e @ np.abs(k)), f * (np.swapaxes(e, -1, -2) @ np.abs(q)), None


def compare_gradients(got, ref, dq_term=None, zero_bounds=None):
    """got, ref: (dQ, dK, dV) arrays; dq_term: d_term(...) or None;
    zero_bounds: zero_gradient_bounds(...) or None (then a gradient that is
    exactly zero must come out exactly zero)."""
    out = []
    for idx, (name, g, w) in enumerate(zip(("dq", "dk", "dv"), got, ref)):
        g = np.asarray(g, dtype=np.float64)
        w = np.asarray(w, dtype=np.float64)
        assert np.all(np.isfinite(g)), f"{name}: non-finite"
        err = np.abs(g - w)
        wmax = float(np.abs(w).max()) if w.size else 0.0
        wrms = float(np.sqrt(np.mean(w ** 2))) if w.size else 0.0
        if wmax == 0.0:
            bound = zero_bounds[idx] if zero_bounds is not None else None
            if bound is None:
                assert float(err.max()) == 0.0, f"{name}: nonzero where the gradient is 0"
            else:
                worst = float(np.max(err - bound))
                assert worst <= 0.0, (f"{name}: |err| exceeds the rounding bound where the "
                                      f"gradient is 0 (max err {float(err.max()):.3e}, "
                                      f"max bound {float(np.max(bound)):.3e})")
            out.append((0.0, 0.0))
            continue
        extra_rms = extra_max = 0.0
        if idx == 0 and dq_term is not None:
            extra_rms = float(np.sqrt(np.mean(dq_term ** 2)))
            extra_max = float(dq_term.max())
        rms = float(np.sqrt(np.mean(err ** 2)))
        mx = float(err.max())
        assert rms <= GRAD_REL_RMS * wrms + extra_rms, \
            f"{name}: RMS err {rms:.3e} > {GRAD_REL_RMS} * {wrms:.3e} + {extra_rms:.3e}"
        assert mx <= GRAD_MAX_REL * wmax + extra_max, \
            f"{name}: max err {mx:.3e} > {GRAD_MAX_REL} * {wmax:.3e} + {extra_max:.3e}"
        out.append((rms / wrms, mx / wmax))
    return out
