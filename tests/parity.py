"""Comparison rules shared by the GPU-vs-oracle parity tests.

- Floats: max_i |g_i - o_i| / max(|o_i|, rms(o)) <= tol, with tol = 1e-2 for
  the bf16 tensor-core path and 1e-4 for the fp32 path (elementwise relative
  error, floored at the tensor's RMS so entries that cancel to ~0 do not
  dominate).
- Top-k: the ordered index lists must match exactly, except that at a rank
  where they differ the two splits' oracle scores must be within 1e-3
  relative (a near tie); the GPU list must never contain the target itself
  or a repeated split, and its top-1 weight must be exactly 1 (unless the
  best score is <= 0, where the weights divide by the 1e-30 floor).
"""
import numpy as np

TOL = {"bf16": 1e-2, "f32": 1e-4}
TIE = 1e-3


def rel_err(g, o) -> float:
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    assert g.shape == o.shape, (g.shape, o.shape)
    if o.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(o * o)))
    den = np.maximum(np.abs(o), rms if rms > 0 else 1.0)
    return float(np.max(np.abs(g - o) / den))


def check_topk(g_idx, g_w, o_idx, o_scores, targets, tol_w):
    """Returns the boolean mask of rows whose lists match exactly.

    g_idx, g_w: GPU [rows, k]; o_idx: oracle [rows, k]; o_scores: oracle
    scores [rows, n] (fp64); targets: target split of each row.
    """
    rows, k = g_idx.shape
    exact = np.ones(rows, dtype=bool)
    for r in range(rows):
        gi, oi = g_idx[r], o_idx[r]
        valid = gi[gi >= 0]
        assert targets[r] not in valid, f"row {r}: selected itself"
        assert len(set(valid.tolist())) == len(valid), f"row {r}: repeated split"
        assert np.array_equal(gi < 0, oi < 0), f"row {r}: padding differs"
        if valid.size and o_scores[r, gi[0]] > 1e-30:
            # w_1 = s_1 / s_1; when s_1 <= 0 the weights divide by the 1e-30 floor
            assert g_w[r, 0] == 1.0, f"row {r}: top-1 weight {g_w[r, 0]!r} != 1"
        if not np.array_equal(gi, oi):
            exact[r] = False
            for j in range(k):
                if gi[j] != oi[j] and oi[j] >= 0:
                    a, b = o_scores[r, gi[j]], o_scores[r, oi[j]]
                    assert abs(a - b) <= TIE * abs(b), (
                        f"row {r} rank {j}: GPU chose {gi[j]} (oracle score {a}), oracle {oi[j]} ({b})")
        # weights against the oracle's scores of the GPU's own choices
        sel = gi[gi >= 0]
        if sel.size:
            s = o_scores[r, sel]
            ref = s / max(s[0], 1e-30)
            assert rel_err(g_w[r, :sel.size], ref) <= tol_w, f"row {r}: weights"
    return exact
