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
- Downstream (compression and every layer): every compared row is checked
  twice.  Once end to end, on the GPU's own selection, for the rows whose
  list matches the oracle's exactly; and once with the GPU's compression and
  layers run on the ORACLE's selection (idx and w of the sampled rows
  replaced by the oracle's), for every row.  Values only ever flow from the
  oracle to the GPU side, never back.
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


def degenerate_rows(o_idx, o_scores):
    """Rows whose best selected score is <= 1e-30: their weights divide by the
    1e-30 floor, so the compressed values are meaningless (only reachable with
    the unidirectional ranker, whose first splits have one or no candidate)."""
    best = np.array([o_scores[r, o_idx[r, 0]] if o_idx[r, 0] >= 0 else 1.0
                     for r in range(o_idx.shape[0])])
    return best <= 1e-30


def oracle_selection(g_idx, g_w, sel, o_idx, o_w):
    """Copies of the GPU's selection tensors [B, n, k] (torch, on the device)
    whose rows of the sampled targets ``sel`` ((b, t) pairs) hold the
    oracle's idx / w instead; the other rows keep the GPU's, which no sampled
    row reads."""
    import torch
    idx = g_idx.clone()
    w = g_w.clone()
    sb = torch.from_numpy(np.asarray(sel[:, 0], dtype=np.int64)).to(idx.device)
    st = torch.from_numpy(np.asarray(sel[:, 1], dtype=np.int64)).to(idx.device)
    idx[sb, st] = torch.from_numpy(np.asarray(o_idx, dtype=np.int32)).to(idx.device)
    w[sb, st] = torch.from_numpy(np.asarray(o_w, dtype=np.float32)).to(idx.device)
    return idx, w
