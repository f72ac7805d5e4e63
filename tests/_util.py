"""Shared helpers of the GPU parity tests: moving the seeded numpy inputs to
the device, and the comparison rules (tolerances, near-tie exemption)."""
import numpy as np
import torch

# bf16 inputs, fp32 accumulation: max-abs / mean-abs bars on O and LSE
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
# fp32 path
F32_MAX_ABS = 1e-4
# top-k / retrieval near-tie exemption (relative gap of k-th and (k+1)-th)
TIE_REL = 1e-4


def to_dev(a, dtype=None, device="cuda"):
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    t = torch.from_numpy(a).to(device)
    return t if dtype is None else t.to(dtype)


def gather_rows(t, rows):
    """t [B,H,T,...] on device -> numpy float64 [n, ...] at rows (b, h, i)."""
    r = torch.from_numpy(np.ascontiguousarray(rows)).to(t.device)
    out = t[r[:, 0], r[:, 1], r[:, 2]]
    return out.float().cpu().numpy().astype(np.float64)


def compare(name, got, ref, max_abs, mean_abs=None):
    err = np.abs(got - ref)
    mx = float(np.nanmax(err)) if err.size else 0.0
    mn = float(np.nanmean(err)) if err.size else 0.0
    ok = np.isfinite(got).all() and mx <= max_abs and (mean_abs is None or mn <= mean_abs)
    msg = "%s: max-abs %.3e (bar %.1e), mean-abs %.3e%s" % (
        name, mx, max_abs, mn, "" if mean_abs is None else " (bar %.1e)" % mean_abs)
    print(msg)
    assert ok, msg
    return mx, mn


# oracle picks listed beyond the k-th, so that a near-tied run at the k-th
# position can be followed past it
TOPK_EXT = 4


def _near(a, b):
    return bool(np.isfinite(a) and np.isfinite(b) and abs(a - b) <= TIE_REL * max(abs(a), abs(b), 1e-30))


def topk_row_verdict(g, o, z, k):
    """One row: 'exact', 'exempt' or a reason string for a mismatch.

    g: the GPU's k picks; o, z: the oracle's first k + e picks (e >= 1) and
    their fp64 logits.  A row whose set differs from the oracle's passes only
    under the near-tie rule ("LM-Infinite", section 方法, optional top-k: the
    k largest logits; a fp32 selector may swap keys whose logits the fp32
    rounding cannot separate): the oracle's k-th and (k+1)-th logits are
    within TIE_REL relative, every oracle pick clearly above the k-th logit
    is in the GPU set, and every GPU pick is an oracle candidate whose logit
    is within TIE_REL of the k-th.  The GPU's list must also be ordered by
    the oracle's logits, up to swaps of near-equal pairs, and pad with -1
    exactly where the oracle does."""
    g = [int(x) for x in g]
    o = [int(x) for x in o]
    if g == o[:k]:
        return "exact"
    n_pad = sum(1 for x in o[:k] if x < 0)
    real = [x for x in g if x >= 0]
    if len(real) != k - n_pad or any(x >= 0 for x in g[k - n_pad:]):
        return "padding differs"
    if len(set(real)) != len(real):
        return "repeated key"
    zof = {o[x]: float(z[x]) for x in range(len(o)) if o[x] >= 0}
    if any(x not in zof for x in real):
        return "a GPU pick is not among the oracle's first %d" % len(o)
    ref = set(x for x in o[:k] if x >= 0)
    if set(real) != ref:
        zk = float(z[k - 1])
        if not (k < len(o) and _near(zk, float(z[k]))):
            return "set differs without a near tie at the k-th logit"
        strict = set(o[x] for x in range(k) if o[x] >= 0 and not _near(float(z[x]), zk))
        if not strict <= set(real):
            return "an oracle pick above the tied run is missing"
        if any(zof[x] < zk and not _near(zof[x], zk) for x in real):
            return "a GPU pick is below the tied run"
    for a, b in zip(real, real[1:]):
        if zof[a] < zof[b] and not _near(zof[a], zof[b]):
            return "order differs beyond a near tie"
    return "exempt"


def topk_agreement(gpu_idx, ref_idx_ext, ref_z_ext, k):
    """Rows of GPU selections [n, k] against the oracle's first k + e picks
    and logits [n, k + e]; see topk_row_verdict.  Returns (n_exact, n_exempt,
    bad) with bad a list of (row, reason)."""
    n_exact = n_exempt = 0
    bad = []
    for r in range(gpu_idx.shape[0]):
        v = topk_row_verdict(gpu_idx[r], ref_idx_ext[r], ref_z_ext[r], k)
        if v == "exact":
            n_exact += 1
        elif v == "exempt":
            n_exempt += 1
        else:
            bad.append((r, v))
    return n_exact, n_exempt, bad
