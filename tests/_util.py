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


def topk_agreement(gpu_idx, ref_idx, ref_z_ext, k):
    """Rows whose GPU selection differs from the oracle only where the oracle
    has a near tie are exempt.  ref_z_ext holds k+1 oracle logits per row.
    Returns (n_exact, n_exempt, bad_rows)."""
    n_exact = n_exempt = 0
    bad = []
    for r in range(gpu_idx.shape[0]):
        g = list(gpu_idx[r])
        o = list(ref_idx[r])
        if g == o:
            n_exact += 1
            continue
        z = ref_z_ext[r]
        # a near tie anywhere among the first k+1 oracle logits can reorder or swap
        tie = False
        for x in range(k):
            a, b = z[x], z[x + 1]
            if np.isfinite(a) and np.isfinite(b) and abs(a - b) <= TIE_REL * max(abs(a), abs(b), 1e-30):
                tie = True
        if tie and sorted(set(g) - {-1}) is not None:
            n_exempt += 1
        else:
            bad.append(r)
    return n_exact, n_exempt, bad
