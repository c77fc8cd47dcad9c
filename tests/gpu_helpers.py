"""Shared helpers of the GPU parity tests: device copies of the seeded inputs,
the tolerances, and the comparison rules.

Tolerances (fp32 tensor-core arithmetic against the fp64 oracle):
  fused logit   |gpu - oracle| <= 2e-3 * sum_j |w_j * ReLU(q_j . k_s)| + 1e-5
  router score  |gpu - oracle| <= 2e-3 * |w| * sum_m ReLU(q . kbar_m) + 1e-5
                (= 2e-3 * |r_oracle| + 1e-5, since r = w * sum ReLU)
  head sets     must match wherever the oracle's gap between the h-th and the
                (h+1)-th router score exceeds the larger tolerance of the two
  top-k         bit-exact against the oracle's selection run on the GPU's own
                fp32 logits; set recall >= 0.999 against the oracle's fp64 logits
"""
import numpy as np
import torch

import oracle

LOGIT_RTOL = 2e-3
LOGIT_ATOL = 1e-5


def dev(a, dtype=None):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16))
    else:
        t = torch.from_numpy(a)
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def inputs_to_device(inp, fp8=False):
    out = {"Q": dev(inp["Q"]), "K": dev(inp["K"]), "w": dev(inp["w"])}
    if fp8:
        out["K8"] = dev(inp["K8"])
        out["k_scale"] = dev(inp["k_scale"])
    return out


def logit_magnitude(Qd, wd, Kd, heads, t, q_pos0):
    """sum_j |w_j * ReLU(q_j . k_s)| over the routed heads of local row t."""
    pos = q_pos0 + t
    hs = heads[t]
    dots = Qd[t, hs] @ Kd[:pos + 1].T                  # [h, pos+1]
    return (np.abs(wd[t, hs])[:, None] * np.maximum(dots, 0.0)).sum(axis=0)


def assert_logits_close(gpu_row, ora_row, mag, what=""):
    n = len(ora_row)
    diff = np.abs(gpu_row[:n].astype(np.float64) - ora_row)
    tol = LOGIT_RTOL * mag + LOGIT_ATOL
    bad = np.nonzero(diff > tol)[0]
    assert bad.size == 0, (f"{what}: {bad.size} logits outside tolerance, first at s={bad[0]}: "
                           f"gpu={gpu_row[bad[0]]!r} oracle={ora_row[bad[0]]!r} tol={tol[bad[0]]!r}")


def top_h(r_row, h):
    """h heads of largest score, ties to the lower index, ascending."""
    order = sorted(range(len(r_row)), key=lambda j: (-r_row[j], j))
    return sorted(order[:h])


def check_heads(gpu_heads, r_ora, heads_ora, h, r_gpu=None):
    """Head sets equal wherever the oracle's top-h gap exceeds the tolerance.
    Near-tie rows must still be valid: every GPU head scores within tolerance of
    the oracle's h-th score.  With the GPU's own scores, the selection must be
    bit-exact.  Returns the number of near-tie rows."""
    exempt = 0
    H = r_ora.shape[1]
    for t in range(r_ora.shape[0]):
        if r_gpu is not None:
            assert list(gpu_heads[t]) == top_h(r_gpu[t], h), f"row {t}: selection on own scores"
        if h == H:
            assert list(gpu_heads[t]) == list(range(H))
            continue
        order = sorted(range(H), key=lambda j: (-r_ora[t, j], j))
        a, b = order[h - 1], order[h]
        gap = r_ora[t, a] - r_ora[t, b]
        tol = max(LOGIT_RTOL * abs(r_ora[t, a]), LOGIT_RTOL * abs(r_ora[t, b])) + LOGIT_ATOL
        if gap > tol:
            assert list(gpu_heads[t]) == list(heads_ora[t]), (
                f"row {t}: gpu heads {list(gpu_heads[t])} oracle {list(heads_ora[t])} gap {gap}")
        else:
            exempt += 1
            for j in gpu_heads[t]:
                assert r_ora[t, j] >= r_ora[t, a] - tol, f"row {t}: head {j} is not a near-tie"
    return exempt


def recall(gpu_idx, ora_idx):
    tot, hit = 0, 0
    for g, o in zip(gpu_idx, ora_idx):
        og = set(int(x) for x in o if x >= 0)
        gg = set(int(x) for x in g if x >= 0)
        tot += len(og)
        hit += len(og & gg)
    return hit / max(tot, 1)
