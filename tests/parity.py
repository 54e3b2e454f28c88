"""Shared helpers of the GPU parity tests: tolerances and comparisons against the oracle.

Tolerances (bf16 activations, fp32 accumulation): hidden states within a relative L2 error of
2e-2 per layer, logits within max |delta| 0.1, and greedy ids identical wherever the oracle's
top-1 minus top-2 logit margin exceeds 0.05.
"""
import numpy as np
import torch

HIDDEN_REL_L2 = 2e-2
LOGIT_ABS = 0.1
GREEDY_MARGIN = 0.05


def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))


def hidden_errors(gpu_hidden: torch.Tensor, ref_hidden, rows=None):
    """Relative L2 error per layer (list over L+1 taps)."""
    g = gpu_hidden.float().cpu().numpy()
    out = []
    for li, ref in enumerate(ref_hidden):
        a = g[li] if rows is None else g[li][rows]
        b = ref if rows is None else ref[rows]
        out.append(rel_l2(a, b))
    return out


def assert_hidden(gpu_hidden, ref_hidden, rows=None, tol=HIDDEN_REL_L2, what=""):
    errs = hidden_errors(gpu_hidden, ref_hidden, rows)
    assert np.all(np.isfinite(errs)), (what, errs)
    assert max(errs) <= tol, (what, [f"{e:.2e}" for e in errs])
    return errs


def assert_logits(gpu_logits, ref_logits, gpu_argmax=None, what=""):
    g = np.asarray(gpu_logits.float().cpu().numpy() if isinstance(gpu_logits, torch.Tensor) else gpu_logits,
                   dtype=np.float64)
    r = np.asarray(ref_logits, dtype=np.float64)
    d = float(np.abs(g - r).max())
    assert np.isfinite(d) and d <= LOGIT_ABS, (what, d)
    if gpu_argmax is not None:
        r2 = np.atleast_2d(r)
        part = np.partition(r2, -2, axis=1)
        margin = part[:, -1] - part[:, -2]
        ids = np.atleast_1d(gpu_argmax.cpu().numpy() if isinstance(gpu_argmax, torch.Tensor) else gpu_argmax)
        ref_ids = np.argmax(r2, axis=1)
        for i in range(len(ids)):
            if margin[i] > GREEDY_MARGIN:
                assert ids[i] == ref_ids[i], (what, i, ids[i], ref_ids[i], margin[i])
    return d


def bf16_rows(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def f64_rows(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
