"""Error metrics for parity tests (max relative error and Pearson correlation).

The tt-metal Llama-2 thread asserts on the Pearson correlation coefficient of
each submodule against a golden model; the parity bar used here is
``max|y - y_ref| / max|y_ref|`` (2e-2 for bf16-weight paths), with PCC reported.
"""
import numpy as np

BF16_TOL = 2e-2


def max_rel(y, ref) -> float:
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.max(np.abs(ref))
    if scale == 0:
        return float(np.max(np.abs(y)))
    return float(np.max(np.abs(y - ref)) / scale)


def pcc(y, ref) -> float:
    y = np.asarray(y, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    if y.size < 2 or np.std(y) == 0 or np.std(ref) == 0:
        return 1.0 if np.allclose(y, ref) else 0.0
    return float(np.corrcoef(y, ref)[0, 1])


def report(name, y, ref):
    r, p = max_rel(y, ref), pcc(y, ref)
    print(f"[parity] {name}: max_rel={r:.3e} pcc={p:.8f}")
    return r, p
