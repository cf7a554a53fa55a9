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


def assert_q8_codes_exact(xn, xq, xd, rows, dim, name="xnorm"):
    """The Q8 codes and scales a kernel wrote equal, bit for bit, the oracle's Q8 of
    the kernel's own float32 normalised rows (identical float32 inputs: the
    distributed-llama Quantize step after RMSNorm, checked on the hot path)."""
    import oracle

    xn = np.asarray(xn, dtype=np.float32)[:rows * dim].reshape(rows, dim)
    q_ref, d_ref = oracle.q8_quantize(xn)
    q = np.asarray(xq)[:rows * dim].reshape(rows, dim)
    d = np.asarray(xd, dtype=np.float32)[:rows * (dim // 32)].reshape(rows, dim // 32)
    np.testing.assert_array_equal(q, q_ref, err_msg=f"{name}: Q8 codes")
    np.testing.assert_array_equal(d.view(np.uint32), np.asarray(d_ref, np.float32).view(np.uint32),
                                  err_msg=f"{name}: Q8 scales")
    print(f"[parity] {name}: Q8 codes and scales bit-exact ({rows} x {dim})")
