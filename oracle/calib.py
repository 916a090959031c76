"""CPU oracle of the offline calibration steps -- TEST INFRASTRUCTURE.

Only the test suite and the benchmark's CPU-baseline leg may import this
module.  Plain numpy in float64 (integers for the index work); it shares
nothing with the CUDA library.

Sources (page title, section):

* Top-1 PCA: keep, per calibration sequence, the single token of largest
  L-infinity norm; the principal eigenvector of the covariance of those
  tokens; rotate so that this direction lands in the first channel --
  "OffQ: Taming Structured Outliers in LLM Quantization by Offsetting",
  Methodology 1;
* channels partitioned into groups of 128, sorted grouping preferred over
  zigzag -- same page, Methodology 3 and the ablation among the
  contributions;
* static per-channel flattening in the manner of SmoothQuant, folded into the
  adjacent weights -- "SERQ: Saliency-Aware Low-Rank Error Reconstruction for
  LLM Quantization", technical summary section 1;
* offline permutation of the weights, activations arriving permuted -- same
  page, section 3.

Readings where the pages leave a step open:

* "covariance of these tokens" is the uncentred second moment
  C = T^T T / S (centring would subtract the shared outlier direction itself
  when the extreme tokens all carry it);
* only the top eigenvector is computed (Top-1); the rotation that sends it to
  the first channel is completed to an orthogonal matrix by the Householder
  reflection Q = I - 2 w w^T / (w^T w), w = v' - e0, v' = +-v with v'[0] <= 0;
* the eigenvector's sign: its component of largest magnitude is positive
  (ties to the lower index);
* the sorting statistic of sorted grouping is the per-channel calibration
  max |x| after the rotation, in decreasing order, ties to the lower index
  (NaN as -infinity);
* flattening: s = xmax^alpha / wmax^(1-alpha), 1 where either is not
  positive; alpha is not given by the pages (SmoothQuant's 0.5 is the
  default the library's callers use).
"""
import numpy as np


def _f64(X):
    return np.asarray(X, dtype=np.float64)


def extreme_tokens(Xf32, S, L):
    """Per sequence s (rows s*L .. s*L+L-1): the token of largest max |x|
    (first on ties; NaN ignored by the maximum), and that token as float32.
    Xf32: [S*L, K] float32 (the inputs widened exactly)."""
    X = np.asarray(Xf32, np.float32).reshape(S, L, -1)
    tok = np.zeros(S, np.int32)
    for s in range(S):
        linf = np.fmax.reduce(np.abs(X[s]), axis=1, initial=0.0)
        tok[s] = int(np.argmax(linf))          # first maximum
    T = np.stack([X[s, tok[s]] for s in range(S)]).astype(np.float32)
    return tok, T


def sign_convention(v):
    """Flip v so that its component of largest magnitude (first on ties) is positive."""
    v = _f64(v)
    k = int(np.argmax(np.abs(v)))
    return v if v[k] >= 0 else -v


def top1_pca(T):
    """Principal eigenvector (unit length, sign_convention) and eigenvalue of
    C = T^T T / S, in float64.  A library SVD does the eigen step: the top
    right singular vector of T is the top eigenvector of T^T T, with
    eigenvalue sigma_1^2 (so lambda = sigma_1^2 / S), without forming the
    K x K matrix."""
    T = _f64(T)
    S = T.shape[0]
    _, sig, Vt = np.linalg.svd(T, full_matrices=False)
    v = sign_convention(Vt[0])
    return v / np.linalg.norm(v), float(sig[0] ** 2 / S)


def householder_w(v):
    """w = v' - e0 with v' = -v if v[0] > 0 else v."""
    v = _f64(v)
    vp = -v if v[0] > 0 else v.copy()
    w = vp.copy()
    w[0] -= 1.0
    return w


def householder_dense(v):
    """The dense reflection Q = I - 2 w w^T / (w^T w) (for pins on small K)."""
    w = householder_w(v)
    return np.eye(w.size) - 2.0 * np.outer(w, w) / (w @ w)


def householder_apply(X, v):
    """Y = X Q row by row, y = x - (2 (x . w) / (w . w)) w, in float64."""
    X = _f64(X)
    w = householder_w(v)
    c = 2.0 * (X @ w) / (w @ w)
    return X - np.outer(c, w)


def channel_absmax(Xf32):
    """amax[k] = max over rows |X[m, k]| (exact; NaN entries ignored; 0 for no rows)."""
    X = np.abs(np.asarray(Xf32, np.float32))
    return np.fmax.reduce(X, axis=0, initial=np.float32(0)).astype(np.float32)


def sorted_perm(stat):
    """perm[j] = channel at position j in decreasing stat (ties: lower index;
    NaN as -inf)."""
    key = np.where(np.isnan(stat), -np.inf, _f64(stat))
    idx = np.arange(key.size)
    return np.lexsort((idx, -key)).astype(np.int32)


def flatten_scales(xmax, wmax, alpha):
    """s[k] = xmax^alpha / wmax^(1-alpha) in float64; 1 where either is not positive."""
    xm, wm = _f64(xmax), _f64(wmax)
    ok = (xm > 0) & (wm > 0)
    s = np.ones_like(xm)
    s[ok] = xm[ok] ** alpha / wm[ok] ** (1.0 - alpha)
    return s


def permute_channels(Xf32, perm=None, s=None, op=0):
    """Y[:, j] = X[:, c], c = perm[j]; op 1 divides by s[c], op 2 multiplies,
    each a single operation on float32 values, evaluated in float64 and rounded
    once to float32 (exact for op 0; for ops 1 and 2 the float64 result rounded
    to float32 is the correctly rounded float32 result, since 53 >= 2*24 + 2)."""
    X = np.asarray(Xf32, np.float32)
    c = np.arange(X.shape[1]) if perm is None else np.asarray(perm)
    Y = _f64(X[:, c])
    if op == 1:
        Y = Y / _f64(np.asarray(s, np.float32)[c])
    elif op == 2:
        Y = Y * _f64(np.asarray(s, np.float32)[c])
    return Y.astype(np.float32)


def energy_in_first_channel(Y):
    """Fraction of the squared norm of rows Y held by channel 0 (reporting / pins)."""
    Y = _f64(Y)
    return float((Y[:, 0] ** 2).sum() / max((Y ** 2).sum(), 1e-300))
