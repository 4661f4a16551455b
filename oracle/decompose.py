"""Spectral split M = U S V^T + M_R by randomized low-rank decomposition.

Source: "Metis: Training LLMs with FP4 Quantization" (papernotes.org notes):
* 关键设计 1 -- every matrix of a GeMM is split into a rank-k dominant part
  U_k S_k V_k^T kept in high precision plus a residual M_R that is quantized;
* 关键设计 2 -- the dominant subspace is estimated from l_k << l randomly
  sampled rows, and a Gaussian test matrix Omega projects the hidden dimension
  to k + s before a small SVD recovers the subspace;
* 关键设计 3 -- the low-rank factors are reused across steps and the
  decomposition is refreshed every 8 steps (训练策略: rank 1.5%, refresh 8).

Steps (readings R7, R8, R10, R12 of the pages):

refresh_basis (every R steps):
  1. sample l_k distinct rows: each row i gets the Philox word (i & 3) of
     counter i >> 2 on the SAMPLE stream; the l_k smallest (word, i) pairs
     are taken and the indices sorted ascending (uniform without
     replacement).  l_k == rows keeps every row (used for W).
  2. Omega (c x (k+s)), element e = i*(k+s) + j: the words (w0,w1,w2,w3) of
     OMEGA counter t give elements 4t, 4t+1 from (w0, w1) and 4t+2, 4t+3
     from (w2, w3) by Box-Muller in fp64: u1 = (a+1) 2^-32, u2 = b 2^-32,
     z = sqrt(-2 ln u1) (cos 2 pi u2, sin 2 pi u2), each rounded to fp32.
  3. Y = M_s Omega;  (Q, R) = CholQR(Y);  Bm = Q^T M_s   ((k+s) x c)
  4. (Q2, R2) = CholQR(Bm^T);  one-sided Jacobi SVD of R2^T = U' Sigma W'^T
  5. V_k = Q2 W'[:, :k]   (right singular vectors of Bm, sigma descending)

step_factors (every step, on the current M and the reused basis V):
  6. P = M V;  (Q_P, R_P) = CholQR(P);  R_P = U_r S_r V_r^T (Jacobi)
  7. U = Q_P U_r,  S = S_r,  V <- V V_r, then each column pair (U_j, V_j) is
     sign-fixed so the largest-magnitude entry of V_j is positive (first
     index on ties).  Hence U S V^T = P V^T = M V V^T: the projection of M
     onto the reused subspace.

residual (关键设计 1, reading R6): M_R = M - U S V^T in fp64 from the
unquantized factors, rounded to fp32.

Pins (tests/test_oracle_decompose.py): sampling is a uniform permutation
prefix (frequency test) with distinct sorted indices; Omega moments; exact
recovery of a planted rank-k subspace against numpy.linalg.svd; the split is
exact (U S V^T + M_R == M); the residual spectrum of the tiny workload keeps
exactly the two spikes beyond rank 4 and is flat (below the bulk edge) once
k covers all spikes.
"""

import numpy as np

from . import linalg, philox


def sample_rows(rows, l_k, seed, operand_id, step):
    if not (1 <= l_k <= rows):
        raise ValueError("need 1 <= l_k <= rows")
    if l_k == rows:
        return np.arange(rows, dtype=np.int64)
    words = philox.element_words(seed, philox.tag(operand_id, philox.PURPOSE_SAMPLE), step, rows)
    order = np.lexsort((np.arange(rows), words))   # by word, then by index
    return np.sort(order[:l_k]).astype(np.int64)


def box_muller(a, b):
    """Two N(0,1) draws (fp64) from two 32-bit words a, b (arrays of equal shape).

    u1 = (a + 1) 2^-32 lies in (0, 1], so the logarithm is finite for every word
    (a = 0xffffffff gives u1 = 1 and radius 0); u2 = b 2^-32 lies in [0, 1).
    """
    u1 = (np.asarray(a, dtype=np.float64) + 1.0) * 2.0 ** -32
    u2 = np.asarray(b, dtype=np.float64) * 2.0 ** -32
    rad = np.sqrt(-2.0 * np.log(u1))
    return rad * np.cos(2.0 * np.pi * u2), rad * np.sin(2.0 * np.pi * u2)


def omega(cols, width, seed, operand_id, step):
    n = cols * width
    ncalls = (n + 3) // 4
    w = philox.stream_words(seed, philox.tag(operand_id, philox.PURPOSE_OMEGA), step,
                            np.arange(ncalls, dtype=np.uint64))
    out = np.empty(ncalls * 4, dtype=np.float64)
    for first, second, dst in ((0, 1, 0), (2, 3, 2)):
        out[dst::4], out[dst + 1::4] = box_muller(w[:, first], w[:, second])
    return out[:n].astype(np.float32).reshape(cols, width)


def refresh_basis(M, k, s, l_k, seed, operand_id, step):
    """Returns dict(V=c x k basis, rows=sampled indices, omega=Omega, sigma=sketch spectrum)."""
    M = np.asarray(M, dtype=np.float64)
    r, c = M.shape
    width = k + s
    if not (1 <= k and width <= min(l_k, c)):
        raise ValueError("need 1 <= k and k + s <= min(l_k, cols)")
    idx = sample_rows(r, l_k, seed, operand_id, step)
    Om = omega(c, width, seed, operand_id, step)
    Ms = M[idx, :]
    Y = Ms @ Om.astype(np.float64)
    Q, _, _ = linalg.cholqr(Y)
    Bm = Q.T @ Ms
    Q2, R2, _ = linalg.cholqr(Bm.T)
    _, sig, Wp = linalg.jacobi_svd(R2.T)
    V = Q2 @ Wp[:, :k]
    return {"V": V, "rows": idx, "omega": Om, "sigma": sig}


def sign_fix(U, V):
    """Flip column pairs so the largest-|.| entry of each V column is positive."""
    U = U.copy()
    V = V.copy()
    for j in range(V.shape[1]):
        i = int(np.argmax(np.abs(V[:, j])))
        if V[i, j] < 0:
            V[:, j] = -V[:, j]
            U[:, j] = -U[:, j]
    return U, V


def step_factors(M, V):
    """Per-step factors on the reused basis V (c x k): returns (U, S, V_new)."""
    M = np.asarray(M, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    P = M @ V
    QP, RP, _ = linalg.cholqr(P)
    Ur, Sr, Vr = linalg.jacobi_svd(RP)
    U = QP @ Ur
    Vn = V @ Vr
    U, Vn = sign_fix(U, Vn)
    return U, Sr, Vn


def residual(M, U, S, V):
    """M_R = M - U diag(S) V^T evaluated in fp64, rounded to fp32."""
    M = np.asarray(M, dtype=np.float64)
    low = (np.asarray(U, dtype=np.float64) * np.asarray(S, dtype=np.float64)[None, :]) @ \
        np.asarray(V, dtype=np.float64).T
    return (M - low).astype(np.float32)
