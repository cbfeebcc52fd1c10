"""AWQ in FP64 -- TEST INFRASTRUCTURE ONLY (tests, smoke and the bench's CPU baseline use it;
the library never does).

Follows "4.3 Weight-only INT4", section 3 "AWQ: find channels to protect from activations":

- 3.1: how much a weight matters depends on the activation it multiplies, so salient input
  channels are found from the activation distribution.
- 3.2: instead of keeping them in FP16, the weights of input channel j are multiplied by s_j and
  the matching inputs divided by s_j: Y = (X S^-1)(S W), Y_hat = (X S^-1) D(Q(S W)), where Q
  gives the low-bit codes and D dequantizes with scale and zero. The scale factors are searched
  on calibration data and paired with clipping to control the total error; the deployed result
  is a regular INT4 layout plus the factors s (folded into whatever produces X).

Readings where the page leaves the procedure open (the plainest ones, stated once):

- activation statistic a_j = mean over the calibration rows of |x_j|;
- candidates s_j(alpha) = fp16(max(a_j, 2^-14) ^ alpha), alpha = 0, 1/20, ..., 19/20 (alpha = 0
  is plain RTN); the factor is rounded to fp16 because it is stored and applied as fp16;
- search objective: the layer-output error ||X W - (X S^-1) D(Q(S W))||_F^2 on the calibration
  rows, in FP64; the smallest wins, the first on ties;
- Q is the library's RTN group quantizer applied to the FP64 products s_j w_jn;
- clipping: for each group and output channel, the RTN range of the scaled weights is shrunk by
  r = 1, 0.95, ..., 0.5 (lo -> r lo, hi -> r hi; symmetric: amax -> r amax) and the r with the
  smallest output error of that group's weights, delta^T (X_g^T X_g) delta with
  delta = w - D(Q(s w)) / s, wins (the first on ties). r = 1 is plain RTN.
"""
import numpy as np

from . import oracle as _o

ALPHAS = [i / 20.0 for i in range(20)]
CLIPS = [1.0 - i / 20.0 for i in range(11)]
S_FLOOR = 2.0 ** -14


def act_stats(X):
    """a_j = mean_s |x_sj| (float64 [K])."""
    return np.mean(np.abs(np.asarray(X, dtype=np.float64)), axis=0)


def scale_candidate(a, alpha):
    """fp16 bits and values of s_j = fp16(max(a_j, 2^-14) ^ alpha)."""
    bits = _o.encode16(np.power(np.maximum(a, S_FLOOR), alpha))
    return bits, _o.decode16(bits)


def rtn_clipped(V, sym, r):
    """RTN of one group's FP64 values V [g, N] with the range shrunk by r (per column): returns
    the scale bits, scales, zeros, codes q [g, N] and the dequantized values (q - z) s."""
    if sym:
        sbits = _o.encode16(r * np.max(np.abs(V), axis=0) / 7.0)
    else:
        lo = r * np.minimum(0.0, np.min(V, axis=0))
        hi = r * np.maximum(0.0, np.max(V, axis=0))
        sbits = _o.encode16((hi - lo) / 15.0)
    s = _o.decode16(sbits)
    degen = s == 0.0
    sbits = np.where(degen, np.uint16(0x3C00), sbits).astype(np.uint16)
    s = np.where(degen, 1.0, s)
    if sym:
        z = np.zeros(V.shape[1], dtype=np.int64)
        q = np.clip(np.rint(V / s), -8, 7).astype(np.int64)
        q = np.where(degen, 0, q)
        return sbits, s, z, q, q * s
    z = np.clip(np.rint(-lo / s), 0, 15).astype(np.int64)
    z = np.where(degen, 0, z)
    q = np.clip(np.rint(V / s) + z, 0, 15).astype(np.int64)
    q = np.where(degen, z, q)
    return sbits, s, z, q, (q - z) * s


def quantize_scaled(W, s, group, sym, r=1.0):
    """RTN of S W (row k of W times s_k, in FP64) with clip ratio r for every group. Returns the
    codes [K, N], scale bits [K/g, N], zeros [K/g, N] and D(Q(S W)) [K, N]."""
    SW = np.asarray(W, dtype=np.float64) * s[:, None]
    K, N = SW.shape
    G = K // group
    q = np.zeros((K, N), dtype=np.int64)
    D = np.zeros((K, N))
    sb = np.zeros((G, N), dtype=np.uint16)
    zz = np.zeros((G, N), dtype=np.int64)
    for g in range(G):
        rows = slice(g * group, (g + 1) * group)
        sb[g], _, zz[g], q[rows], D[rows] = rtn_clipped(SW[rows], sym, r)
    return q, sb, zz, D


def output_error(X, W, s, D):
    """||X W - (X S^-1) D||_F^2 = ||X (W - S^-1 D)||_F^2 in FP64."""
    X = np.asarray(X, dtype=np.float64)
    E = X @ (np.asarray(W, dtype=np.float64) - D / s[:, None])
    return float(np.sum(E * E))


def search_scale(X, W, group, sym):
    """The alpha search: returns (index of the best alpha, the errors of every alpha)."""
    a = act_stats(X)
    errs = []
    for alpha in ALPHAS:
        _, s = scale_candidate(a, alpha)
        _, _, _, D = quantize_scaled(W, s, group, sym)
        errs.append(output_error(X, W, s, D))
    return int(np.argmin(errs)), errs


def search_clip(X, W, s, group, sym):
    """The clip search for fixed factors s: per group and output channel, the ratio in CLIPS whose
    weights give the smallest delta^T (X_g^T X_g) delta. Returns codes, scale bits, zeros, the
    chosen ratio indices [K/g, N] and the errors [len(CLIPS), K/g, N]."""
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    K, N = W.shape
    G = K // group
    errs = np.zeros((len(CLIPS), G, N))
    cand = []
    for ci, r in enumerate(CLIPS):
        q, sb, zz, D = quantize_scaled(W, s, group, sym, r)
        cand.append((q, sb, zz))
        delta = W - D / s[:, None]
        for g in range(G):
            rows = slice(g * group, (g + 1) * group)
            Hg = X[:, rows].T @ X[:, rows]
            dg = delta[rows]
            errs[ci, g] = np.einsum("an,ab,bn->n", dg, Hg, dg)
    best = np.argmin(errs, axis=0)   # [G, N], first on ties
    q = np.zeros((K, N), dtype=np.int64)
    sb = np.zeros((G, N), dtype=np.uint16)
    zz = np.zeros((G, N), dtype=np.int64)
    for g in range(G):
        rows = slice(g * group, (g + 1) * group)
        for ci in range(len(CLIPS)):
            m = best[g] == ci
            q[rows, m] = cand[ci][0][rows, m]
            sb[g, m] = cand[ci][1][g, m]
            zz[g, m] = cand[ci][2][g, m]
    return q, sb, zz, best, errs


def awq(W_bits, X_bits, x_dtype, group, sym):
    """AWQ of an fp16 weight W [K, N] with 16-bit calibration inputs X [S, K]. Returns the plain
    packed (codes, scales, zeros), the input factors s as fp16 bits [K], and the chosen alpha
    index."""
    from .gptq import pack
    W = _o.decode16(W_bits, _o.F16)
    X = _o.decode16(X_bits, x_dtype)
    ai, _ = search_scale(X, W, group, sym)
    sbits, s = scale_candidate(act_stats(X), ALPHAS[ai])
    q, sb, zz, _, _ = search_clip(X, W, s, group, sym)
    codes, scales, zeros = pack(q, sb, zz, sym)
    return codes, scales, zeros, sbits, ai
