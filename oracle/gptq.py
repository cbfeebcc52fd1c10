"""GPTQ in FP64 -- TEST INFRASTRUCTURE ONLY (tests, smoke and the bench's CPU baseline use it;
the library never does).

Follows "4.3 Weight-only INT4", section 2 "GPTQ: quantize and compensate as you go":

- 2.1: the objective is the layer-output error ||X W - X W_hat||^2 over calibration inputs X,
  whose curvature is H = 2 X^T X (input channels x input channels).
- 2.2: the input channels are fixed one at a time, in order. After channel i is set to its
  dequantized value w_hat_i, the channels F still free move by
  dw_F = -(w_i - w_hat_i) / [H_F^-1]_ii * [H_F^-1]_{:,i}, and i leaves F.
- 2.2: damping is added to H for numerical stability (the amount is not given; read here as
  1% of the mean of diag(H), added to the diagonal).

Here W is [K, N] (K input channels, N output channels), so "weight column w" of the page is a
column W[:, n] and channel i is row i. Every output channel uses the same H, so one step updates
all N columns at once. The quantizer is the RTN group quantizer of the library format (FP16 scale
rounded once from the FP64 quotient, optional INT4 zero, round half to even), applied to a group
when its first channel comes up, on the group's current (already compensated) weights -- the
plainest reading, since the page fixes the error-feedback order but not when a group's scale is
taken. The page's own speed-ups (Cholesky factorisation, block updates) are not used: each step
is written exactly as stated, with an explicit inverse and its rank-1 removal of channel i.
"""
import numpy as np

from . import oracle as _o

DAMP = 0.01


def hessian(X):
    """H = 2 X^T X for calibration inputs X [S, K] (float64)."""
    X = np.asarray(X, dtype=np.float64)
    return 2.0 * (X.T @ X)


def damped(H, damp=DAMP):
    """H + damp * mean(diag H) * I."""
    H = np.array(H, dtype=np.float64, copy=True)
    H[np.diag_indices_from(H)] += damp * float(np.mean(np.diag(H)))
    return H


def rtn_params(Wg, sym):
    """Scale (fp16 bits and value) and zero of each column of one group's FP64 weights Wg [g, N]:
    the library's RTN reading. Degenerate groups (the scale rounds to 0) store s = 1, z = 0 and
    code 0 for every weight."""
    if sym:
        sbits = _o.encode16(np.max(np.abs(Wg), axis=0) / 7.0)
    else:
        lo = np.minimum(0.0, np.min(Wg, axis=0))
        hi = np.maximum(0.0, np.max(Wg, axis=0))
        sbits = _o.encode16((hi - lo) / 15.0)
    s = _o.decode16(sbits)
    degen = s == 0.0
    sbits = np.where(degen, np.uint16(0x3C00), sbits).astype(np.uint16)
    s = np.where(degen, 1.0, s)
    if sym:
        z = np.zeros(Wg.shape[1], dtype=np.int64)
    else:
        z = np.clip(np.rint(-lo / s), 0, 15).astype(np.int64)
        z = np.where(degen, 0, z)
    return sbits, s, z, degen


def rtn_codes(w, s, z, degen, sym):
    """Codes of one channel's weights w [N] with the group's parameters; and their dequantized
    values (q - z) * s (sym: q * s with q in -8..7)."""
    r = np.rint(w / s)
    if sym:
        q = np.clip(r, -8, 7).astype(np.int64)
        q = np.where(degen, 0, q)
        return q, q * s
    q = np.clip(r + z, 0, 15).astype(np.int64)
    q = np.where(degen, z, q)
    return q, (q - z) * s


def compensate(W, Hinv, i, w_hat):
    """Section 2.2, one step: channel i is fixed to w_hat (its row of W is set to it), the rows
    still free move by -(w_i - w_hat_i) / [H_F^-1]_ii * [H_F^-1]_{F,i}, and channel i is removed
    from the inverse: H_F'^-1 = H_F^-1 - [H_F^-1]_{:,i} [H_F^-1]_{i,:} / [H_F^-1]_ii. W and Hinv
    are updated in place; rows and columns < i of Hinv are no longer read."""
    d = Hinv[i, i]
    err = (W[i] - w_hat) / d
    W[i + 1:] -= np.outer(Hinv[i + 1:, i], err)
    W[i] = w_hat
    Hinv[i + 1:, i + 1:] -= np.outer(Hinv[i + 1:, i], Hinv[i, i + 1:]) / d
    return err


def gptq_values(W, H, group, sym):
    """The GPTQ sweep on FP64 weights W [K, N] with the (damped) H [K, K]. Returns the integer
    codes q [K, N] (sym: -8..7), the scale bits [K/g, N], the zeros [K/g, N] and the dequantized
    weights [K, N]."""
    W = np.array(W, dtype=np.float64, copy=True)
    K, N = W.shape
    G = K // group
    Hinv = np.linalg.inv(np.asarray(H, dtype=np.float64))
    q = np.zeros((K, N), dtype=np.int64)
    What = np.zeros((K, N), dtype=np.float64)
    sb = np.zeros((G, N), dtype=np.uint16)
    zz = np.zeros((G, N), dtype=np.int64)
    for i in range(K):
        if i % group == 0:
            g = i // group
            sb[g], s, zz[g], degen = rtn_params(W[i:i + group], sym)
        q[i], What[i] = rtn_codes(W[i], s, zz[g], degen, sym)
        compensate(W, Hinv, i, What[i])
    return q, sb, zz, What


def pack(q, sbits, z, sym):
    """Codes [K, N], scale bits [K/g, N], zeros [K/g, N] -> the plain packed format (codes int32
    [K/8, N] least significant nibble first; zeros int32 [K/g, N/8]; None when sym)."""
    K, N = q.shape
    u = (q & 0xF).astype(np.uint32).reshape(K // 8, 8, N)
    codes = np.zeros((K // 8, N), dtype=np.uint32)
    for i in range(8):
        codes |= u[:, i, :] << np.uint32(4 * i)
    zeros = None
    if not sym:
        zu = (z & 0xF).astype(np.uint32).reshape(z.shape[0], N // 8, 8)
        zeros = np.zeros((z.shape[0], N // 8), dtype=np.uint32)
        for i in range(8):
            zeros |= zu[:, :, i] << np.uint32(4 * i)
        zeros = zeros.view(np.int32)
    return codes.view(np.int32), np.ascontiguousarray(sbits, dtype=np.uint16), zeros


def gptq(W_bits, X_bits, x_dtype, group, sym, damp=DAMP):
    """GPTQ of an fp16 weight W [K, N] (uint16 bits) with 16-bit calibration inputs X [S, K]
    (bits of dtype x_dtype). Returns (codes, scales, zeros) in the plain packed format."""
    W = _o.decode16(W_bits, _o.F16)
    X = _o.decode16(X_bits, x_dtype)
    H = damped(hessian(X), damp)
    q, sb, zz, _ = gptq_values(W, H, group, sym)
    return pack(q, sb, zz, sym)


def output_error(X, W, What):
    """||X W - X W_hat||_F^2, the objective of section 2.1."""
    X = np.asarray(X, dtype=np.float64)
    D = X @ (np.asarray(W, dtype=np.float64) - np.asarray(What, dtype=np.float64))
    return float(np.sum(D * D))
