"""Work accounting for the Kronecker layer: parameter count, algorithmic flops and bytes.

These are the figures a roofline divides by.  They count what the method must do,
not what a kernel happens to execute:

* multiply-adds per row and rank, vec trick with X.B first:  K1 = p*m1*m2 (T = X B_i)
  and K2 = p*q*m2 (Y = C_i^T T); with C first: K1' = q*p*m1 and K2' = q*m1*m2.
  The page "kronecker-layer-benchmark" (section "2. The vec trick") states the
  result as about r/m of a dense layer's multiply-adds.
* forward = r*min(K1+K2, K1'+K2') MACs per row; the backward needs twice that
  (dX and U share one contraction pair, dB and dC the other), so forward plus
  backward is 3x the forward, i.e. 6*r*min(...) flops per row.  Recomputing T in
  the backward is executed work, not credited.
* bytes per row, forward plus backward: read x, write y; read x and dY, write dX
  -> elt * (3*d_in + 2*d_out).  The factors (kilobytes) are not counted.

The Kronecker-sparse factor of pattern (a, b, c, d) (page "Fast Inference with
Kronecker-Sparse Matrices") has a*b*c*d non-zeros, a fraction 1/(a*d) of a dense
(a*b*d) x (a*c*d) matrix; its forward is one multiply-add per non-zero and row, and
the backward two more (dX and dw), so 6*a*b*c*d flops per row; bytes as above.
"""
from __future__ import annotations


def param_count(p, q, m1, m2, r, bias=True, with_s=True):
    """Trainable values of the layer: S (p x q), A (r x p x q), B (r x m1 x m2), bias."""
    n = r * p * q + r * m1 * m2
    if with_s:
        n += p * q
    if bias:
        n += q * m2
    return n


def dense_param_count(d_in, d_out, bias=True):
    return d_in * d_out + (d_out if bias else 0)


def macs_per_row_forward(p, q, m1, m2, r):
    k_xb = p * m1 * m2 + p * q * m2
    k_cx = q * p * m1 + q * m1 * m2
    return r * min(k_xb, k_cx)


def mac_ratio_vs_dense(p, q, m1, m2, r):
    return macs_per_row_forward(p, q, m1, m2, r) / float(p * m1 * q * m2)


def flops_per_row(p, q, m1, m2, r, backward=True, skip_fraction=None):
    """Algorithmic flops per row (forward, or forward + backward).

    ``skip_fraction``: fraction of (a, c) blocks of S that are non-zero when
    zero-block skipping is on; it scales the two contractions with C_i that
    produce y and U, while dC stays complete.
    """
    k1, k2 = p * m1 * m2, p * q * m2
    k1c, k2c = q * p * m1, q * m1 * m2
    if skip_fraction is None:
        fwd = r * min(k1 + k2, k1c + k2c)
        return 2 * (3 * fwd if backward else fwd)
    f = float(skip_fraction)
    fwd = r * (k1 + f * k2)
    if not backward:
        return 2 * fwd
    bwd = r * (f * k2 + k1) + r * (k1 + k2)  # U, dX ; dB, dC
    return 2 * (fwd + bwd)


def bytes_per_row(d_in, d_out, elt_bytes, backward=True):
    if backward:
        return elt_bytes * (3 * d_in + 2 * d_out)
    return elt_bytes * (d_in + d_out)


def ks_param_count(a, b, c, d, bias=True):
    """Values of a Kronecker-sparse factor of pattern (a, b, c, d) (+ bias)."""
    return a * b * c * d + (a * c * d if bias else 0)


def ks_flops_per_row(a, b, c, d, backward=True):
    """Algorithmic flops per row: 2 per non-zero for y, and as many again for dX and dw."""
    return 2 * a * b * c * d * (3 if backward else 1)
