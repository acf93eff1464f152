"""fp64 oracle of the Muon update (test infrastructure only).

Every function takes and returns numpy arrays and computes in float64.  Inputs
that arrive in bf16 or fp32 are widened exactly (every bf16/fp32 value is an
fp64 value), so the oracle sees the same numbers as the GPU path.

Citations name the page title and the passage:

* [Guide §Optimizer] "NanoGPT Speedrun: The Ultimate Guide to Pushing LLM
  Training Efficiency to Its Limits", section "Optimizer and Training Strategy
  Tuning" (Muon paragraph).
* [Overview ¶Six records] "The NanoGPT speedrun", paragraph "Six records
  account for most of the speedup" (record #3).
* [Overview ¶Reading guide] the same page, paragraph "Reading guide": later
  refinements tune the same update, among them Polar Express polynomials
  (per-step coefficients; none are printed on the pages), NorMuon's
  per-neuron rescale and cautious weight decay (no formulas on the pages;
  the readings are stated at ``normuon_rescale`` and ``cautious_mask``).
"""
from __future__ import annotations

import math

import numpy as np

#: Coefficients (a, b, c) of the quintic X <- aX + (bA + cA^2)X.  The pages
#: give only the step count; the form and the triple are the library's
#: specification.
NS_COEFFS = (3.4445, -4.7750, 2.0315)

#: Steps T of the iteration: "five Newton-Schulz steps" [Overview ¶Six records].
NS_STEPS = 5

#: Guard added to the Frobenius norm.  Reading: the pages give no epsilon; a
#: small additive guard only changes an all-zero input (whose output is zero).
NORM_EPS = 1e-7


def frobenius_normalize(X, eps=NORM_EPS):
    """X / (||X||_F + eps), in fp64.

    The pages say only that the update is brought to its nearest
    semi-orthogonal matrix [Overview ¶Six records]; Newton-Schulz needs the
    singular values inside the quintic's basin (0, 1.26), which Frobenius
    normalisation guarantees (sigma_max <= ||X||_F).
    """
    X = np.asarray(X, dtype=np.float64)
    return X / (np.sqrt(np.sum(X * X)) + eps)


def newton_schulz(G, steps=NS_STEPS, coeffs=NS_COEFFS, eps=NORM_EPS, schedule=None):
    """Newton-Schulz orthogonalisation of one matrix, fp64.

    Follows, in order: transpose so that rows <= cols (a view choice; undone
    at the end), Frobenius-normalise, then ``steps`` times
    A = X X^T, B = bA + c A A, X = aX + B X [Overview ¶Six records: "five
    Newton-Schulz steps"; Guide §Optimizer: orthogonalisation by
    Newton-Schulz iteration].  Square matrices are not transposed.

    ``schedule``: optional list of (a, b, c) triples, one per step, in the
    order applied (the per-step polynomials the Overview's ¶Reading guide
    names as Polar Express; the pages give no coefficients).  When given it
    replaces ``steps`` and ``coeffs``.
    """
    if schedule is None:
        schedule = [coeffs] * steps
    X = np.asarray(G, dtype=np.float64)
    if X.ndim != 2:
        raise ValueError("newton_schulz expects one 2-D matrix")
    transposed = X.shape[0] > X.shape[1]
    if transposed:
        X = X.T
    X = frobenius_normalize(X, eps)
    for triple in schedule:
        a, b, c = (float(v) for v in triple)
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    if transposed:
        X = X.T
    return np.ascontiguousarray(X)


def newton_schulz_batch(Gs, steps=NS_STEPS, coeffs=NS_COEFFS, eps=NORM_EPS):
    """``newton_schulz`` applied to each matrix of a list (independent units)."""
    return [newton_schulz(G, steps, coeffs, eps) for G in Gs]


def momentum(grad, buf, beta, nesterov=True):
    """Momentum buffer update and the vector that is orthogonalised, fp64.

    Reading of "Nesterov momentum" [Guide §Optimizer], which gives no formula:
    the lerp form  buf' = beta*buf + (1-beta)*g  and, with Nesterov,
    u = (1-beta)*g + beta*buf'  (otherwise u = buf').  Returns (buf', u).
    """
    g = np.asarray(grad, dtype=np.float64)
    m = np.asarray(buf, dtype=np.float64)
    beta = float(beta)
    new_buf = beta * m + (1.0 - beta) * g
    u = (1.0 - beta) * g + beta * new_buf if nesterov else new_buf
    return new_buf, u


def update_scale(rows, cols):
    """Post-orthogonalisation scale sqrt(max(1, rows/cols)).

    Reading of "then scaled and applied": the pages give no scale, so a fixed
    shape rule is used; it makes the update's RMS independent of the aspect
    ratio for tall matrices and is 1 for square and wide ones.
    """
    return math.sqrt(max(1.0, rows / cols))


#: NorMuon's second-moment coefficient and the guard inside its 1/sqrt
#: (reading; the pages give neither).
NORMUON_BETA2 = 0.95
NORMUON_EPS = 1e-10


def cautious_mask(W, O):
    """Cautious weight decay's mask [Overview ¶Reading guide], fp64.

    Reading: decay acts only where it pushes the same way as the update, i.e.
    where the weight and the update O (which is subtracted) have the same
    sign, W*O > 0.  Elements where either is zero are not decayed.
    """
    W = np.asarray(W, dtype=np.float64)
    O = np.asarray(O, dtype=np.float64)
    return (W * O > 0).astype(np.float64)


def apply_update(W, O, lr, wd, scale, cautious=False):
    """W' = W - lr*wd*W - lr*scale*O (decoupled weight decay from the pre-update W).

    With ``cautious`` the decay term is multiplied by ``cautious_mask(W, O)``.
    """
    W = np.asarray(W, dtype=np.float64)
    O = np.asarray(O, dtype=np.float64)
    decay = lr * wd * W
    if cautious:
        decay = decay * cautious_mask(W, O)
    return W - decay - lr * scale * O


def normuon_rescale(O, v, beta2=NORMUON_BETA2, eps=NORMUON_EPS):
    """NorMuon's per-neuron rescale of the orthogonalised update [Overview ¶Reading guide], fp64.

    Reading (the pages name it and give no formula): a neuron is a row of W
    in the caller's layout.  Each row keeps an exponential moving average of
    its update's mean square, and the update's rows are divided by the root
    of that average (an Adam-like second moment per neuron); the result is
    scaled back to the Frobenius norm of O, so the rescale only changes how
    the update is split over the neurons, not its size:

        r_i  = mean_j O_ij^2
        v'_i = beta2 v_i + (1 - beta2) r_i
        D    = diag(1 / sqrt(v' + eps))
        O'   = (||O||_F / ||D O||_F) D O        (O' = D O when ||D O||_F = 0)

    Returns (O', v').
    """
    O = np.asarray(O, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    r = np.mean(O * O, axis=1)
    v_new = beta2 * v + (1.0 - beta2) * r
    DO = O / np.sqrt(v_new + eps)[:, None]
    n_do = np.linalg.norm(DO)
    g = np.linalg.norm(O) / n_do if n_do > 0 else 1.0
    return g * DO, v_new


def muon_step(W, grad, buf, beta=0.95, nesterov=True, lr=0.05, wd=0.0,
              steps=NS_STEPS, coeffs=NS_COEFFS, eps=NORM_EPS):
    """One Muon step for one hidden matrix, fp64.

    Momentum -> orthogonalise (``newton_schulz``) -> scale and apply
    [Guide §Optimizer; Overview ¶Six records].  Returns (W', buf', O).
    """
    new_buf, u = momentum(grad, buf, beta, nesterov)
    O = newton_schulz(u, steps, coeffs, eps)
    r, s = O.shape
    W_new = apply_update(W, O, lr, wd, update_scale(r, s))
    return W_new, new_buf, O


def muon_step_ex(W, grad, buf, beta=0.95, nesterov=True, lr=0.05, wd=0.0, steps=NS_STEPS,
                 coeffs=NS_COEFFS, eps=NORM_EPS, cautious=False, neuron_state=None,
                 beta2=NORMUON_BETA2, schedule=None):
    """``muon_step`` with the refinements of [Overview ¶Reading guide], fp64.

    Momentum -> orthogonalise (per-step triples when ``schedule`` is given,
    the Polar Express reading of ``newton_schulz``) -> (NorMuon rescale when
    ``neuron_state`` is given) -> scale and apply (cautious decay when
    ``cautious``).  Returns (W', buf', O', v') with O' the update applied and
    v' the new state (None without NorMuon).
    """
    new_buf, u = momentum(grad, buf, beta, nesterov)
    O = newton_schulz(u, steps, coeffs, eps, schedule=schedule)
    v_new = None
    if neuron_state is not None:
        O, v_new = normuon_rescale(O, neuron_state, beta2)
    r, s = O.shape
    W_new = apply_update(W, O, lr, wd, update_scale(r, s), cautious=cautious)
    return W_new, new_buf, O, v_new


def ns_flops(rows, cols, steps=NS_STEPS):
    """Nominal FLOPs of the iteration: steps * (4 m^2 n + 2 m^3), m = min, n = max.

    Per step: X X^T is 2 m^2 n, A A is 2 m^3, B X is 2 m^2 n.
    """
    m, n = min(rows, cols), max(rows, cols)
    return steps * (4 * m * m * n + 2 * m ** 3)


def quintic(sigma, coeffs=NS_COEFFS):
    """The scalar map the iteration applies to each singular value: a s + b s^3 + c s^5."""
    a, b, c = coeffs
    return a * sigma + b * sigma ** 3 + c * sigma ** 5
