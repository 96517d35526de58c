"""CPU oracle for user-written cells: plain fp64 numpy, loops over time.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle/``): only ``tests/``
may import it; the product library never does, and the two share no code.

A cell is given as two Python functions on float64 arrays, vectorised over
the (b, d) channels:
    step(s, u, a) -> s'   s [NS, B, D] (state at l-1), u [G, B, D] (gates at
                          l), a [G, D] (recurrence weights) -> s' [NS, B, D]
    jac(s, u, a)  -> J    J [NS, NS, B, D], J[q, r] = d s'_q / d s_r
Follows the page "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares
e escala pra 7B parâmetros": "O compromisso que SSMs fizeram" (the recurrence
applied one step at a time) and "A sacada: método de Newton" (every Newton
iteration linearises each step around the current iterate and solves the
resulting linear recurrence), with the same readings as the C oracle: H^0 = 0,
residual r_k = max |F(H^k)| checked before each update, stop at r_k <= tol or
k = max_iters, delta form of the update.  Small cases only (pure-Python loop
over L).
"""
import numpy as np

OK = 0
NOT_CONVERGED = 1
NONFINITE = -5


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def _gates(u):
    """[B, L, G, D] -> [L, G, B, D]."""
    return np.ascontiguousarray(np.transpose(_f64(u), (1, 2, 0, 3)))


def generic_seq(step, u, a, s0, ns):
    """Sequential application s_l = step(s_{l-1}, u_l, a), l = 1..L, from
    s_0 = s0 ([NS, B, D], None = zeros).  Returns [NS, B, L, D]."""
    ug, a = _gates(u), _f64(a)
    L, G, B, D = ug.shape
    s = np.zeros((ns, B, D)) if s0 is None else _f64(s0).reshape(ns, B, D).copy()
    out = np.empty((ns, B, L, D))
    for l in range(L):
        s = step(s, ug[l], a)
        out[:, :, l] = s
    return out


def _prev(H, s0):
    """States entering each step: [s0, H_1, ..., H_{L-1}] along axis 2."""
    P = np.empty_like(H)
    P[:, :, 0] = s0
    P[:, :, 1:] = H[:, :, :-1]
    return P


def residual(step, ug, a, H, s0):
    """F_l = H_l - step(H_{l-1}, u_l) for every l: [NS, B, L, D]."""
    P = _prev(H, s0)
    F = np.empty_like(H)
    for l in range(H.shape[2]):
        F[:, :, l] = H[:, :, l] - step(P[:, :, l], ug[l], a)
    return F


def generic_bptt(step, u, a, s0, ds, ns):
    """Gradients of Loss = sum over l of <ds_l, s_l> for the sequential states
    s_l = step(s_{l-1}, u_l, a) (back-propagation through time), by torch
    autograd in float64; `step` takes the array module as xp=torch.  ds
    [NS, B, L, D].  Returns (du [B, L, G, D], da [G, D], ds0 [NS, B, D])."""
    import torch
    ug = torch.tensor(_gates(u), requires_grad=True)  # [L, G, B, D]
    at = torch.tensor(_f64(a), requires_grad=True)
    L, G, B, D = ug.shape
    s0t = torch.zeros((ns, B, D), dtype=torch.float64) if s0 is None else torch.tensor(_f64(s0).reshape(ns, B, D))
    s0t.requires_grad_(True)
    dst = torch.tensor(_f64(ds))
    s, loss = s0t, torch.zeros((), dtype=torch.float64)
    for l in range(L):
        s = step(s, ug[l], at, xp=torch)
        loss = loss + (dst[:, :, l] * s).sum()
    loss.backward()
    du = ug.grad.permute(2, 0, 1, 3).numpy()
    return du, at.grad.numpy(), s0t.grad.numpy()


def generic_newton(step, jac, u, a, s0, ns, tol=1e-6, max_iters=10):
    """Serial Newton.  Returns (H [NS, B, L, D], iters, residual, status,
    residual history)."""
    ug, a = _gates(u), _f64(a)
    L, G, B, D = ug.shape
    s0 = np.zeros((ns, B, D)) if s0 is None else _f64(s0).reshape(ns, B, D)
    H = np.zeros((ns, B, L, D))
    hist = []
    k = 0
    while True:
        F = residual(step, ug, a, H, s0)
        r = float(np.max(np.abs(F))) if F.size else 0.0
        hist.append(r)
        if not np.isfinite(r):
            return H, k, r, NONFINITE, hist
        if r <= tol or k == max_iters:
            return H, k, r, (OK if r <= tol else NOT_CONVERGED), hist
        # linear recurrence delta_l = J_l delta_{l-1} - F_l, delta_0 = 0, with
        # J_l the step's Jacobian at the current iterate's state H_{l-1}
        P = _prev(H, s0)
        delta = np.zeros((ns, B, D))
        for l in range(L):
            J = jac(P[:, :, l], ug[l], a)
            delta = np.einsum("qrbd,rbd->qbd", J, delta) - F[:, :, l]
            H[:, :, l] += delta
        k += 1
