"""Gradients of the second-order masked forward, fp64, for the backward pass.

TEST INFRASTRUCTURE ONLY (see the package docstring).

"Higher-order Linear Attention" summary (gist.science 2510.27258), Metodología 4 and
Contribuciones 2: the scan reproduces the serial activations exactly, which the page offers as
the basis of exact parallel training; it prints no gradient.  The reference here is therefore
the plain one: reverse-mode differentiation (torch autograd, CPU, float64) of the masked-matrix
definitions, for a given output gradient dO: O = (L (.) (A A^T)) V for the second order and
O = A (A V) for AHLA (Metodología 2) and O = (M A) V, M = L (.) (A A^T), for the third order
(Metodología 3), with A = L (.) Q K^T.
"""
from __future__ import annotations

import numpy as np

from . import _f64


def hla2_forward_matrix(q, k, v):
    """The masked second-order output as torch float64 ops (differentiable)."""
    import torch
    T = q.shape[-2]
    L = torch.tril(torch.ones(T, T, dtype=torch.float64))
    A = L * (q @ k.transpose(-1, -2))
    W = L * (A @ A.transpose(-1, -2))
    return W @ v


def hla2_grads(q, k, v, do):
    """(dQ, dK, dV) of sum(O * dO) for O = hla2(q, k, v), fp64 numpy arrays of q's shape."""
    import torch
    tq, tk, tv = (torch.tensor(_f64(x), requires_grad=True) for x in (q, k, v))
    o = hla2_forward_matrix(tq, tk, tv)
    o.backward(torch.tensor(_f64(do)))
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


def hla2n_grads(q, k, v, do, eps: float = 1e-6):
    """(dQ, dK, dV) for the ratio-normalised output O = num / (den + eps), den the masked
    operator on a ones value column (Metodología 1, Normalización)."""
    import torch
    tq, tk, tv = (torch.tensor(_f64(x), requires_grad=True) for x in (q, k, v))
    num = hla2_forward_matrix(tq, tk, tv)
    den = hla2_forward_matrix(tq, tk, torch.ones(tv.shape[:-1] + (1,), dtype=torch.float64))
    o = num / (den + eps)
    o.backward(torch.tensor(_f64(do)))
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


def ahla_grads(q, k, v, do):
    """(dQ, dK, dV) for the AHLA output O = A (A V), A = L (.) Q K^T."""
    import torch
    tq, tk, tv = (torch.tensor(_f64(x), requires_grad=True) for x in (q, k, v))
    T = tq.shape[-2]
    L = torch.tril(torch.ones(T, T, dtype=torch.float64))
    A = L * (tq @ tk.transpose(-1, -2))
    o = A @ (A @ tv)
    o.backward(torch.tensor(_f64(do)))
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


def hla3_grads(q, k, v, do):
    """(dQ, dK, dV) for the third-order output O = (M A) V, M = L (.) (A A^T), A = L (.) Q K^T."""
    import torch
    tq, tk, tv = (torch.tensor(_f64(x), requires_grad=True) for x in (q, k, v))
    T = tq.shape[-2]
    L = torch.tril(torch.ones(T, T, dtype=torch.float64))
    A = L * (tq @ tk.transpose(-1, -2))
    M = L * (A @ A.transpose(-1, -2))
    o = (M @ A) @ tv
    o.backward(torch.tensor(_f64(do)))
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()
