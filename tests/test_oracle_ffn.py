"""Pins for the oracle's feed-forward step: GELU between the up- and down-projection.

The note names no activation; the plain reading of the producer step of a
feed-forward block is GELU in its exact form, GELU(y) = y Phi(y) with Phi the
standard normal CDF.  Each check compares the oracle with something other than
its own formula: printed values of Phi, the odd-part identity, the saturation
limits, and Phi by numerical quadrature of the Gaussian density.
"""
import math

import numpy as np
import pytest

import oracle
import synth


def _phi_simpson(y, n=2000):
    """Phi(y) = 1/2 + int_0^y exp(-t^2/2) dt / sqrt(2 pi), composite Simpson over n intervals."""
    y = np.asarray(y, dtype=np.float64)
    t = np.linspace(0.0, 1.0, n + 1)[None, :] * y[..., None]
    f = np.exp(-0.5 * t * t)
    w = np.ones(n + 1)
    w[1:-1:2], w[2:-1:2] = 4.0, 2.0
    return 0.5 + (y / (3.0 * n)) * (f @ w) / math.sqrt(2.0 * math.pi)


@pytest.mark.parametrize("y,phi", [(0.0, 0.5), (1.0, 0.8413447460685429), (-1.0, 0.15865525393145707),
                                   (2.0, 0.9772498680518208), (-2.0, 0.022750131948179195),
                                   (3.0, 0.9986501019683699)])
def test_gelu_printed_normal_cdf_values(y, phi):
    # standard normal table values Phi(y): GELU(y) = y Phi(y)
    g = oracle.gelu_erf(np.array([y]))[0]
    assert abs(g - y * phi) <= 4e-16 * max(1.0, abs(y))


def test_gelu_odd_part_is_identity():
    # Phi(y) + Phi(-y) = 1, so GELU(y) - GELU(-y) = y
    y = np.random.default_rng(7).uniform(-9.0, 9.0, 4096)
    d = oracle.gelu_erf(y) - oracle.gelu_erf(-y)
    assert np.all(np.abs(d - y) <= 1e-15 * np.maximum(1.0, np.abs(y)))


def test_gelu_limits():
    g = oracle.gelu_erf(np.array([40.0, 1e3, -40.0, -1e3, 0.0, -0.0]))
    assert g[0] == 40.0 and g[1] == 1e3               # Phi = 1 in fp64
    assert abs(g[2]) < 1e-300 and g[3] == 0.0          # Phi underflows
    assert g[4] == 0.0 and g[5] == 0.0
    # the minimum of y Phi(y): where Phi(y) + y phi(y) = 0, y = -0.75179..., value -0.169971207...
    y = np.linspace(-6.0, 6.0, 12001)
    g = oracle.gelu_erf(y)
    assert abs(g.min() - (-0.1699712075)) < 2e-7
    assert abs(y[np.argmin(g)] - (-0.7518)) < 1e-3


def test_gelu_against_quadrature():
    y = np.array([-6.5, -3.0, -1.25, -0.5, -1e-3, 0.25, 0.75, 1.7, 3.0, 5.5])
    assert np.all(np.abs(oracle.gelu_erf(y) - y * _phi_simpson(y)) <= 1e-12 * np.maximum(1.0, np.abs(y)))


def test_ffn_hidden_rows_is_gelu_of_the_producer_rows():
    # composition of the two oracle steps on the tiny workload: the hidden rows are
    # y Phi(y) of the up-projection's Y rows, Phi by quadrature
    wl = synth.WORKLOADS["tiny"]
    X, Wb = synth.activations(wl), synth.weight(wl)
    L1, L2, _ = oracle.lowrank_factors(Wb, wl.rank)
    act = oracle.quantize_activations(X, wl.T, wl.H, wl.W, wl.cube)
    wq = oracle.quantize_weight(Wb, L1, L2)
    rows = np.arange(0, wl.N, 3)
    Y = oracle.output_rows(act, wq, X, L1, L2, rows)
    Hh = oracle.ffn_hidden_rows(act, wq, X, L1, L2, rows)
    assert Hh.shape == Y.shape
    assert np.all(np.abs(Hh - Y * _phi_simpson(Y)) <= 1e-12 * np.maximum(1.0, np.abs(Y)))
    # GELU is what separates them: equal where Y is far above zero, about 0 far below
    big, neg = Y > 6.0, Y < -6.0
    assert np.allclose(Hh[big], Y[big], rtol=1e-8)
    assert np.all(np.abs(Hh[neg]) < 1e-7)
