"""Pins of the oracle's smooth switch s(r) and its reproducible cos(pi u).

The switch is the cosine taper of the "smooth" attention in the NeighborGraph
issue (Measurements: graph smooth / dense smooth), defined from r_on to rcut
(cosine from 5.5 to 6 A for the first benchmark system). The pins below use
only libm's cos (through Python's math module) and closed forms.
"""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.filterwarnings("ignore")


def test_cos_pi_matches_libm(oracle_mod):
    # absolute error within 2 ulp of 1.0 over the whole switching interval
    rng = np.random.default_rng(7)
    us = np.concatenate([rng.uniform(0.0, 1.0, 100_000), np.linspace(0.0, 1.0, 4097)])
    err = max(abs(oracle_mod.cos_pi(u) - math.cos(math.pi * u)) for u in us)
    assert err <= 4.5e-16, err


def test_cos_pi_special_values(oracle_mod):
    assert oracle_mod.cos_pi(0.0) == 1.0
    assert oracle_mod.cos_pi(1.0) == -1.0
    assert oracle_mod.cos_pi(0.5) == 0.0
    # cos(pi/3) = 1/2 and cos(2 pi/3) = -1/2 to within one ulp
    assert abs(oracle_mod.cos_pi(1.0 / 3.0) - 0.5) <= 2.3e-16
    assert abs(oracle_mod.cos_pi(2.0 / 3.0) + 0.5) <= 2.3e-16
    # odd symmetry about u = 1/2: cos(pi (1 - u)) = -cos(pi u)
    for u in (0.1, 0.25, 0.4, 0.49):
        assert abs(oracle_mod.cos_pi(1.0 - u) + oracle_mod.cos_pi(u)) <= 2.3e-16


def test_switch_shape(oracle_mod):
    rcut, r_on = 6.0, 5.5
    r = np.array([0.0, 1.0, 5.499999999, 5.5, 5.75, 6.0, 7.0])
    s = oracle_mod.switch(r, rcut, r_on)
    assert s[0] == 1.0 and s[1] == 1.0 and s[2] == 1.0
    assert s[3] == 1.0                 # s(r_on) = 1
    assert s[4] == 0.5                 # midpoint: cos(pi/2) = 0 exactly
    assert s[5] == 0.0 and s[6] == 0.0  # s(rcut) = 0 and beyond
    # closed form 0.5 (1 + cos(pi u)) against libm, and monotone decrease
    grid = np.linspace(r_on, rcut, 20001)
    sg = oracle_mod.switch(grid, rcut, r_on)
    ref = 0.5 * (1.0 + np.cos(np.pi * (grid - r_on) / (rcut - r_on)))
    assert np.max(np.abs(sg - ref)) <= 6e-16
    assert np.all(np.diff(sg) <= 0.0)
    # s(r_on + t) + s(rcut - t) = 1 (cosine antisymmetry about the midpoint)
    t = np.linspace(0.0, 0.25, 101)
    tot = oracle_mod.switch(r_on + t, rcut, r_on) + oracle_mod.switch(rcut - t, rcut, r_on)
    assert np.max(np.abs(tot[1:] - 1.0)) <= 1e-15
    # near rcut the taper is quadratic: s ~ (pi^2 / 4) ((rcut - r) / (rcut - r_on))^2
    eps = 1e-4
    approx = (math.pi ** 2 / 4.0) * (eps / (rcut - r_on)) ** 2
    assert abs(oracle_mod.switch([rcut - eps], rcut, r_on)[0] - approx) <= 1e-6 * approx
