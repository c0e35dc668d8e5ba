"""Helpers shared by the GPU parity tests: conversions and the acceptance rule."""
import json
import os

import numpy as np
import torch

import oracle as O


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def store_of(dtype):
    return "bf16" if dtype == torch.bfloat16 else "f32"


def bf16_ulps_above_rms(got, want):
    """Largest distance, in bf16 units in the last place, between a bf16 result and the oracle
    value rounded to bf16, over the elements whose oracle value exceeds the tensor's RMS (0 if
    there are none). 0 means the correctly rounded result; 1, the neighbour of it. One bf16 ulp
    at x is 2^(e - 7) with 2^e <= |x| < 2^(e + 1), the spacing of the 8-bit significand."""
    rms = float(np.sqrt(np.mean(want ** 2)))
    big = np.abs(want) > rms
    if not big.any():
        return 0.0
    w = torch.from_numpy(want[big]).to(torch.bfloat16).double().numpy()
    ulp = np.ldexp(1.0, np.frexp(np.abs(w))[1] - 8)  # frexp: |w| = m 2^e with m in [0.5, 1)
    return float((np.abs(got[big] - w) / ulp).max())


def assert_close(got, want, dtype, what="", mode="scaled"):
    """The acceptance rule.

    mode "literal": absolute error, for O on unit-variance workloads.
    mode "scaled": each error divided by max(|oracle element|, RMS of the oracle tensor), for
    gradients and for row-scaled workloads (heavy-tailed tensors).
    bf16: max <= 2e-2 and mean <= 2e-3; fp32: max <= 1e-4.
    """
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    if got.size == 0:
        return 0.0, 0.0
    err = np.abs(got - want)
    if mode == "scaled":
        rms = float(np.sqrt(np.mean(want ** 2))) or 1.0
        err = err / np.maximum(np.abs(want), rms)
    mx, mean = float(err.max()), float(err.mean())
    msg = f"{what} ({mode}): max {mx:.3g} mean {mean:.3g}"
    log = os.environ.get("LH_ACCEPT_LOG")
    if log:  # measurement of the margins, for choosing bounds; no effect on pass or fail
        with open(log, "a") as f:
            f.write(json.dumps({"test": os.environ.get("PYTEST_CURRENT_TEST", ""), "what": what,
                                "mode": mode, "dtype": str(dtype), "max": mx, "mean": mean,
                                "ulps_above_rms": bf16_ulps_above_rms(got, want)}) + "\n")
    if dtype == torch.bfloat16:
        assert mx <= 2e-2 and mean <= 2e-3, msg
        if is_bf16_valued(got):  # a result stored in bf16 (not an fp32 intermediate)
            bound = ulp_bound(what)
            ulps = bf16_ulps_above_rms(got, want)
            assert ulps <= bound, f"{what}: {ulps:.2f} bf16 ulps from the rounded oracle (bound {bound})"
    else:
        assert mx <= 1e-4, msg
    return mx, mean


def is_bf16_valued(x):
    x = np.asarray(x, np.float64)
    return bool(np.array_equal(torch.from_numpy(x).to(torch.bfloat16).double().numpy(), x))


def ulp_bound(what):
    """Largest distance in bf16 ulps, for elements above the RMS, between a bf16 layer output and
    the correctly rounded oracle value: 1 (the rounded value or its neighbour) for O, dK and dV;
    2 for dQ, whose fp32 sums arrive by atomic adds in an order that varies from run to run."""
    return 2 if what.lower().startswith("dq") else 1


def assert_pyramid(got, x, geo, dtype, what="pyramid"):
    """Pooled cells against the exact span means, within a derived forward-error bound.

    The GPU adds p children per level in fp32 (at most (p-1)(L-1) additions deep, each with
    relative error 2^-24 of the running sum of |x|), scales by 1/p^l once, and rounds once to
    the storage type (half an ulp: at most 2^-8 relative for bf16, 2^-24 for fp32).
    """
    want = O.build_pyramid(x, geo)
    mean_abs = O.build_pyramid(np.abs(x), geo)
    depth = max(1, (geo.p - 1) * (geo.L - 1) + 1)
    half_ulp = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -24  # unit roundoff
    bound = 1.01 * (depth * 2.0 ** -24 * mean_abs + half_ulp * (np.abs(want) + depth * 2.0 ** -24 * mean_abs)) + 1e-30
    bad = np.abs(np.asarray(got, np.float64) - want) > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} cells outside the bound"


def g_of(dtype):
    """Score group size: the coordinates in 16 bytes of the storage dtype."""
    return 8 if dtype == torch.bfloat16 else 4
