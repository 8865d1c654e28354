"""Shared helpers of the GPU parity tests (inputs and comparisons only)."""
import numpy as np
import torch

import oracle

# Tolerances. The attention outputs and gradients are stored in the input
# dtype, so every element carries one rounding of its exact value to that
# dtype (half a unit in the last place: |x| * 2^-9 for bf16, |x| * 2^-24 for
# fp32). The max-abs bounds apply to the error beyond that final rounding:
#   |got - want| <= TOL + ROUND * |want|
# With bf16 gradients of magnitude 8..16 the rounding alone reaches 0.03, so a
# flat 2e-2 bound could not be met by any bf16 result.
BF16_TOL = 2e-2      # max-abs, bf16 (outputs and gradients)
F32_TOL = 1e-5       # max-abs, fp32
BF16_ROUND = 2.0 ** -9
F32_ROUND = 2.0 ** -24
GRAD_REL_L2 = 1e-2   # relative L2 on gradients
# The bf16 path's log-sum-exp is stored in fp32, so it gets no bf16 allowance.
# Its error is set by the arithmetic of the forward: the row sum adds
# exponentials with relative error <= 7.5e-5 (the FMA-pipe cubic; ex2.approx is
# far tighter), which moves ln(sum) by at most 7.5e-5, and the fp32 scores of the
# bf16 products carry about 1e-4 of accumulated rounding at |<q,k>| ~ 45. 1e-3
# leaves a factor of five above that sum.
LSE_TOL = 1e-3

# Every comparison is recorded (check, flat max |got - want|, max excess beyond
# the stored value's rounding, tolerance) so that a run can report the flat
# max-abs beside the rounding-aware figure the assertion uses.
REPORT = []


def dev(x, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def events_dev(ev):
    ev = np.asarray(ev, dtype=np.int32).reshape(-1, 4)
    return torch.from_numpy(ev).cuda()


def compare_mask(gm, ev, B, N):
    """GPU mask == oracle brute force, bit for bit."""
    kap = oracle.kappa(ev, B, N)
    om = oracle.tile_mask(kap)
    assert np.array_equal(gm.kappa.cpu().numpy(), kap)
    assert np.array_equal(gm.cls.cpu().numpy(), om["cls"])
    assert gm.nnz == om["nnz"] and gm.n_partial == om["n_partial"]
    assert gm.visible_pairs == oracle.visible_pairs(kap)
    for f in ("row_ptr", "col_ptr"):
        assert np.array_equal(getattr(gm, f).cpu().numpy(), om[f]), f
    for f in ("row_col", "row_pidx", "col_row", "col_pidx"):
        assert np.array_equal(getattr(gm, f).cpu().numpy()[: om["nnz"]], om[f]), f
    gb = gm.bits.cpu().numpy().view(np.uint32)[: om["n_partial"]]
    assert np.array_equal(gb, om["bits"])
    return kap


def assert_close(got, want, tol, what="", rnd=None):
    """max |got - want| - rnd*|want| <= tol (rnd defaults to the dtype's rounding
    for the two standard tolerances)."""
    if rnd is None:
        rnd = BF16_ROUND if tol == BF16_TOL else (F32_ROUND if tol == F32_TOL else 0.0)
    if not got.size:
        return 0.0
    diff = np.abs(got - want)
    excess = diff - rnd * np.abs(want)
    i = np.unravel_index(np.argmax(excess), excess.shape)
    err = float(excess[i])
    REPORT.append((what, float(diff.max()), err, tol))
    assert err <= tol, (f"{what}: max-abs beyond output rounding {err:.3g} > {tol} "
                        f"at {i} (got {got[i]:.6g}, want {want[i]:.6g}; flat max-abs {diff.max():.3g})")
    return err


def rel_l2(got, want):
    """Relative L2 error; None when the exact value is (numerically) zero."""
    den = np.linalg.norm(want.ravel())
    if den <= 1e-6 * np.sqrt(max(want.size, 1)):
        return None
    return float(np.linalg.norm((got - want).ravel()) / den)
