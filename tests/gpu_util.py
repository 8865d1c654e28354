"""Shared helpers of the GPU parity tests (inputs and comparisons only)."""
import numpy as np
import torch

import oracle

BF16_TOL = 2e-2      # max-abs on attention outputs and gradients (bf16)
F32_TOL = 1e-5       # max-abs (fp32)
GRAD_REL_L2 = 1e-2   # relative L2 on gradients


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


def assert_close(got, want, tol, what=""):
    err = float(np.abs(got - want).max()) if got.size else 0.0
    assert err <= tol, f"{what}: max-abs {err:.3g} > {tol}"
    return err


def rel_l2(got, want):
    return float(np.linalg.norm((got - want).ravel()) / max(np.linalg.norm(want.ravel()), 1e-30))
