"""Helpers for the GPU parity tests: the error metric and oracle sampling."""
import numpy as np
import torch

import oracle

# Tolerances on max|gpu - oracle| / rms(oracle), for o and for the final state.
TOL = {"fp32": 1e-4, "bf16": 2e-2}


# Storing o in bf16 rounds each element by up to half a bf16 ulp, at most 2^-8 |o|: an error
# no kernel can avoid. Small cases, where max|o| / rms(o) can exceed 10, allow that
# rounding on top of the tolerance (rel_err_excess); the five workloads use the plain
# metric (rel_err).
OUT_ROUND = {"fp32": 0.0, "bf16": 2.0 ** -8}


def rel_err_excess(got, ref, dtype):
    got = got.detach().double().cpu().numpy() if torch.is_tensor(got) else np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    excess = np.maximum(np.abs(got - ref) - OUT_ROUND[dtype] * np.abs(ref), 0.0)
    return float(np.max(excess) / max(rms, 1e-30))


def rel_err(got, ref):
    got = got.detach().double().cpu().numpy() if torch.is_tensor(got) else np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    return float(np.max(np.abs(got - ref)) / max(rms, 1e-30))


def oracle_units(inp, units):
    """Run the oracle on a list of (b, h) units of a chunked-forward input set.

    Returns (o [n,T,Dv], hT [n,Dk,Dv]) in unit order. Each unit becomes one
    batch row with a single key/value head, so all run in parallel threads.
    """
    q, k, v, g, beta, h0 = (inp[n] for n in ("q", "k", "v", "g", "beta", "h0"))
    Hk, Hv = q.shape[2], v.shape[2]
    grp = Hv // Hk
    sel = lambda x, b, h: x[b:b + 1, :, h:h + 1]
    qs = torch.cat([sel(q, b, h // grp) for b, h in units]).cpu()
    ks = torch.cat([sel(k, b, h // grp) for b, h in units]).cpu()
    vs = torch.cat([sel(v, b, h) for b, h in units]).cpu()
    gs = torch.cat([sel(g, b, h) for b, h in units]).cpu()
    bs = torch.cat([sel(beta, b, h) for b, h in units]).cpu()
    h0s = None if h0 is None else torch.cat([h0[b:b + 1, h:h + 1] for b, h in units]).cpu()
    o, hT = oracle.recurrent(qs, ks, vs, gs, bs, h0s)
    return o[:, :, 0], hT[:, 0]


def sample_units(B, Hv, n, seed=0):
    rng = np.random.default_rng(seed)
    units = {(0, 0), (B - 1, Hv - 1)}
    while len(units) < n:
        units.add((int(rng.integers(B)), int(rng.integers(Hv))))
    return sorted(units)
