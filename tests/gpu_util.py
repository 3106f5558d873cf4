"""Helpers for the GPU parity tests: device buffers, the acceptance checks."""
import numpy as np

import int4_expert_routing_b200 as F

# Acceptance: |gpu - oracle| <= 1e-2 * (|oracle| + rms(oracle row)) per element;
# expert indices bit-exact except where the oracle's 6th/7th biased-score gap
# is below 1e-6 (logged and excluded).
REL_TOL = 1e-2
TIE_GAP = 1e-6


def torch():
    import torch as _t
    return _t


def dev_bf16(bits: np.ndarray):
    return torch().from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()


def host_bf16(t) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def bf16_to_f64(bits):
    b = np.asarray(bits, np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def workspace(op: int, n: int):
    nbytes = F.flint_workspace_bytes(op, n)
    assert nbytes > 0
    ws = torch().zeros(nbytes, dtype=torch().uint8, device="cuda")
    F.flint_workspace_init(ws, nbytes)
    return ws, nbytes


def check_close(gpu: np.ndarray, ref: np.ndarray, rows=None, what="output"):
    """The per-element acceptance bound on the given rows; returns the worst
    ratio |err| / bound."""
    gpu = np.atleast_2d(np.asarray(gpu, np.float64))
    ref = np.atleast_2d(np.asarray(ref, np.float64))
    rows = range(ref.shape[0]) if rows is None else rows
    worst = 0.0
    for r in rows:
        rms = np.sqrt(np.mean(ref[r] ** 2))
        bound = REL_TOL * (np.abs(ref[r]) + rms)
        err = np.abs(gpu[r] - ref[r])
        ratio = float(np.max(err / bound))
        worst = max(worst, ratio)
        if ratio > 1.0:
            bad = int(np.argmax(err / bound))
            raise AssertionError(f"{what} row {r} elem {bad}: gpu {gpu[r][bad]!r} oracle "
                                 f"{ref[r][bad]!r} bound {bound[bad]:.3e}")
    return worst


def routing_rows(idx_gpu, idx_ref, gap, log=print):
    """Rows whose expert indices must match exactly; asserts them, returns the
    list of compared rows (rows with an oracle near-tie are logged, skipped)."""
    keep = []
    for r in range(idx_ref.shape[0]):
        if gap[r] < TIE_GAP:
            log(f"row {r}: 6th/7th biased-score gap {gap[r]:.3e} < {TIE_GAP}: excluded")
            continue
        assert list(idx_gpu[r]) == list(idx_ref[r]), (r, idx_gpu[r], idx_ref[r], gap[r])
        keep.append(r)
    return keep
