"""Observed error headroom of the products against the oracle.

Every output check in the GPU parity tests records, per (format, kernel
path), the observed relative L2 error and the worst per-element ratio
|y - y_ref| / (1e-2 * sum_k |x_k| |w_hat_k|); the session prints the worst of
each at the end, so a drift toward the 5e-3 / 1e-2 bounds shows up before it
fails a test."""
from __future__ import annotations

import json
import os

_WORST: dict[tuple[str, str], dict] = {}


def path_of(fmt: str, M: int) -> str:
    import weight_only_quantized_rq_b200 as rq
    return "tensor-core" if rq.tc_path(fmt, M) else "gemv"


def record(fmt: str, M: int, rel_l2: float, elem_ratio: float) -> None:
    key = (fmt, path_of(fmt, M))
    w = _WORST.setdefault(key, {"checks": 0, "rel_l2": 0.0, "elem_ratio": 0.0, "M": []})
    w["checks"] += 1
    w["rel_l2"] = max(w["rel_l2"], float(rel_l2))
    w["elem_ratio"] = max(w["elem_ratio"], float(elem_ratio))
    if M not in w["M"]:
        w["M"].append(M)


def summary_lines() -> list[str]:
    if not _WORST:
        return []
    out = ["product error headroom (worst observed; bounds: rel-L2 5e-3, element ratio 1.0):",
           f"  {'format':8s} {'path':12s} {'checks':>6s} {'rel-L2':>10s} {'elem ratio':>11s}  M"]
    for (fmt, path), w in sorted(_WORST.items()):
        ms = ",".join(str(m) for m in sorted(w["M"]))
        out.append(f"  {fmt:8s} {path:12s} {w['checks']:6d} {w['rel_l2']:10.3e} {w['elem_ratio']:11.3e}  {ms}")
    return out


def dump(path: str) -> None:
    rows = [{"format": f, "path": p, **w} for (f, p), w in sorted(_WORST.items())]
    with open(path, "w") as fh:
        json.dump(rows, fh, indent=1)


def dump_dir() -> str | None:
    d = os.environ.get("RQ_HEADROOM_DIR")
    return d if d and os.path.isdir(d) else None


def check_y(y, y_ref, xbits, w_hat, fmt, rel=5e-3, elem=1e-2):
    """The products' acceptance test: relative L2 error <= rel and, per
    element, |y - y_ref| <= elem * sum_k |x_k| |w_hat_k| against the oracle's
    fp64 sums; records the observed headroom."""
    import numpy as np
    xf = (xbits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    bound = elem * (np.abs(xf) @ np.abs(w_hat.astype(np.float64)).T)
    err = np.abs(y.astype(np.float64) - y_ref)
    nrm = np.linalg.norm(y_ref)
    rel_l2 = np.linalg.norm(err) / max(nrm, 1e-30)
    ratio = float(np.max(err / (bound + 1e-30))) if err.size else 0.0
    record(fmt, int(y.shape[0]), rel_l2, ratio)
    assert rel_l2 <= rel, rel_l2
    bad = err > bound + 1e-30
    assert not bad.any(), f"{bad.sum()} elements outside 1e-2*sum|x||w|"
