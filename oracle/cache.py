"""Full-size oracle outputs of the named workloads, computed on all host cores and cached on disk.

TEST INFRASTRUCTURE ONLY, like the rest of oracle/: the parity tests, the smoke check and the
bench's CPU arm may use it; nothing on the product path imports it. It calls only the functions
of oracle/__init__.py (the fp64 definition) on the seeded inputs of mfa_inputs, and it never
reads anything the CUDA path produced.

What it adds is a schedule, not arithmetic: a workload is cut into independent units (one query
head, or one kv head of one sequence), each unit is handed to the oracle function of its
workload kind in a worker process, and the pieces are put back in place. Rows, heads and
sequences of attention are independent in the definition, so the assembled arrays are exactly
what one call of the same oracle function over the whole workload returns.

Workers are started with the "spawn" method (safe after the parent has initialised CUDA), each
with one BLAS thread. Inputs reach them through .npy files that they map read-only.

Results are cached under oracle/_cache/ (not part of the repository), one directory per
(workload, seed, digest), the digest being a hash of this file, oracle/__init__.py and the input
generator's sources, so a change to any of them recomputes.

python -m oracle.cache [NAME ...]   precomputes (default: every workload, then the backwards).
"""
from __future__ import annotations

import atexit
import concurrent.futures as cf
import hashlib
import multiprocessing as mp
import os
import shutil
import sys
import tempfile
import time

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(_HERE)
CACHE_DIR = os.path.join(_HERE, "_cache")

# Workloads whose backward is cached as NAME + ":backward".
BACKWARD = ("causal_b2_h8_n4096_d128_fp16", "noncausal_b2_h8_n4096_d128_fp16")


def _mi():
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import mfa_inputs
    return mfa_inputs


def digest() -> str:
    h = hashlib.sha256()
    for f in (os.path.join(_HERE, "__init__.py"), os.path.abspath(__file__),
              os.path.join(ROOT, "mfa_inputs", "__init__.py"), os.path.join(ROOT, "mfa_inputs", "gen.c")):
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def _split(name: str):
    base, _, part = name.partition(":")
    return base, part


def cache_path(name: str) -> str:
    base, part = _split(name)
    case = _mi().workloads()[base]
    tag = base + ("-backward" if part == "backward" else "")
    return os.path.join(CACHE_DIR, f"{tag}-seed{case.seed}-{digest()}")


# ---------------------------------------------------------------- worker side
class _Widened:
    """Read-only view of a 16-bit page pool that widens exactly what is indexed to fp64, so the
    oracle's paged gather reads GB-sized pools without converting all of them."""

    def __init__(self, bits, dtype):
        self.bits = bits
        self.dtype = dtype
        self.shape = bits.shape

    def __getitem__(self, idx):
        return _mi().widen(np.ascontiguousarray(self.bits[idx]), self.dtype)


def _worker_init():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def _load(files, key):
    return np.load(files[key], mmap_mode="r")


def _unit(task):
    """One unit of a workload: returns (unit, {array name: piece})."""
    import oracle
    mi = _mi()
    name, unit, files = task
    base, part = _split(name)
    case = mi.workloads()[base]
    w = lambda x: mi.widen(np.ascontiguousarray(x), case.dtype)
    if part == "backward":
        b, g = unit
        G = case.Hq // case.Hkv
        hs = slice(g * G, (g + 1) * G)
        q, k, v, do = (_load(files, n) for n in ("q", "k", "v", "do"))
        dq, dk, dv = oracle.attention_backward(
            w(q[b:b + 1, hs]), w(k[b:b + 1, g:g + 1]), w(v[b:b + 1, g:g + 1]), w(do[b:b + 1, hs]),
            case.scale_f32(), case.causal, case.win_l, case.win_r, case.softcap)
        return unit, {"dq": dq[0], "dk": dk[0, 0], "dv": dv[0, 0]}
    if isinstance(case, mi.SparseCase):
        b, h = unit
        g = h // (case.Hq // case.Hkv)
        q, k, v, m = (_load(files, n) for n in ("q", "k", "v", "mask"))
        o, lse = oracle.attention_blocksparse(
            w(q[b:b + 1, h:h + 1]), w(k[b:b + 1, g:g + 1]), w(v[b:b + 1, g:g + 1]),
            np.ascontiguousarray(m[b:b + 1, h:h + 1]), case.scale_f32(), case.causal, case.win_l,
            case.win_r, case.softcap, block=mi.SPARSE_BLOCK)
        return unit, {"o": o[0, 0], "lse": lse[0, 0]}
    if isinstance(case, mi.PrefillCase):
        b, h = unit
        g = h // (case.Hq // case.Hkv)
        q, k, v = (_load(files, n) for n in ("q", "k", "v"))
        o, lse = oracle.attention(w(q[b:b + 1, h:h + 1]), w(k[b:b + 1, g:g + 1]),
                                  w(v[b:b + 1, g:g + 1]), case.scale_f32(), case.causal,
                                  case.win_l, case.win_r, case.softcap)
        return unit, {"o": o[0, 0], "lse": lse[0, 0]}
    if isinstance(case, mi.VarlenCase):
        b, h = unit
        g = h // (case.Hq // case.Hkv)
        q, k, v, cq, ck = (_load(files, n) for n in ("q", "k", "v", "cq", "ck"))
        q0, q1, k0, k1 = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
        o, lse = oracle.attention_varlen(w(q[q0:q1, h:h + 1]), w(k[k0:k1, g:g + 1]),
                                         w(v[k0:k1, g:g + 1]), [0, q1 - q0], [0, k1 - k0],
                                         case.scale_f32(), case.causal, case.win_l, case.win_r,
                                         case.softcap)
        return unit, {"o": o[:, 0], "lse": lse[0]}
    if isinstance(case, mi.PagedPrefillCase):
        b, h = unit
        g = h // (case.Hq // case.Hkv)
        q, kp, vp, table, lens, cq = (_load(files, n) for n in ("q", "kp", "vp", "table", "lens", "cq"))
        q0, q1 = int(cq[b]), int(cq[b + 1])
        o, lse = oracle.attention_paged_prefill(
            w(q[q0:q1, h:h + 1]), _Widened(kp[:, :, g:g + 1], case.dtype),
            _Widened(vp[:, :, g:g + 1], case.dtype), np.asarray(table[b:b + 1]),
            np.asarray(lens[b:b + 1]), [0, q1 - q0], case.scale_f32(), case.causal, case.win_l,
            case.win_r, case.softcap)
        return unit, {"o": o[:, 0], "lse": lse[0]}
    if isinstance(case, mi.DecodeCase):
        b, g = unit
        G = case.Hq // case.Hkv
        q, kp, vp, table, lens = (_load(files, n) for n in ("q", "kp", "vp", "table", "lens"))
        o, lse = oracle.decode(w(q[b:b + 1, g * G:(g + 1) * G]), _Widened(kp[:, :, g:g + 1], case.dtype),
                               _Widened(vp[:, :, g:g + 1], case.dtype), np.asarray(table[b:b + 1]),
                               np.asarray(lens[b:b + 1]), case.scale_f32(), case.causal,
                               case.softcap, win_l=case.win_l)
        return unit, {"o": o[0], "lse": lse[0]}
    raise TypeError(f"no oracle for {type(case).__name__}")


# ---------------------------------------------------------------- parent side
_POOL = None
_POOL_N = 0


def _pool(n):
    global _POOL, _POOL_N
    if _POOL is None or _POOL_N < n:
        if _POOL is not None:
            _POOL.shutdown()
        _POOL = cf.ProcessPoolExecutor(n, mp_context=mp.get_context("spawn"), initializer=_worker_init)
        _POOL_N = n
        atexit.register(_shutdown)
    return _POOL


def _shutdown():
    global _POOL
    if _POOL is not None:
        _POOL.shutdown(cancel_futures=True)
        _POOL = None


def _layout(name, tensors):
    """(inputs by name, units, output shapes and where a unit's pieces go)."""
    mi = _mi()
    base, part = _split(name)
    case = mi.workloads()[base]
    if part == "backward":
        q, k, v = tensors if tensors is not None else case.tensors()
        ins = {"q": q, "k": k, "v": v, "do": case.dout()}
        units = [(b, g) for b in range(case.B) for g in range(case.Hkv)]
        G = case.Hq // case.Hkv
        shapes = {"dq": q.shape, "dk": k.shape, "dv": k.shape}
        place = lambda u: {"dq": (u[0], slice(u[1] * G, (u[1] + 1) * G)), "dk": (u[0], u[1]),
                           "dv": (u[0], u[1])}
        return ins, units, shapes, place, (case.B * case.Hq) * case.Nq * case.Nk
    if isinstance(case, mi.SparseCase):
        q, k, v, m = tensors if tensors is not None else case.tensors()
        ins = {"q": q, "k": k, "v": v, "mask": m}
    elif isinstance(case, mi.PrefillCase):
        q, k, v = tensors if tensors is not None else case.tensors()
        ins = {"q": q, "k": k, "v": v}
    if isinstance(case, (mi.SparseCase, mi.PrefillCase)):
        units = [(b, h) for b in range(case.B) for h in range(case.Hq)]
        shapes = {"o": q.shape, "lse": q.shape[:3]}
        place = lambda u: {"o": (u[0], u[1]), "lse": (u[0], u[1])}
        return ins, units, shapes, place, case.B * case.Hq * case.Nq * case.Nk
    if isinstance(case, mi.VarlenCase):
        q, k, v = tensors if tensors is not None else case.tensors()
        cq, ck = case.cu_seqlens()
        ins = {"q": q, "k": k, "v": v, "cq": cq, "ck": ck}
        units = [(b, h) for b in range(case.B) for h in range(case.Hq)]
        shapes = {"o": q.shape, "lse": (case.Hq, q.shape[0])}
        place = lambda u: {"o": (slice(int(cq[u[0]]), int(cq[u[0] + 1])), u[1]),
                           "lse": (u[1], slice(int(cq[u[0]]), int(cq[u[0] + 1])))}
        work = case.Hq * int(np.sum(np.diff(cq).astype(np.int64) * np.diff(ck)))
        return ins, units, shapes, place, work
    if isinstance(case, mi.PagedPrefillCase):
        q, kp, vp, table, lens, cq = tensors if tensors is not None else case.tensors()
        ins = {"q": q, "kp": kp, "vp": vp, "table": table, "lens": lens, "cq": cq}
        units = [(b, h) for b in range(case.B) for h in range(case.Hq)]
        shapes = {"o": q.shape, "lse": (case.Hq, q.shape[0])}
        place = lambda u: {"o": (slice(int(cq[u[0]]), int(cq[u[0] + 1])), u[1]),
                           "lse": (u[1], slice(int(cq[u[0]]), int(cq[u[0] + 1])))}
        work = case.Hq * int(np.sum(np.diff(cq).astype(np.int64) * lens))
        return ins, units, shapes, place, work
    if isinstance(case, mi.DecodeCase):
        q, kp, vp, table, lens = tensors if tensors is not None else case.tensors()
        ins = {"q": q, "kp": kp, "vp": vp, "table": table, "lens": lens}
        units = [(b, g) for b in range(case.B) for g in range(case.Hkv)]
        G = case.Hq // case.Hkv
        shapes = {"o": q.shape, "lse": q.shape[:3]}
        place = lambda u: {"o": (u[0], slice(u[1] * G, (u[1] + 1) * G)),
                           "lse": (u[0], slice(u[1] * G, (u[1] + 1) * G))}
        return ins, units, shapes, place, case.Hq * case.Nq * int(np.sum(lens))
    raise TypeError(f"no oracle for {type(case).__name__}")


def _workers(n_units, per_unit_bytes):
    n = min(os.cpu_count() or 1, n_units)
    try:
        import psutil
        avail = psutil.virtual_memory().available
        n = min(n, max(1, int(avail * 0.6 // max(per_unit_bytes, 1))))
    except Exception:
        pass
    return max(1, n)


def compute(name, tensors=None, verbose=False):
    """The oracle's full outputs of workload `name` (NAME or NAME:backward) as a dict of fp64
    arrays: o / lse in the workload's layouts, or dq / dk / dv. `tensors` may pass the inputs the
    caller already drew (exactly those of the workload's tensors())."""
    t0 = time.time()
    ins, units, shapes, place, work = _layout(name, tensors)
    out = {k: np.full(s, -np.inf if k == "lse" else 0.0) for k, s in shapes.items()}
    os.makedirs(CACHE_DIR, exist_ok=True)
    tmp = tempfile.mkdtemp(prefix="inputs-", dir=CACHE_DIR)
    try:
        files = {}
        for k, a in ins.items():
            files[k] = os.path.join(tmp, k + ".npy")
            np.save(files[k], np.ascontiguousarray(a))
        # per-unit memory: a 512-row score block and its temporaries, or whole score matrices
        # for the backward (6 arrays of Nq x Nk fp64 per query head)
        mi = _mi()
        case = mi.workloads()[_split(name)[0]]
        if _split(name)[1] == "backward":
            per = 10 * (case.Hq // case.Hkv) * case.Nq * case.Nk * 8
        else:
            nk = getattr(case, "Nk", None) or getattr(case, "len_hi", 0) or 1 << 17
            per = 8 * 512 * max(int(nk), 1) * 8 + (2 << 30 if isinstance(case, mi.DecodeCase) else 0)
        n = _workers(len(units), per)
        ex = _pool(n)
        futs = [ex.submit(_unit, (name, u, files)) for u in units]
        for f in cf.as_completed(futs):
            u, pieces = f.result()
            for key, idx in place(u).items():
                out[key][idx] = pieces[key]
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    if verbose:
        print(f"oracle {name}: {len(units)} units on {n} processes, {time.time() - t0:.1f} s "
              f"({work:.3g} score entries)", flush=True)
    return out


def reference(name, tensors=None, verbose=False):
    """compute(name) through the on-disk cache."""
    path = cache_path(name)
    keys = ("dq", "dk", "dv") if _split(name)[1] == "backward" else ("o", "lse")
    if all(os.path.exists(os.path.join(path, k + ".npy")) for k in keys):
        return {k: np.load(os.path.join(path, k + ".npy")) for k in keys}
    res = compute(name, tensors, verbose)
    os.makedirs(CACHE_DIR, exist_ok=True)
    tmp = tempfile.mkdtemp(prefix="write-", dir=CACHE_DIR)
    for k in keys:
        np.save(os.path.join(tmp, k + ".npy"), res[k])
    try:
        os.replace(tmp, path)  # whole directories appear at once
    except OSError:
        shutil.rmtree(tmp, ignore_errors=True)
    return res


def all_names():
    return sorted(_mi().workloads()) + [n + ":backward" for n in BACKWARD]


if __name__ == "__main__":
    for nm in (sys.argv[1:] or all_names()):
        reference(nm, verbose=True)
