"""ctypes front end of the fp64 CPU oracle (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this module.  The product path (``token_dynamic_expert_b200``)
never does; it shares no code with it.

Every function takes numpy arrays or CPU torch tensors, widens activations
and tables to float64 and weights to float32 (exact copies of bf16 or fp32
storage), calls the C oracle, and returns numpy arrays.  Formulas are cited in
``ace_oracle.c``; the one rule written here, the quantile mapping for tau,
is cited at :func:`tau_quantile`.
"""
import ctypes
import math

import numpy as np

from . import build as _build

_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_F = ctypes.POINTER(ctypes.c_float)
_I = ctypes.POINTER(ctypes.c_int)
_U8 = ctypes.POINTER(ctypes.c_ubyte)


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i, d = ctypes.c_int, ctypes.c_double
        L.ora_set_threads.argtypes = [i]
        L.ora_get_threads.restype = i
        L.ora_rmsnorm.argtypes = [i, i, _D, _D, d, _D, _D]
        L.ora_swiglu.argtypes = [i, i, _D, _F, _F, _F, _D, _D]
        L.ora_router.argtypes = [i, i, i, i, _D, _F, _F, i, _D, _I, _D]
        L.ora_sigma_factors.argtypes = [i, i, i, _D, _F, _F, _F, i, _D]
        L.ora_gsp.argtypes = [i, i, i, _D, _F, _F, _F, i, i, d, _D, _D, _D, _D, _D]
        L.ora_rcr.argtypes = [i, i, i, _D, _F, _F, _F, _F, d, d, _D, _D, _D, _D]
        L.ora_mask.argtypes = [i, i, _I, _D, _D, _D, d, i, _D, _D, _D, _U8]
        L.ora_mask.restype = i
        L.ora_compact.argtypes = [i, i, i, _I, _U8, _I, _I, _I, _I, _I]
        L.ora_compact.restype = i
        L.ora_combine.argtypes = [i, i, i, i, _D, _I, _D, _U8, _F, _F, _F, _D]
        _lib = L
    return _lib


def set_threads(n: int) -> None:
    lib().ora_set_threads(int(n))


def threads() -> int:
    return int(lib().ora_get_threads())


# ---------------------------------------------------------------- marshalling
def _np(a, dtype):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().cpu()
        if str(a.dtype) == "torch.bfloat16":
            a = a.float()
        a = a.numpy()
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctype)


# ------------------------------------------------------------------ functions
def rmsnorm(u, gamma, eps_rms=1e-6):
    u = _np(u, np.float64)
    gamma = _np(gamma, np.float64)
    T, d = u.shape
    xbar = np.empty_like(u)
    x = np.empty_like(u)
    lib().ora_rmsnorm(T, d, _p(u, _D), _p(gamma, _D), eps_rms, _p(xbar, _D), _p(x, _D))
    return xbar, x


def swiglu(z, wg_e, wu_e, wd_e):
    """One expert on one already-scaled row z = xbar Gamma; returns (h, f)."""
    z = _np(z, np.float64)
    wg_e, wu_e, wd_e = (_np(w, np.float32) for w in (wg_e, wu_e, wd_e))
    m, d = wg_e.shape
    h = np.empty(m)
    out = np.empty(d)
    lib().ora_swiglu(d, m, _p(z, _D), _p(wg_e, _F), _p(wu_e, _F), _p(wd_e, _F), _p(h, _D), _p(out, _D))
    return h, out


def router(x, wr, bias, k, renorm=True):
    x = _np(x, np.float64)
    wr = _np(wr, np.float32)
    bias = _np(bias, np.float32)
    T, d = x.shape
    E = wr.shape[0]
    logits = np.empty((T, E))
    idx = np.empty((T, k), dtype=np.int32)
    gate = np.empty((T, k))
    lib().ora_router(T, d, E, k, _p(x, _D), _p(wr, _F), _p(bias, _F), int(bool(renorm)),
                     _p(logits, _D), _p(idx, _I), _p(gate, _D))
    return logits, idx, gate


def sigma_factors(gamma, wg, wu, wd, iters=200):
    """sigma_1 of Gamma W^gate, Gamma W^up and W^down per expert, [E, 3]."""
    gamma = _np(gamma, np.float64)
    wg, wu, wd = (_np(w, np.float32) for w in (wg, wu, wd))
    E, m, d = wg.shape
    out = np.empty((E, 3))
    lib().ora_sigma_factors(E, d, m, _p(gamma, _D), _p(wg, _F), _p(wu, _F), _p(wd, _F), iters, _p(out, _D))
    return out


def gsp(gamma, wg, wu, wd, spectral=False, iters=200, eps=1e-6):
    gamma = _np(gamma, np.float64)
    wg, wu, wd = (_np(w, np.float32) for w in (wg, wu, wd))
    E, m, d = wg.shape
    norms = np.empty((E, 4))
    a_up, a_gate, a_tilde, A = (np.empty(E) for _ in range(4))
    lib().ora_gsp(E, d, m, _p(gamma, _D), _p(wg, _F), _p(wu, _F), _p(wd, _F),
                  int(bool(spectral)), iters, eps, _p(norms, _D), _p(a_up, _D),
                  _p(a_gate, _D), _p(a_tilde, _D), _p(A, _D))
    return dict(norms=norms, a_up=a_up, a_gate=a_gate, a_tilde=a_tilde, A=A)


def rcr(gamma, wr, wg, wu, wd, rho=1.0, eps=1e-6):
    gamma = _np(gamma, np.float64)
    wr = _np(wr, np.float32)
    wg, wu, wd = (_np(w, np.float32) for w in (wg, wu, wd))
    E, m, d = wg.shape
    q = np.empty((E, d))
    fnorm, a_tilde, A = (np.empty(E) for _ in range(3))
    lib().ora_rcr(E, d, m, _p(gamma, _D), _p(wr, _F), _p(wg, _F), _p(wu, _F), _p(wd, _F),
                  rho, eps, _p(q, _D), _p(fnorm, _D), _p(a_tilde, _D), _p(A, _D))
    return dict(q=q, fnorm=fnorm, a_tilde=a_tilde, A=A)


def tables(layer, spectral=False, iters=200, rho=1.0, eps=1e-6):
    """GSP and RCR tables of one layer and their elementwise max."""
    g = gsp(layer["gamma"], layer["wg"], layer["wu"], layer["wd"], spectral, iters, eps)
    r = rcr(layer["gamma"], layer["wr"], layer["wg"], layer["wu"], layer["wd"], rho, eps)
    return dict(gsp=g, rcr=r, A_gsp=g["A"], A_rcr=r["A"], Amax=np.maximum(g["A"], r["A"]))


FUSIONS = {"max": 0, "min": 1, "mean": 2, "gsp": 3, "rcr": 4}


def mask(idx, gate, A_gsp, A_rcr, tau, fusion="max"):
    idx = _np(idx, np.int32)
    gate = _np(gate, np.float64)
    A_gsp = _np(A_gsp, np.float64)
    A_rcr = _np(A_rcr, np.float64)
    T, k = idx.shape
    s_gsp, s_rcr, c = (np.empty((T, k)) for _ in range(3))
    keep = np.empty((T, k), dtype=np.uint8)
    dis = lib().ora_mask(T, k, _p(idx, _I), _p(gate, _D), _p(A_gsp, _D), _p(A_rcr, _D),
                         float(tau), FUSIONS[fusion], _p(s_gsp, _D), _p(s_rcr, _D), _p(c, _D),
                         _p(keep, _U8))
    return dict(s_gsp=s_gsp, s_rcr=s_rcr, c=c, keep=keep, disagree=int(dis))


def compact(idx, keep, E):
    idx = _np(idx, np.int32)
    keep = _np(keep, np.uint8)
    T, k = idx.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    slot_token = np.empty(T * k, dtype=np.int32)
    slot_rank = np.empty(T * k, dtype=np.int32)
    slot_of = np.empty((T, k), dtype=np.int32)
    S = lib().ora_compact(T, k, E, _p(idx, _I), _p(keep, _U8), _p(counts, _I), _p(offsets, _I),
                          _p(slot_token, _I), _p(slot_rank, _I), _p(slot_of, _I))
    return dict(S=int(S), counts=counts, offsets=offsets, slot_token=slot_token[:S].copy(),
                slot_rank=slot_rank[:S].copy(), slot_of=slot_of)


def combine(x, idx, gate, keep, wg, wu, wd):
    x = _np(x, np.float64)
    idx = _np(idx, np.int32)
    gate = _np(gate, np.float64)
    keep = _np(keep, np.uint8)
    wg, wu, wd = (_np(w, np.float32) for w in (wg, wu, wd))
    T, d = x.shape
    k = idx.shape[1]
    m = wg.shape[1]
    y = np.empty((T, d))
    lib().ora_combine(T, d, m, k, _p(x, _D), _p(idx, _I), _p(gate, _D), _p(keep, _U8),
                      _p(wg, _F), _p(wu, _F), _p(wd, _F), _p(y, _D))
    return y


def n_skip_for(T, k, rate, of="slots"):
    """Number of slots a skip rate asks for: rate of all T*k slots, or of the
    T*(k-1) non-top-1 slots; rounded half up."""
    total = T * k if of == "slots" else T * (k - 1)
    return int(math.floor(rate * total + 0.5))


def tau_quantile(c, n_skip):
    """Quantile mapping for the threshold ([ACE] "Efficiency Results", Table 6:
    thresholds are set by mapping a target skip rate to a score quantile).

    The candidates are the scores of the non-top-1 slots (column 0 of ``c`` is
    the top-1 slot, never skipped).  Sorted ascending c_(1) <= ... <= c_(N),
    tau = c_(n+1), so that exactly n slots satisfy c < tau when the scores
    have no ties; tau = +inf when n >= N and every candidate is skipped."""
    c = _np(c, np.float64)
    cand = np.sort(c[:, 1:].reshape(-1))
    if n_skip <= 0:
        return float(cand[0]) if cand.size else math.inf
    if n_skip >= cand.size:
        return math.inf
    return float(cand[n_skip])


def moe_forward(layer, u, tau, A_gsp, A_rcr, renorm=True, keep=None, eps_rms=1e-6, outputs=True,
                fusion="max"):
    """Whole layer: RMSNorm, router, top-k, scores, skip mask (views fused by
    ``fusion``), compaction and the gate-weighted combine of the kept slots.
    ``keep`` overrides the mask (to evaluate the outputs the GPU produced with
    its own mask)."""
    xbar, x = rmsnorm(u, layer["gamma"], eps_rms)
    logits, idx, gate = router(x, layer["wr"], layer.get("bias"), layer["k"], renorm)
    mk = mask(idx, gate, A_gsp, A_rcr, tau, fusion)
    kp = mk["keep"] if keep is None else _np(keep, np.uint8)
    E = layer["wr"].shape[0]
    cp = compact(idx, kp, E)
    y = combine(x, idx, gate, kp, layer["wg"], layer["wu"], layer["wd"]) if outputs else None
    return dict(xbar=xbar, x=x, logits=logits, idx=idx, gate=gate, keep=kp, y=y,
                s_gsp=mk["s_gsp"], s_rcr=mk["s_rcr"], c=mk["c"], disagree=mk["disagree"], **cp)
