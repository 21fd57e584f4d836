"""Hyper-parameter tuning by the L1 error rule.

The method's three hyper-parameters tau (TopCdf mass), theta (self-similarity
threshold) and lambda (P~V skip threshold) are set per layer against the error
of the sparse output O' relative to full attention O (paper review page,
section 三 "超参数确定策略"; rebuttal page, reply to Weakness 2):

    L1 = sum |O - O'| / sum |O|,   band (l1, l2) per model family
    (Llama3.1 (0.08, 0.09); CogVideoX / Mochi (0.05, 0.06); SD3.5 / Flux (0.07, 0.08)).

The page states the rule for tau only, and garbled: "L1 < l1: increase tau
(raise sparsity)", but a larger tau keeps more probability mass and so LESS
sparsity.  Readings taken here:

  * every parameter has a dense end (least skipping, least error) and a sparse
    end: tau 1 -> 0.05, lambda -50 -> -0.5 (natural-log units; -50 skips
    nothing a float32 softmax can see), theta 1 -> -1 (theta >= 1 makes every
    block a fix block, theta < -1 none);
  * when L1 < l1 a parameter moves toward its sparse end, when L1 > l2 toward
    its dense end, and the search stops inside the band (bisection, since L1
    grows monotonically toward the sparse end);
  * the three are searched one after another, tau first, then lambda, then
    theta (the page's "三个超参数 ... 通过 L1 误差约束自适应确定"), each over
    its whole range with the others held at their current values (the
    caller's, for those not searched yet); the next one is searched only
    while L1 is still below the band.

O is computed by the library itself in its dense limit (theta > 1 makes every
block a fix block and lambda = -inf skips nothing: plain softmax attention).
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Optional, Sequence, Tuple

import torch

BANDS = {"llama": (0.08, 0.09), "video": (0.05, 0.06), "image": (0.07, 0.08)}

# (dense end, sparse end) of each hyper-parameter
RANGES = {"tau": (1.0, 0.05), "lambda": (-50.0, -0.5), "theta": (1.0, -1.0)}
ORDER = ("tau", "lambda", "theta")


@dataclasses.dataclass
class TuneResult:
    tau: float
    l1: float
    sparsity: float
    in_band: bool
    trace: list
    theta: Optional[float] = None
    lam: Optional[float] = None


def search_param(l1_of: Callable[[float], Tuple[float, float]], band, dense: float,
                 sparse: float, iters: int = 12):
    """Bisection of one parameter between its dense and its sparse end.
    l1_of(x) -> (L1, sparsity); L1 grows from the dense toward the sparse end.

    Returns (x, L1, sparsity, in_band, trace): the first x whose L1 lies in the
    band; otherwise the x nearest the sparse end among those tried whose L1
    stays at or below l2 (the sparsest admissible), or the dense end when
    even that exceeds l2."""
    l1_lo, l1_hi = band
    trace = []
    e_d, s_d = l1_of(dense)
    trace.append((dense, e_d, s_d))
    if e_d > l1_hi or l1_lo <= e_d <= l1_hi:
        return dense, e_d, s_d, l1_lo <= e_d <= l1_hi, trace
    best = (dense, e_d, s_d)
    a, b = dense, sparse                  # a: admissible side, b: sparse side
    for _ in range(iters):
        mid = 0.5 * (a + b)
        e, sp = l1_of(mid)
        trace.append((mid, e, sp))
        if e > l1_hi:
            b = mid                       # too much error: back toward dense
        else:
            best = (mid, e, sp)
            if e >= l1_lo:
                return mid, e, sp, True, trace
            a = mid                       # room for more sparsity
    return best[0], best[1], best[2], False, trace


def search_tau(l1_of: Callable[[float], Tuple[float, float]], band=(0.08, 0.09),
               lo: float = 0.05, hi: float = 1.0, iters: int = 12) -> TuneResult:
    """Bisection on tau alone (dense end hi, sparse end lo)."""
    x, e, sp, ok, trace = search_param(l1_of, band, hi, lo, iters)
    return TuneResult(x, e, sp, ok, trace)


def search_params(l1_of: Callable[[dict], Tuple[float, float]], start: dict, band,
                  order: Sequence[str] = ORDER, ranges=RANGES, iters: int = 12) -> TuneResult:
    """Coordinate search over the hyper-parameters in `order`.  l1_of(hp) ->
    (L1, sparsity) for a dict hp with keys tau, theta, lambda.  Each parameter
    in turn is bisected over its whole range, from its dense to its sparse
    end, with the others held at their current values (the caller's, for those
    not searched yet); the search goes on to the next parameter only while L1
    is still below the band."""
    hp = dict(start)
    trace = []
    e = sp = None
    for name in order:
        dense, sparse = ranges[name]
        f = lambda x, name=name: l1_of({**hp, name: x})
        x, e, sp, ok, tr = search_param(f, band, dense, sparse, iters)
        trace.extend((name,) + t for t in tr)
        hp[name] = x
        if ok or e > band[1]:
            break
    return TuneResult(hp["tau"], e, sp, band[0] <= e <= band[1], trace, theta=hp["theta"],
                      lam=hp["lambda"])


def _with(params, **kw):
    p = type(params)()
    ctypes_fields = [f[0] for f in params._fields_]
    for f in ctypes_fields:
        setattr(p, f, getattr(params, f))
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def layer_l1(params, q, k, v, stream=None):
    """Returns l1_of(hp) -> (L1, sparsity) for one layer's calibration tensors
    (device, [B,H,N,d]) against the library's dense limit."""
    import free_block_sparse_predict_b200 as fb
    dev = q.device
    # dense reference O: every block kept, no P~V skipped
    dense_p = _with(params, theta=2.0, lam=float("-inf"), qk_int8=0, o_dtype=2)
    ws = fb.workspace(dense_p, dev)
    mask, idx, cnt, _, _ = fb.predict_outputs(dense_p, dev)
    fb.sparge_predict_mask(dense_p, q, k, mask, idx, cnt, None, None, ws, stream)
    o_ref = torch.empty(q.shape, dtype=torch.float32, device=dev)
    fb.sparge_attn_fwd(dense_p, q, k, v, idx, cnt, o_ref, ws, None, stream)
    ref_abs = o_ref.abs().sum()
    vis = int(mask.sum())                     # blocks kept by the dense mask = visible
    o = torch.empty_like(o_ref)
    stats = torch.zeros(5, dtype=torch.int64, device=dev)

    def l1_of(hp: dict):
        p = _with(params, tau=float(hp["tau"]), theta=float(hp["theta"]),
                  lam=float(hp["lambda"]), o_dtype=2)
        wsp = fb.workspace(p, dev)
        m2, i2, c2, _, _ = fb.predict_outputs(p, dev)
        fb.sparge_predict_mask(p, q, k, m2, i2, c2, None, None, wsp, stream)
        stats.zero_()
        fb.sparge_attn_fwd(p, q, k, v, i2, c2, o, wsp, stats, stream)
        l1 = float((o - o_ref).abs().sum() / ref_abs)
        st = stats.cpu().tolist()
        sparsity = 1.0 - (st[1] + st[3] / 4.0) / (2.0 * vis)
        return l1, sparsity

    return l1_of


def tune_layer(params, q, k, v, band=(0.08, 0.09), order: Sequence[str] = ORDER,
               iters: int = 12, stream=None) -> TuneResult:
    """Tunes tau, lambda and theta (in `order`) for one layer's calibration
    tensors, starting from the values in params."""
    l1_of = layer_l1(params, q, k, v, stream)
    start = {"tau": float(params.tau), "theta": float(params.theta),
             "lambda": float(params.lam)}
    return search_params(l1_of, start, band, order, iters=iters)


def tune_heads(params, q, k, v, band=(0.08, 0.09), **kw) -> list:
    """Per-head hyper-parameters: each query head with its KV head, tuned on its own."""
    g = params.Hq // params.Hkv
    out = []
    for h in range(params.Hq):
        p = _with(params, Hq=1, Hkv=1)
        qs = q[:, h:h + 1].contiguous()
        ks = k[:, h // g:h // g + 1].contiguous()
        vs = v[:, h // g:h // g + 1].contiguous()
        out.append(tune_layer(p, qs, ks, vs, band, **kw))
    return out
