"""float64 CPU oracle of the routed mixture-of-experts FFN step.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It shares no code with the CUDA path; its inputs come from the
seeded generator package ``synth`` only.

What is computed, and where it comes from:

* Weights use the self-defined block format: 32 consecutive weights along the
  reduction axis share an fp16 scale ``d`` and fp16 min ``m``; ``w = d*q + m``
  with 2-bit (Q2) or 4-bit (Q4) codes ``q``.  The pages name only third-party
  GGUF quant types (pyshine Strata tour, "How It Works"); the format here is
  the one the workload definitions fix.
* Router: logits ``l = Wr x (+ b)``; the ``k`` largest are selected (ten
  experts per token in the pyshine Strata tour's end-to-end walk-through;
  router kernel ``router_top10.cu``, same page, "Understanding the
  Architecture"), ties to the lower expert index; gates are the softmax over
  the selected logits, which equals softmax over all experts followed by
  renormalisation over the selection.
* Expert FFN: ``h = silu(Wg x) * (Wu x)``, ``y_e = Wd h`` with
  ``silu(a) = a / (1 + exp(-a))``.
* Combine: ``y = sum_j g_j y_{e_j}`` in slot order, applied once on the device
  side of the engine (the device-side ``moe_combine`` of the pyshine Strata
  tour, "Understanding the Architecture").
* Residual stack: ``x <- RMSNorm(x + y)`` with ``eps = 1e-6`` and no learned
  gain (the gated residual stream shared by all blocks, same section; the
  reduced form is the plainest reading).

Logits are certified: they are computed with a float64 matrix product, and
every token whose top-(k+1) ordering could be changed by that product's
rounding error is recomputed with correctly rounded sums (``math.fsum`` of
exact products; fp32 x fp32 and bf16 x fp32 products are exact in float64).
"""
from __future__ import annotations

import math

import numpy as np

U53 = 2.0 ** -53


# ---------------------------------------------------------------- format ----
def unpack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """uint8 [rows, K*bits/8] -> int64 [rows, K] codes.

    Q2: code j in byte j//4 at bits 2*(j%4).  Q4: code j in byte j//2, low
    nibble for even j.
    """
    codes = np.asarray(codes, dtype=np.uint8)
    rows, nb = codes.shape
    per = 8 // bits
    mask = (1 << bits) - 1
    q = np.empty((rows, nb, per), dtype=np.int64)
    for p in range(per):
        q[:, :, p] = (codes >> (bits * p)) & mask
    return q.reshape(rows, nb * per)


def dequantize(codes: np.ndarray, scales: np.ndarray, bits: int) -> np.ndarray:
    """Canonical block-quantised matrix -> float64 [rows, K]: w = d*q + m.

    ``scales`` is uint16 [rows, K/32, 2] holding fp16 bit patterns of (d, m);
    fp16 -> float64 is exact, so every w here is the format's exact value.
    """
    q = unpack_codes(codes, bits).astype(np.float64)
    rows, K = q.shape
    s = np.asarray(scales, dtype=np.uint16).reshape(rows, K // 32, 2)
    d = s[:, :, 0].view(np.float16).astype(np.float64)
    m = s[:, :, 1].view(np.float16).astype(np.float64)
    w = q.reshape(rows, K // 32, 32) * d[:, :, None] + m[:, :, None]
    return w.reshape(rows, K)


# ---------------------------------------------------------------- router ----
def _exact_logits_row(x: np.ndarray, Wr: np.ndarray, b) -> np.ndarray:
    """Correctly rounded logits of one token (float64 [E])."""
    prods = Wr * x[None, :]          # exact: each factor has <= 24 significant bits
    out = np.empty(Wr.shape[0], dtype=np.float64)
    for e in range(Wr.shape[0]):
        terms = prods[e].tolist()
        if b is not None:
            terms.append(float(b[e]))
        out[e] = math.fsum(terms)
    return out


def order_key(l: np.ndarray) -> np.ndarray:
    """Experts sorted by (logit descending, index ascending)."""
    E = l.shape[0]
    return np.lexsort((np.arange(E), -l))


def logits(x: np.ndarray, Wr: np.ndarray, bias, k: int) -> np.ndarray:
    """Certified router logits float64 [T, E].

    ``x`` [T, H] (fp32 or bf16-valued), ``Wr`` [E, H] fp32, ``bias`` [E] or
    None.  A token is recomputed exactly when two of its top-(k+1) logits are
    closer than twice the float64 product's error bound
    ``gamma_H * sum_h |x_h W_eh|`` with ``gamma_H = H u / (1 - H u)``.
    """
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(Wr, dtype=np.float64)
    T, H = x.shape
    E = W.shape[0]
    l = x @ W.T
    absum = np.abs(x) @ np.abs(W).T
    if bias is not None:
        b = np.asarray(bias, dtype=np.float64)
        l = l + b[None, :]
        absum = absum + np.abs(b)[None, :]
    n = H + 2
    gamma = n * U53 / (1.0 - n * U53)
    bound = 1.01 * gamma * absum.max(axis=1)          # per token, all experts
    kk = min(k + 1, E)
    for t in range(T):
        top = np.sort(l[t])[::-1][:kk]
        if kk > 1 and np.min(top[:-1] - top[1:]) <= 2.0 * bound[t]:
            l[t] = _exact_logits_row(x[t], W, None if bias is None else bias)
    return l


def topk(l_row: np.ndarray, k: int) -> np.ndarray:
    """The ``k`` largest logits' expert indices, ties to the lower index."""
    return order_key(l_row)[:k].astype(np.int32)


def gates(l_row: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """g_j = exp(l_j - max_sel) / sum_sel exp(l_i - max_sel)."""
    sel = l_row[idx]
    e = np.exp(sel - sel.max())
    return e / e.sum()


def gates_via_full_softmax(l_row: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Softmax over all experts, then pick the selection and renormalise."""
    p = np.exp(l_row - l_row.max())
    p = p / p.sum()
    s = p[idx]
    return s / s.sum()


def route(x: np.ndarray, Wr: np.ndarray, bias, k: int):
    """(idx int32 [T, k], gate float64 [T, k], logits float64 [T, E])."""
    l = logits(x, Wr, bias, k)
    T = l.shape[0]
    idx = np.empty((T, k), dtype=np.int32)
    g = np.empty((T, k), dtype=np.float64)
    for t in range(T):
        idx[t] = topk(l[t], k)
        g[t] = gates(l[t], idx[t])
    return idx, g, l


# ------------------------------------------------------------------- FFN ----
def silu(a: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-a))


def expert_ffn(x: np.ndarray, Wg: np.ndarray, Wu: np.ndarray, Wd: np.ndarray) -> np.ndarray:
    """One expert on tokens x [n, H]: Wd (silu(Wg x) * (Wu x)) -> [n, H]."""
    x = np.asarray(x, dtype=np.float64)
    h = silu(x @ Wg.T) * (x @ Wu.T)
    return h @ Wd.T


def combine(y_slots: np.ndarray, g: np.ndarray) -> np.ndarray:
    """y = sum_j g_j y_j in slot order; y_slots [k, H], g [k]."""
    y = np.zeros(y_slots.shape[1], dtype=np.float64)
    for j in range(y_slots.shape[0]):
        y = y + g[j] * y_slots[j]
    return y


def moe_layer(x: np.ndarray, idx: np.ndarray, g: np.ndarray, get_expert) -> np.ndarray:
    """Routed FFN + combine for a batch.

    ``get_expert(e)`` returns float64 (Wg [I,H], Wu [I,H], Wd [H,I]).  Each
    routed expert runs once on the tokens that chose it; the results are
    combined per token in slot order.
    """
    x = np.asarray(x, dtype=np.float64)
    T, k = idx.shape
    out = {}
    for e in sorted(set(int(v) for v in idx.ravel())):
        toks = [t for t in range(T) if e in idx[t]]
        ye = expert_ffn(x[toks], *get_expert(e))
        for r, t in enumerate(toks):
            out[(t, e)] = ye[r]
    y = np.empty((T, x.shape[1]), dtype=np.float64)
    for t in range(T):
        y[t] = combine(np.stack([out[(t, int(e))] for e in idx[t]]), g[t])
    return y


def rmsnorm_residual(x: np.ndarray, y: np.ndarray, eps: float) -> np.ndarray:
    """x' = z / sqrt(mean(z^2) + eps), z = x + y, per token."""
    z = np.asarray(x, dtype=np.float64) + np.asarray(y, dtype=np.float64)
    return z / np.sqrt(np.mean(z * z, axis=-1, keepdims=True) + eps)


def stack(x0: np.ndarray, layers, k: int, eps: float, residual: bool = True):
    """Run the layer stack from ``x0``.

    ``layers`` is a sequence of ``(Wr, bias, get_expert)``.  Returns the final
    activations and per-layer records ``(x_in, idx, gate, y)``.
    """
    x = np.asarray(x0, dtype=np.float64)
    recs = []
    for Wr, b, get_expert in layers:
        idx, g, _ = route(x, Wr, b, k)
        y = moe_layer(x, idx, g, get_expert)
        recs.append((x, idx, g, y))
        x = rmsnorm_residual(x, y, eps) if residual else y
    return x, recs


def rel_rms(a: np.ndarray, ref: np.ndarray) -> float:
    """||a - ref||_2 / ||ref||_2 over all elements."""
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.sqrt(np.sum(ref * ref))
    return float(np.sqrt(np.sum((a - ref) ** 2)) / den) if den > 0 else float(np.sqrt(np.sum(a * a)))
