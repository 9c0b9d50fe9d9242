"""Second, independent fp64 restatement of the attention path, in pure Python.

TEST INFRASTRUCTURE (same import rule as the rest of ``oracle/``).  It is
written differently from the C oracle on purpose, so that the two agreeing on
tiny shapes is evidence about both:

* RoPE is applied pair by pair as a 2-D rotation of (x[i], x[i + D/2]) by the
  angle pos/factor * theta**(-2i/D) (RoFormer frequencies, the rotate-half
  pairing of the HF apply_rotary_pos_emb in the "LlamaAttention source
  walkthrough" page, step 3), instead of the elementwise cos/sin form;
* K/V heads are materialised with an explicit repeat_kv (step 4 of the same
  page) instead of indexing head h // group;
* the softmax is computed over the full score row with masked entries set to
  -inf, then normalised (steps 5.1-5.3), using only the ``math`` module.

Only for tiny inputs (nested lists / small arrays); it is O(S^2 D) Python.
"""
from __future__ import annotations

import math


def _rotate(vec, p, theta, factor):
    D = len(vec)
    h = D // 2
    out = list(vec)
    for i in range(h):
        ang = (p / factor) * theta ** (-2.0 * i / D)
        c, s = math.cos(ang), math.sin(ang)
        a, b = vec[i], vec[i + h]
        out[i] = a * c - b * s
        out[i + h] = b * c + a * s
    return out


def _repeat_kv(kv_heads, group):
    """[Hkv][S][D] -> [Hkv*group][S][D], each K/V head repeated ``group`` times."""
    out = []
    for head in kv_heads:
        for _ in range(group):
            out.append(head)
    return out


def _attend(qrow, keys, vals, allowed, scale, mask_row):
    scores = []
    for j, kr in enumerate(keys):
        if not allowed[j]:
            scores.append(-math.inf)
            continue
        s = scale * sum(a * b for a, b in zip(qrow, kr))
        if mask_row is not None:
            s += mask_row[j]
        scores.append(s)
    mx = max(scores)
    D = len(vals[0]) if vals else len(qrow)
    if mx == -math.inf:
        return [0.0] * D
    w = [0.0 if s == -math.inf else math.exp(s - mx) for s in scores]
    tot = sum(w)
    out = [0.0] * D
    for j, vr in enumerate(vals):
        if w[j] == 0.0:
            continue
        for d in range(D):
            out[d] += (w[j] / tot) * vr[d]
    return out


def prefill(q, k, v, pos=None, theta=10000.0, factor=1.0, scale=None, causal=True, mask=None):
    """q [b][S][H][D], k/v [b][S][Hkv][D] nested lists -> out [b][S][H*D]."""
    bsz, S, H, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv = len(k[0][0])
    group = H // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = []
    for b in range(bsz):
        # per-head sequences, [H][S][D], with RoPE applied to Q and K only
        qh = [[(_rotate(q[b][i][h], pos[b][i], theta, factor) if pos is not None else list(q[b][i][h]))
               for i in range(S)] for h in range(H)]
        kh = [[(_rotate(k[b][j][g], pos[b][j], theta, factor) if pos is not None else list(k[b][j][g]))
               for j in range(S)] for g in range(Hkv)]
        vh = [[list(v[b][j][g]) for j in range(S)] for g in range(Hkv)]
        kh = _repeat_kv(kh, group)
        vh = _repeat_kv(vh, group)
        rows = []
        for i in range(S):
            allowed = [(not causal) or (j <= i) for j in range(S)]
            mrow = mask[b][0][i] if mask is not None else None
            row = []
            for h in range(H):
                row.extend(_attend(qh[h][i], kh[h], vh[h], allowed, scale, mrow))
            rows.append(row)
        out.append(rows)
    return out


def decode(q, k_cache, v_cache, lens, qpos=None, theta=10000.0, factor=1.0, scale=None):
    """q [b][H][D], caches [b][Hkv][L][D] (keys already rotated) -> out [b][H*D]."""
    bsz, H, D = len(q), len(q[0]), len(q[0][0])
    Hkv = len(k_cache[0])
    group = H // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = []
    for b in range(bsz):
        n = lens[b]
        keys = _repeat_kv([k_cache[b][g][:n] for g in range(Hkv)], group)
        vals = _repeat_kv([v_cache[b][g][:n] for g in range(Hkv)], group)
        row = []
        for h in range(H):
            qr = _rotate(q[b][h], qpos[b], theta, factor) if qpos is not None else list(q[b][h])
            if n == 0:
                row.extend([0.0] * D)
            else:
                row.extend(_attend(qr, keys[h], vals[h], [True] * n, scale, None))
        out.append(row)
    return out
