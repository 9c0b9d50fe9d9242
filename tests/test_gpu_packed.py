"""GPU parity of llama_attn_prefill_packed (marked gpu).

Packed sequences: sequence s holds tokens [cu[s], cu[s+1]) of [T, H, D]
tensors, each token at its own position within its sequence.  Expected: each
sequence equals the fp64 oracle's attention over that sequence alone.  Pins:
one sequence of S tokens is bit-identical to llama_attn_prefill with b = 1,
and the same sequences laid out as a right-padded batch give bit-identical
rows through llama_attn_prefill_varlen (the tiles start at each sequence's
first token in both layouts).
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import PARITY_REPORT
from llama_gqa_causal_b200 import api, workloads as W

pytestmark = pytest.mark.gpu

BF16_MAX = 2e-2
BF16_MEAN = 2e-3
THETA = 10000.0

CASES = [
    # (lens, H, Hkv, D, causal)
    ([100, 1, 257, 130], 8, 2, 128, True),
    ([128, 128, 300], 16, 2, 128, True),    # sequence boundaries on tile boundaries
    ([77, 200, 5], 4, 4, 64, False),        # non-causal: later sequences' keys stay out
    ([385, 64], 6, 3, 128, True),           # odd group
]


def _packed_inputs(lens, H, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    T = sum(lens)
    q = W.normal((T, H, D), torch.bfloat16, g)
    k = W.normal((T, Hkv, D), torch.bfloat16, g)
    v = W.normal((T, Hkv, D), torch.bfloat16, g)
    pos = torch.cat([torch.arange(n, dtype=torch.int64) for n in lens])
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    return q, k, v, pos, cu


def _run(q, k, v, pos, cu, max_seqlen, causal, scale):
    dev = torch.device("cuda")
    T, H, D = q.shape
    cos, sin = api.rope_table(pos.view(1, -1).to(dev), D, THETA, 1.0)
    out = api.prefill_packed(q.to(dev), k.to(dev), v.to(dev), cu.to(dev), max_seqlen,
                             cos.view(T, D), sin.view(T, D), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert api.device_status() == api.LLAMA_OK
    return out.cpu()


@pytest.mark.parametrize("case", CASES, ids=lambda c: "n%dH%dKV%dD%d" % (len(c[0]), c[1], c[2], c[3]))
def test_prefill_packed_matches_oracle_per_sequence(case):
    lens, H, Hkv, D, causal = case
    q, k, v, pos, cu = _packed_inputs(lens, H, Hkv, D, seed=sum(lens) + H)
    scale = 1.0 / np.sqrt(D)
    out = _run(q, k, v, pos, cu, max(lens), causal, scale)
    errs = []
    for s, n in enumerate(lens):
        a = int(cu[s])
        ref = oracle.prefill(q[None, a:a + n], k[None, a:a + n], v[None, a:a + n],
                             pos[None, a:a + n], theta=THETA, scale=scale, causal=causal)
        g = out[a:a + n].float().double().numpy()
        assert np.all(np.isfinite(g)), f"sequence {s}: non-finite output"
        errs.append(np.abs(g - ref[0]).reshape(-1))
    err = np.concatenate(errs)
    assert err.max() <= BF16_MAX, f"{case}: max abs {err.max():.3e}"
    assert err.mean() <= BF16_MEAN, f"{case}: mean abs {err.mean():.3e}"


def test_prefill_packed_one_sequence_is_prefill_bitwise():
    lens, H, Hkv, D = [300], 8, 2, 128
    q, k, v, pos, cu = _packed_inputs(lens, H, Hkv, D, seed=21)
    scale = 1.0 / np.sqrt(D)
    out = _run(q, k, v, pos, cu, 300, True, scale)
    dev = torch.device("cuda")
    cos, sin = api.rope_table(pos.view(1, -1).to(dev), D, THETA, 1.0)
    ref = api.prefill(q[None].to(dev), k[None].to(dev), v[None].to(dev), cos, sin, causal=True,
                      scale=scale).cpu()
    assert torch.equal(out.view(torch.int16), ref[0].view(torch.int16))


def test_prefill_packed_equals_padded_batch_rows_bitwise():
    lens, H, Hkv, D = [100, 257, 130], 8, 2, 128
    q, k, v, pos, cu = _packed_inputs(lens, H, Hkv, D, seed=22)
    scale = 1.0 / np.sqrt(D)
    out = _run(q, k, v, pos, cu, max(lens), True, scale)
    S, b = max(lens), len(lens)
    qp = torch.zeros(b, S, H, D, dtype=q.dtype)
    kp = torch.zeros(b, S, Hkv, D, dtype=k.dtype)
    vp = torch.zeros(b, S, Hkv, D, dtype=v.dtype)
    for s, n in enumerate(lens):
        a = int(cu[s])
        qp[s, :n], kp[s, :n], vp[s, :n] = q[a:a + n], k[a:a + n], v[a:a + n]
    dev = torch.device("cuda")
    ppos = torch.arange(S, dtype=torch.int64).view(1, S).expand(b, S).contiguous()
    cos, sin = api.rope_table(ppos.to(dev), D, THETA, 1.0)
    ref = api.prefill_varlen(qp.to(dev), kp.to(dev), vp.to(dev),
                             torch.tensor(lens, dtype=torch.int32, device=dev), cos, sin,
                             causal=True, scale=scale).cpu()
    for s, n in enumerate(lens):
        a = int(cu[s])
        assert torch.equal(out[a:a + n].view(torch.int16), ref[s, :n].view(torch.int16))


def test_prefill_packed_llama7b_shape_sampled_rows():
    # the 7B head shape with four packed sequences of mixed length
    cfg = W.LLAMA7B
    lens = [4096, 2085, 700, 1]
    q, k, v, pos, cu = _packed_inputs(lens, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, seed=23)
    out = _run(q, k, v, pos, cu, max(lens), True, cfg.scale)
    errs = []
    for s, n in enumerate(lens):
        a = int(cu[s])
        for lo, hi in sorted({(0, min(n, 130)), (max(0, n - 130), n)}):
            ref = oracle.prefill(q[None, a:a + n], k[None, a:a + n], v[None, a:a + n],
                                 pos[None, a:a + n], theta=THETA, scale=cfg.scale, causal=True,
                                 rows=(lo, hi))
            errs.append(np.abs(out[a + lo:a + hi].float().double().numpy() - ref[0, lo:hi]).reshape(-1))
    err = np.concatenate(errs)
    assert err.max() <= BF16_MAX and err.mean() <= BF16_MEAN
    PARITY_REPORT.append(("llama7b packed (sampled rows)", "bfloat16", float(err.max()),
                          float(err.mean())))
