"""GPU parity of llama_attn_prefill_varlen (marked gpu).

A right-padded batch: entry b holds seq_lens[b] valid tokens.  The expected
output of each entry is the fp64 oracle's attention over that entry's valid
tokens alone; output rows at or past its length must be exactly zero.  The
padded rows of q, k and v are filled with NaN, so any read of them into a valid
row shows.  Pins: full lengths are bit-identical to llama_attn_prefill, and a
one-token entry returns its value row.
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

CASES = [
    # (bsz, S, H, Hkv, D, lens, causal)
    (3, 300, 8, 2, 128, [300, 1, 129], True),
    (2, 513, 16, 2, 128, [0, 400], True),           # an empty entry
    (4, 200, 4, 4, 64, [128, 127, 200, 65], False),  # non-causal: padded keys masked too
    (2, 385, 6, 3, 128, [384, 256], True),           # odd group: units straddle position blocks
    (3, 256, 8, 8, 128, [-5, 1000, 100], True),      # lengths outside [0, S] are clamped
]


def _poisoned(x, lens):
    y = dict(x)
    for n in ("q", "k", "v"):
        t = x[n].clone()
        for b, L in enumerate(lens):
            t[b, L:] = float("nan")
        y[n] = t
    return y


def _run(cfg, x, lens):
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    cos, sin = api.rope_table(x["pos"].to(dev), cfg.head_dim, cfg.theta, cfg.factor)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    out = api.prefill_varlen(q, k, v, sl, cos, sin, causal=cfg.causal, scale=cfg.scale)
    torch.cuda.synchronize()
    assert api.device_status() == api.LLAMA_OK
    return out.cpu(), (q, k, v, cos, sin)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%dS%dH%dKV%dD%d" % c[:5])
def test_prefill_varlen_matches_oracle_per_entry(case):
    b, S, H, Hkv, D, lens, causal = case
    valid = [min(max(n, 0), S) for n in lens]
    cfg, x = W.small_prefill(b, S, H, Hkv, D, torch.bfloat16, causal=causal, rope=True,
                             seed=S + sum(valid))
    xp = _poisoned(x, valid)
    out, _ = _run(cfg, xp, lens)
    errs = []
    for i, n in enumerate(valid):
        if n < S:
            assert torch.all(out[i, n:] == 0), f"entry {i}: padded output rows are not zero"
        if n == 0:
            continue
        sl = slice(i, i + 1)
        ref = oracle.prefill(x["q"][sl, :n], x["k"][sl, :n], x["v"][sl, :n], x["pos"][sl, :n],
                             theta=cfg.theta, factor=cfg.factor, scale=cfg.scale, causal=causal)
        g = out[i, :n].float().double().numpy()
        assert np.all(np.isfinite(g)), f"entry {i}: non-finite output"
        errs.append(np.abs(g - ref[0]))
    err = np.concatenate([e.reshape(-1) for e in errs])
    assert err.max() <= BF16_MAX, f"{case}: max abs {err.max():.3e}"
    assert err.mean() <= BF16_MEAN, f"{case}: mean abs {err.mean():.3e}"


def test_prefill_varlen_full_lengths_are_prefill_bitwise():
    cfg, x = W.small_prefill(2, 300, 8, 2, 128, torch.bfloat16, causal=True, rope=True, seed=4)
    out, (q, k, v, cos, sin) = _run(cfg, x, [300, 300])
    ref = api.prefill(q, k, v, cos, sin, causal=True, scale=cfg.scale).cpu()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_prefill_varlen_one_token_entry_returns_v():
    b, S, H, Hkv, D = 2, 160, 8, 2, 128
    cfg, x = W.small_prefill(b, S, H, Hkv, D, torch.bfloat16, causal=False, rope=True, seed=8)
    out, _ = _run(cfg, _poisoned(x, [1, 1]), [1, 1])
    got = out.view(b, S, H, D)
    g = H // Hkv
    for h in range(H):
        assert torch.equal(got[:, 0, h].view(torch.int16), x["v"][:, 0, h // g].view(torch.int16))
    assert torch.all(got[:, 1:] == 0)


def test_prefill_varlen_llama7b_shape_sampled_rows():
    # the 7B-shaped workload with the second entry padded to half its length
    cfg = W.LLAMA7B
    lens = [cfg.seq, cfg.seq // 2 + 37]
    x = _poisoned(W.prefill_inputs(cfg), lens)
    out, _ = _run(cfg, x, lens)
    clean = W.prefill_inputs(cfg)
    errs = []
    for i, n in enumerate(lens):
        assert torch.all(out[i, n:] == 0)
        for lo, hi in [(0, 130), (n - 130, n)]:
            sl = slice(i, i + 1)
            ref = oracle.prefill(clean["q"][sl, :n], clean["k"][sl, :n], clean["v"][sl, :n],
                                 clean["pos"][sl, :n], theta=cfg.theta, factor=cfg.factor,
                                 scale=cfg.scale, causal=True, rows=(lo, hi))
            errs.append(np.abs(out[i, lo:hi].float().double().numpy() - ref[0, lo:hi]))
    err = np.concatenate([e.reshape(-1) for e in errs])
    assert err.max() <= BF16_MAX and err.mean() <= BF16_MEAN
    PARITY_REPORT.append(("llama7b varlen (sampled rows)", "bfloat16", float(err.max()),
                          float(err.mean())))
