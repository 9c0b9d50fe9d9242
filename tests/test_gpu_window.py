"""GPU parity of llama_attn_prefill_window (marked gpu).

Causal attention in which query i sees keys i - window < j <= i.  The oracle
computes it as causal attention plus an additive mask of -inf below the
window; pins: a window of seq keys or more is plain causal attention (the
output is bit-identical to llama_attn_prefill), and a window of one key makes
every output row its own value row.
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
    # (bsz, S, H, Hkv, D, window)
    (1, 385, 8, 2, 128, 100),    # window shorter than a tile: whole tiles skipped
    (2, 300, 8, 8, 64, 128),     # window of exactly one tile
    (1, 513, 16, 2, 128, 200),
    (1, 256, 6, 3, 128, 129),    # odd group: a CTA's two units start at different tiles
    (1, 600, 4, 4, 128, 250),    # MHA: units are adjacent position blocks
    (2, 77, 4, 4, 128, 5),
]


def _window_mask(S, window):
    i = torch.arange(S).view(S, 1)
    j = torch.arange(S).view(1, S)
    m = torch.zeros(1, 1, S, S, dtype=torch.float32)
    return m.masked_fill(j <= i - window, float("-inf"))


def _run(cfg, x, window):
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    cos, sin = api.rope_table(x["pos"].to(dev), cfg.head_dim, cfg.theta, cfg.factor)
    out = api.prefill_window(q, k, v, cos, sin, window=window, scale=cfg.scale)
    torch.cuda.synchronize()
    assert api.device_status() == api.LLAMA_OK
    return out, (q, k, v, cos, sin)


def _check(out, ref, what, report=False):
    g = out.float().cpu().double().numpy()
    sel = ~np.isnan(ref)
    assert sel.any()
    assert np.all(np.isfinite(g[sel])), f"{what}: non-finite output"
    err = np.abs(g[sel] - ref[sel])
    assert err.max() <= BF16_MAX, f"{what}: max abs {err.max():.3e}"
    assert err.mean() <= BF16_MEAN, f"{what}: mean abs {err.mean():.3e}"
    if report:
        PARITY_REPORT.append((what, "bfloat16", float(err.max()), float(err.mean())))


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%dS%dH%dKV%dD%dW%d" % c)
def test_prefill_window_matches_oracle(case):
    b, S, H, Hkv, D, window = case
    cfg, x = W.small_prefill(b, S, H, Hkv, D, torch.bfloat16, causal=True, rope=True,
                             seed=S + window)
    out, _ = _run(cfg, x, window)
    mask = _window_mask(S, window).expand(b, 1, S, S).contiguous()
    ref = oracle.prefill(x["q"], x["k"], x["v"], x["pos"], theta=cfg.theta, factor=cfg.factor,
                         scale=cfg.scale, causal=True, mask=mask)
    _check(out, ref, str(case))


@pytest.mark.parametrize("window", [300, 301, 10000])
def test_prefill_window_of_seq_or_more_is_causal_bitwise(window):
    cfg, x = W.small_prefill(1, 300, 8, 2, 128, torch.bfloat16, causal=True, rope=True, seed=3)
    out, (q, k, v, cos, sin) = _run(cfg, x, window)
    ref = api.prefill(q, k, v, cos, sin, causal=True, scale=cfg.scale)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_prefill_window_of_one_key_returns_v():
    b, S, H, Hkv, D = 2, 333, 8, 2, 128
    cfg, x = W.small_prefill(b, S, H, Hkv, D, torch.bfloat16, causal=True, rope=True, seed=9)
    out, _ = _run(cfg, x, 1)
    got = out.cpu().view(b, S, H, D)
    g = H // Hkv
    for h in range(H):
        assert torch.equal(got[:, :, h].view(torch.int16), x["v"][:, :, h // g].view(torch.int16))


def test_prefill_window_llama70b_shape_sampled_rows():
    # the 70B-shaped workload with a 4096-key window: every head, three row windows
    cfg = W.LLAMA70B
    window = 4096
    x = W.prefill_inputs(cfg)
    out, _ = _run(cfg, x, window)
    S = cfg.seq
    mask = _window_mask(S, window)
    ref = np.full(out.shape, np.nan)
    for lo, hi in [(0, 130), (S // 2 - 65, S // 2 + 65), (S - 130, S)]:
        part = oracle.prefill(x["q"], x["k"], x["v"], x["pos"], theta=cfg.theta, factor=cfg.factor,
                              scale=cfg.scale, causal=True, mask=mask, rows=(lo, hi))
        ref[:, lo:hi] = part[:, lo:hi]
    _check(out, ref, "llama70b window 4096 (sampled rows)", report=True)
