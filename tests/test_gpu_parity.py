"""GPU-vs-oracle parity through the C ABI (marked gpu).

Inputs come from llama_gqa_causal_b200.workloads (seeded, drawn on the CPU,
cast to the workload dtype); the very same bytes go to the fp64 oracle and to
the device.  Tolerances:
  fp32 inputs: max |gpu - oracle| <= 1e-5
  bf16 inputs: max |gpu - oracle| <= 2e-2 and mean |gpu - oracle| <= 2e-3
At the full workload sizes the oracle computes every head on sampled row
windows that cross tile boundaries (first, middle and last rows), covering
every K/V group.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import PARITY_REPORT
from llama_gqa_causal_b200 import api, workloads as W

pytestmark = pytest.mark.gpu

FP32_TOL = 1e-5
BF16_MAX = 2e-2
BF16_MEAN = 2e-3


def _check(gpu, ref, dtype, what="", report=False):
    g = gpu.detach().float().cpu().double().numpy()
    sel = ~np.isnan(ref)
    assert sel.any()
    assert np.all(np.isfinite(g[sel])), f"{what}: non-finite output"
    err = np.abs(g[sel] - ref[sel])
    if dtype == torch.float32:
        assert err.max() <= FP32_TOL, f"{what}: max abs {err.max():.3e}"
    else:
        assert err.max() <= BF16_MAX, f"{what}: max abs {err.max():.3e}"
        assert err.mean() <= BF16_MEAN, f"{what}: mean abs {err.mean():.3e}"
    if report:
        PARITY_REPORT.append((what, str(dtype).split(".")[-1], float(err.max()), float(err.mean())))
    return err.max(), err.mean()


def _gpu_prefill(cfg, x, causal=None, mask=None):
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    cos = sin = None
    if x["pos"] is not None:
        cos, sin = api.rope_table(x["pos"].to(dev), cfg.head_dim, cfg.theta, cfg.factor)
    m = None if mask is None else mask.to(dev).contiguous()
    out = api.prefill(q, k, v, cos, sin, causal=cfg.causal if causal is None else causal,
                      scale=cfg.scale, mask=m)
    torch.cuda.synchronize()
    assert api.device_status() == api.LLAMA_OK
    return out


def _oracle_prefill(cfg, x, rows=None, mask=None, causal=None):
    return oracle.prefill(x["q"], x["k"], x["v"], x["pos"], theta=cfg.theta, factor=cfg.factor,
                          scale=cfg.scale, causal=cfg.causal if causal is None else causal,
                          mask=mask, rows=rows)


# ----------------------------------------------------------------------------- RoPE table

@pytest.mark.parametrize("D,factor", [(128, 1.0), (128, 2.0), (64, 1.0)])
def test_rope_table_matches_oracle(D, factor):
    pos = torch.cat([torch.arange(0, 8192), torch.randint(0, 1 << 20, (512,),
                                                          generator=torch.Generator().manual_seed(1))])
    cos, sin = api.rope_table(pos.view(1, -1).cuda(), D, 10000.0, factor)
    c, s = oracle.rope_cos_sin(pos.numpy(), D, 10000.0, factor)
    assert np.abs(cos[0].cpu().double().numpy() - c).max() < 2e-7
    assert np.abs(sin[0].cpu().double().numpy() - s).max() < 2e-7


@pytest.mark.parametrize("D,alpha", [(128, 1.0), (128, 4.0), (64, 8.0)])
def test_rope_table_ntk_matches_oracle(D, alpha):
    pos = torch.cat([torch.arange(0, 8192), torch.randint(0, 1 << 17, (512,),
                                                          generator=torch.Generator().manual_seed(2))])
    cos, sin = api.rope_table_ntk(pos.view(1, -1).cuda(), D, 10000.0, alpha)
    c, s = oracle.rope_cos_sin_ntk(pos.numpy(), D, 10000.0, alpha)
    assert np.abs(cos[0].cpu().double().numpy() - c).max() < 2e-7
    assert np.abs(sin[0].cpu().double().numpy() - s).max() < 2e-7


@pytest.mark.parametrize("D", [64, 128])
def test_rope_tables_repeat_their_first_half(D):
    # the prefill kernel reads only the first half of each row, which the
    # header requires to repeat in the second: both table entry points write
    # the two halves bit for bit alike
    pos = torch.randint(0, 1 << 20, (2, 300), generator=torch.Generator().manual_seed(3)).cuda()
    for cos, sin in (api.rope_table(pos, D, 10000.0, 2.0), api.rope_table_ntk(pos, D, 10000.0, 4.0)):
        assert torch.equal(cos[..., :D // 2], cos[..., D // 2:])
        assert torch.equal(sin[..., :D // 2], sin[..., D // 2:])


# ----------------------------------------------------------------------------- named workloads

def test_tiny_fp32_workload():
    cfg = W.TINY_FP32
    x = W.prefill_inputs(cfg)
    out = _gpu_prefill(cfg, x)
    _check(out, _oracle_prefill(cfg, x), torch.float32, cfg.name, report=True)


def test_mha_bf16_workload_shape_and_values():
    cfg = W.MHA_BF16
    x = W.prefill_inputs(cfg)
    out = _gpu_prefill(cfg, x)
    assert tuple(out.shape) == (4, 128, 4096)  # the tensor-parallel demo's full output shape
    _check(out, _oracle_prefill(cfg, x), torch.bfloat16, cfg.name, report=True)


def _windows(S):
    w = [(0, min(S, 130)), (S // 2 - 65, S // 2 + 65), (S - 130, S)]
    return [(max(0, a), min(S, b)) for a, b in w]


@pytest.mark.parametrize("name", ["llama7b", "llama70b"])
def test_full_size_prefill_workloads_sampled(name):
    cfg = W.PREFILL_CONFIGS[name]
    x = W.prefill_inputs(cfg)
    out = _gpu_prefill(cfg, x)
    ref = np.full(out.shape, np.nan)
    for lo, hi in _windows(cfg.seq):
        part = _oracle_prefill(cfg, x, rows=(lo, hi))
        ref[:, lo:hi] = part[:, lo:hi]
    _check(out, ref, torch.bfloat16, name + " (sampled rows)", report=True)


@pytest.mark.parametrize("name", ["llama7b", "llama70b"])
def test_full_size_prefill_every_row_of_a_head_per_kv_group(name):
    # every row of one query head per K/V group (the group's last head), so all
    # position blocks, diagonal tiles and K/V heads are compared in full
    cfg = W.PREFILL_CONFIGS[name]
    x = W.prefill_inputs(cfg)
    out = _gpu_prefill(cfg, x)
    g, D = cfg.n_heads // cfg.n_kv_heads, cfg.head_dim
    ref = np.full(out.shape, np.nan)
    for kvh in range(cfg.n_kv_heads):
        h = kvh * g + g - 1
        part = oracle.prefill(x["q"], x["k"], x["v"], x["pos"], theta=cfg.theta, factor=cfg.factor,
                              scale=cfg.scale, causal=cfg.causal, heads=(h, h + 1))
        ref[:, :, h * D:(h + 1) * D] = part[:, :, h * D:(h + 1) * D]
    _check(out, ref, torch.bfloat16, name + " (all rows, a head per K/V group)", report=True)


def test_decode70b_workload():
    cfg = W.DECODE70B
    x = W.decode_inputs(cfg)  # cache tail past each length is NaN
    dev = torch.device("cuda")
    cos, sin = api.rope_table(x["qpos"].view(-1, 1).to(dev), cfg.head_dim, cfg.theta, cfg.factor)
    out = api.decode(x["q"].to(dev), x["k_cache"].to(dev), x["v_cache"].to(dev), x["lens"].to(dev),
                     cos.view(cfg.bsz, cfg.head_dim), sin.view(cfg.bsz, cfg.head_dim),
                     scale=cfg.scale)
    torch.cuda.synchronize()
    ref = oracle.decode(x["q"], x["k_cache"], x["v_cache"], x["lens"], x["qpos"],
                        theta=cfg.theta, factor=cfg.factor, scale=cfg.scale)
    _check(out, ref, torch.bfloat16, cfg.name, report=True)
    assert api.device_status() == api.LLAMA_OK


# ----------------------------------------------------------------------------- small shapes

PREFILL_CASES = [
    # (bsz, S, H, Hkv, D, causal, rope)
    (1, 1, 4, 2, 128, True, True),
    (2, 77, 8, 8, 128, True, True),
    (1, 128, 8, 1, 128, True, True),
    (2, 200, 8, 2, 64, True, True),
    (1, 385, 16, 2, 128, True, True),
    (1, 385, 6, 3, 128, True, True),     # odd group: units straddle position blocks
    (3, 129, 4, 4, 64, False, True),
    (1, 256, 8, 8, 128, False, False),
    (2, 300, 12, 4, 128, False, True),
    (1, 1000, 8, 1, 128, True, True),    # MQA
]


@pytest.mark.parametrize("case", PREFILL_CASES, ids=lambda c: "b%dS%dH%dKV%dD%d%s%s" % (
    c[0], c[1], c[2], c[3], c[4], "c" if c[5] else "n", "r" if c[6] else ""))
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_prefill_small(case, dtype):
    b, S, H, Hkv, D, causal, rope = case
    cfg, x = W.small_prefill(b, S, H, Hkv, D, dtype, causal=causal, rope=rope, factor=2.0,
                             seed=hash(case) & 0xffff)
    out = _gpu_prefill(cfg, x)
    _check(out, _oracle_prefill(cfg, x), dtype, str(case))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("causal", [True, False])
def test_prefill_additive_mask(dtype, causal):
    cfg, x = W.small_prefill(2, 150, 8, 2, 128, dtype, causal=causal, rope=True, seed=31,
                             with_mask=True)
    out = _gpu_prefill(cfg, x, mask=x["mask"])
    _check(out, _oracle_prefill(cfg, x, mask=x["mask"]), dtype, "mask")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_prefill_fully_masked_row_is_zero(dtype):
    cfg, x = W.small_prefill(1, 140, 4, 4, 64, dtype, causal=False, rope=False, seed=32)
    m = torch.zeros(1, 1, 140, 140)
    m[0, 0, 5, :] = float("-inf")
    m[0, 0, 130, :] = float("-inf")
    out = _gpu_prefill(cfg, x, mask=m)
    o = out.float().cpu()
    assert torch.all(o[0, 5] == 0) and torch.all(o[0, 130] == 0)
    _check(out, _oracle_prefill(cfg, x, mask=m), dtype, "masked rows")


def test_prefill_ignores_memory_past_seq():
    # allocate more rows than seq and poison the excess: nothing past seq may be read
    cfg, x = W.small_prefill(1, 200, 8, 2, 128, torch.bfloat16, causal=True, seed=33)
    dev = torch.device("cuda")
    pad = 56
    big = {n: torch.cat([x[n], torch.full((1, pad) + x[n].shape[2:], float("nan"),
                                          dtype=x[n].dtype)], dim=1) for n in ("q", "k", "v")}
    cos, sin = api.rope_table(x["pos"].to(dev), 128, cfg.theta, cfg.factor)
    q, k, v = (big[n].to(dev) for n in ("q", "k", "v"))
    out = api.prefill(q[:, :200], k[:, :200], v[:, :200], cos, sin, causal=True, scale=cfg.scale)
    torch.cuda.synchronize()
    _check(out, _oracle_prefill(cfg, x), torch.bfloat16, "poisoned tail")


DECODE_CASES = [
    # (bsz, H, Hkv, D, L, lens)
    (4, 8, 2, 128, 100, [1, 37, 64, 100]),
    (3, 64, 8, 128, 1100, [512, 513, 1100]),
    (2, 16, 1, 128, 700, [0, 700]),          # MQA, an empty cache row
    (2, 32, 2, 64, 2000, [1024, 1999]),      # group 16: two head chunks
    (5, 12, 4, 128, 130, [63, 64, 65, 128, 129]),
    (300, 8, 8, 64, 96, None),              # prefix runs of several batch entries per thread
    (3, 8, 2, 128, 200, [0, 0, 0]),          # no work at all: zero output everywhere
    (4, 16, 2, 128, 300, [-3, 301, 1000, 150]),  # lengths outside [0, L] are clamped
    (4096, 8, 1, 64, 64, None),             # the largest batch the bf16 decode takes
    (2, 8, 1, 128, 32768, [32768, 20001]),  # long caches: shares of hundreds of chunks
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: "b%dH%dKV%dD%dL%d" % c[:5])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_decode_small(case, dtype):
    b, H, Hkv, D, L, lens = case
    if lens is None:
        lens = torch.randint(0, L + 1, (b,), generator=torch.Generator().manual_seed(b)).tolist()
    clamped = [min(max(n, 0), L) for n in lens]
    cfg, x = W.small_decode(b, H, Hkv, D, L, dtype, seed=sum(clamped) + H,
                            lens=torch.tensor(clamped, dtype=torch.int32))
    x["lens"] = torch.tensor(lens, dtype=torch.int32)  # the device sees the raw lengths
    dev = torch.device("cuda")
    cos, sin = api.rope_table(x["qpos"].view(-1, 1).to(dev), D, cfg.theta, cfg.factor)
    out = api.decode(x["q"].to(dev), x["k_cache"].to(dev), x["v_cache"].to(dev),
                     x["lens"].to(dev), cos.view(b, D), sin.view(b, D), scale=cfg.scale)
    torch.cuda.synchronize()
    ref = oracle.decode(x["q"], x["k_cache"], x["v_cache"], torch.tensor(clamped), x["qpos"],
                        theta=cfg.theta, factor=cfg.factor, scale=cfg.scale)
    if max(clamped) > 0:
        _check(out, ref, dtype, str(case))
    for i, n in enumerate(clamped):
        if n == 0:
            assert torch.all(out[i].float().cpu() == 0)


def test_prefill_long_sequence_sampled_rows():
    # S = 16384: the (batch, K/V head) pairs whose K/V fit in L2 run as bundles
    # of several pairs, and the last position blocks stream 128 K/V tiles
    cfg, x = W.small_prefill(2, 16384, 16, 2, 128, torch.bfloat16, causal=True, seed=43)
    out = _gpu_prefill(cfg, x)
    ref = np.full(out.shape, np.nan)
    for lo, hi in [(0, 64), (8160, 8224), (16320, 16384)]:
        part = _oracle_prefill(cfg, x, rows=(lo, hi))
        ref[:, lo:hi] = part[:, lo:hi]
    _check(out, ref, torch.bfloat16, "S 16384 (sampled rows)", report=True)


def test_decode_equals_last_prefill_row_on_gpu():
    # decode over the rotated cache of a prefill == that prefill's last row
    b, S, H, Hkv, D = 2, 333, 16, 2, 128
    cfg, x = W.small_prefill(b, S, H, Hkv, D, torch.bfloat16, causal=True, seed=40)
    dev = torch.device("cuda")
    cos, sin = api.rope_table(x["pos"].to(dev), D)
    pre = api.prefill(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), cos, sin, causal=True)
    # rotated keys from the oracle's fp64 RoPE, rounded to bf16 like a cache would hold them
    c, s = oracle.rope_cos_sin(x["pos"].numpy(), D)
    krot = oracle.rope_rotate(x["k"].double().numpy(), c.reshape(b, S, 1, D), s.reshape(b, S, 1, D))
    kc = torch.from_numpy(krot).to(torch.bfloat16).permute(0, 2, 1, 3).contiguous().to(dev)
    vc = x["v"].permute(0, 2, 1, 3).contiguous().to(dev)
    lens = torch.full((b,), S, dtype=torch.int32, device=dev)
    dec = api.decode(x["q"][:, S - 1].contiguous().to(dev), kc, vc, lens,
                     cos[:, S - 1].contiguous(), sin[:, S - 1].contiguous())
    torch.cuda.synchronize()
    diff = (dec.float() - pre[:, S - 1].float()).abs()
    assert diff.max().item() <= BF16_MAX and diff.mean().item() <= BF16_MEAN


def test_repeated_runs_are_bitwise_identical():
    cfg, x = W.small_prefill(1, 700, 16, 2, 128, torch.bfloat16, causal=True, seed=41)
    a = _gpu_prefill(cfg, x)
    b = _gpu_prefill(cfg, x)
    assert torch.equal(a, b)
    cfg2, y = W.small_decode(4, 64, 8, 128, 3000, torch.bfloat16, min_len=100, seed=42)
    dev = torch.device("cuda")
    args = (y["q"].to(dev), y["k_cache"].to(dev), y["v_cache"].to(dev), y["lens"].to(dev))
    d1 = api.decode(*args)
    d2 = api.decode(*args)
    torch.cuda.synchronize()
    assert torch.equal(d1, d2)


def test_decode_over_more_caches_than_the_tensor_map_memo_holds():
    # the library memoises 32 encoded tensor maps (a map is a pure function of
    # base address, dimensions, strides and box); 20 cache pairs need 40, so
    # the second pass, in reverse order, runs on maps evicted and encoded again
    dev = torch.device("cuda")
    b, H, Hkv, D, L = 2, 8, 2, 64, 200
    cases = []
    for i in range(20):
        cfg, x = W.small_decode(b, H, Hkv, D, L, torch.bfloat16, seed=500 + i)
        cos, sin = api.rope_table(x["qpos"].view(-1, 1).to(dev), D, cfg.theta, cfg.factor)
        cases.append((cfg, x, {n: x[n].to(dev) for n in ("q", "k_cache", "v_cache", "lens")},
                      cos.view(b, D), sin.view(b, D)))

    def run(case):
        cfg, _, d, cos, sin = case
        return api.decode(d["q"], d["k_cache"], d["v_cache"], d["lens"], cos, sin, scale=cfg.scale)

    first = [run(c) for c in cases]
    again = [run(c) for c in reversed(cases)][::-1]
    torch.cuda.synchronize()
    assert api.device_status() == api.LLAMA_OK
    for o1, o2 in zip(first, again):
        assert torch.equal(o1, o2)
    for i in (0, 19):
        cfg, x = cases[i][0], cases[i][1]
        ref = oracle.decode(x["q"], x["k_cache"], x["v_cache"], x["lens"], x["qpos"],
                            theta=cfg.theta, factor=cfg.factor, scale=cfg.scale)
        _check(first[i], ref, torch.bfloat16, f"memo case {i}")
