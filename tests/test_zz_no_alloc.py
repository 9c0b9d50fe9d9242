"""Decode for callers that cannot allocate device memory (GPU).

Some integrations hand the library nothing but their input and output
buffers: hosts that reserve all device memory up front and forbid any further
cudaMalloc, or plugin interfaces that offer no workspace.  For them
llama_attn_decode_noalloc runs the regular split-KV decode on a fixed scratch
array that lives inside the library.  These tests call it through the C ABI,
on two calls in a row with different problems (the second call reuses the
scratch the first one left), and require:
  - bit-identity with llama_attn_decode given a caller workspace: the two entry
    points run the same kernels on the same inputs, only the scratch differs;
  - agreement with the fp64 oracle on the decode workload's shape, within the
    bf16 tolerance of the other parity tests.
This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle
from llama_gqa_causal_b200 import api, workloads as W

pytestmark = pytest.mark.gpu

BF16_MAX = 2e-2
BF16_MEAN = 2e-3


def _problem(cfg, **kw):
    dev = torch.device("cuda")
    x = W.decode_inputs(cfg, **kw)
    t = {n: x[n].to(dev) for n in ("q", "k_cache", "v_cache", "lens")}
    cos, sin = api.rope_table(x["qpos"].view(-1, 1).to(dev), cfg.head_dim, cfg.theta, cfg.factor)
    t["cos"], t["sin"] = cos.view(cfg.bsz, -1), sin.view(cfg.bsz, -1)
    return cfg, t, x


def _close_to_oracle(out, cfg, x):
    ref = oracle.decode(x["q"], x["k_cache"], x["v_cache"], x["lens"], x["qpos"],
                        theta=cfg.theta, factor=cfg.factor, scale=cfg.scale)
    g = out.float().cpu().double().numpy().reshape(ref.shape)
    assert np.all(np.isfinite(g))
    err = np.abs(g - ref)
    assert err.max() <= BF16_MAX and err.mean() <= BF16_MEAN, (err.max(), err.mean())


def test_noalloc_decode_matches_workspace_decode_on_two_calls():
    big = _problem(W.DECODE70B)  # b32 H64 Hkv8 D128, lengths in [512, 4096], NaN tails
    small_cfg = W.DecodeConfig("small", 4, 16, 2, 128, 1100, 1, 1100, torch.bfloat16, seed=77)
    small = _problem(small_cfg, lens=torch.tensor([0, 1, 640, 1100], dtype=torch.int32))
    refs = []
    for cfg, t, _ in (big, small):
        refs.append(api.decode(t["q"], t["k_cache"], t["v_cache"], t["lens"], t["cos"], t["sin"],
                               scale=cfg.scale))
    outs = []
    for cfg, t, _ in (big, small):  # two calls in a row on the shared scratch
        out = torch.empty(cfg.bsz, cfg.n_heads * cfg.head_dim, device="cuda", dtype=cfg.dtype)
        outs.append(api.decode_noalloc(t["q"], t["k_cache"], t["v_cache"], t["lens"], t["cos"],
                                       t["sin"], scale=cfg.scale, out=out))
    torch.cuda.synchronize()
    assert api.device_status() == api.LLAMA_OK
    for o, r in zip(outs, refs):
        assert torch.equal(o, r)
    assert torch.all(outs[1][0].float() == 0)  # empty cache row
    _close_to_oracle(outs[0], big[0], big[2])
    _close_to_oracle(outs[1], small[0], small[2])


def test_noalloc_rejects_requests_beyond_its_static_scratch():
    lib = api.load()
    fake = 0x10000  # never dereferenced: the request is refused on the host
    # (1024 x 64 heads + 2048) partial rows x 132 floats + the prefix = 35.7 MB > 16 MiB
    st = lib.llama_attn_decode_noalloc(fake, fake, fake, fake, None, None, 1024, 64, 8, 4096, 128,
                                       0.088, fake, api.LLAMA_DT_BF16, None)
    assert st == api.LLAMA_ERR_INVALID_ARG
