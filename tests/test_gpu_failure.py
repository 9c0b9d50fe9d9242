"""Failure detection on the GPU without a fault (marked gpu).

Both failure paths of the library are driven through the C ABI:
  - a bounded device wait that runs out: the self-test kernel waits on a
    shared-memory barrier that nothing arrives on, with a 1 ms limit.  The
    kernel must return by itself, the device status word must then read
    LLAMA_ERR_DEVICE_TIMEOUT exactly once (reading clears it), and the context
    must stay usable: a decode run afterwards still matches the fp64 oracle;
  - a launch the CUDA runtime refuses on the host (an invalid block size):
    the call returns LLAMA_ERR_CUDA, nothing reaches the GPU, and the next
    library call works.
Nothing here faults, traps or hangs the GPU: the wait ends by construction.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from llama_gqa_causal_b200 import api, workloads as W

pytestmark = pytest.mark.gpu


def _decode_matches_oracle():
    cfg, x = W.small_decode(3, 16, 2, 128, 700, torch.bfloat16, seed=5,
                            lens=torch.tensor([1, 300, 700], dtype=torch.int32))
    dev = torch.device("cuda")
    cos, sin = api.rope_table(x["qpos"].view(-1, 1).to(dev), 128, cfg.theta, cfg.factor)
    out = api.decode(x["q"].to(dev), x["k_cache"].to(dev), x["v_cache"].to(dev), x["lens"].to(dev),
                     cos.view(3, 128), sin.view(3, 128), scale=cfg.scale)
    torch.cuda.synchronize()
    assert api.device_status() == api.LLAMA_OK
    ref = oracle.decode(x["q"], x["k_cache"], x["v_cache"], x["lens"], x["qpos"],
                        theta=cfg.theta, factor=cfg.factor, scale=cfg.scale)
    err = np.abs(out.float().cpu().double().numpy() - ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3


def test_device_wait_that_runs_out_is_reported_once_and_the_context_survives():
    torch.cuda.synchronize()
    assert api.device_status() == api.LLAMA_OK  # nothing pending from earlier tests
    t = time.perf_counter()
    assert api.selftest_wait_timeout(1000) == api.LLAMA_OK  # 1 ms limit
    st = api.device_status()  # synchronises: the kernel has returned by itself
    elapsed = time.perf_counter() - t
    assert st == api.LLAMA_ERR_DEVICE_TIMEOUT
    assert elapsed < 5.0
    assert api.device_status() == api.LLAMA_OK  # reading cleared the word
    # two expiries before one read still report a single timeout
    assert api.selftest_wait_timeout(1000) == api.LLAMA_OK
    assert api.selftest_wait_timeout(1000) == api.LLAMA_OK
    assert api.device_status() == api.LLAMA_ERR_DEVICE_TIMEOUT
    assert api.device_status() == api.LLAMA_OK
    _decode_matches_oracle()


def test_refused_launch_surfaces_as_cuda_error_and_the_context_survives():
    torch.cuda.synchronize()
    assert api.selftest_launch_error() == api.LLAMA_ERR_CUDA
    assert api.device_status() == api.LLAMA_OK  # no device-side failure was recorded
    _decode_matches_oracle()
