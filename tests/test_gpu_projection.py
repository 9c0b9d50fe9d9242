"""GPU parity of the projection GEMMs around attention (marked gpu).

llama_attn_qkv_rope: x . W_qkv^T split into q/k/v heads, q and k rotated with
the token's cos/sin row.  Expected: the fp64 product (numpy matmul as the
library routine) split by head, q and k rotated by the oracle's RoPE.
llama_attn_out_proj: attn . W_o^T against the fp64 product.  The whole block
(projections, attention on the pre-rotated q and k, output projection) is
checked against the oracle's chain.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import PARITY_REPORT
from llama_gqa_causal_b200 import api, workloads as W

pytestmark = pytest.mark.gpu

THETA = 10000.0


def _close(got, want, what, max_tol=2e-2, mean_tol=2e-3):
    g = got.float().cpu().double().numpy()
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - want)
    assert err.max() <= max_tol, f"{what}: max abs {err.max():.3e}"
    assert err.mean() <= mean_tol, f"{what}: mean abs {err.mean():.3e}"
    return err


def _weights(n_out, n_in, g):
    # N(0, 1/n_in) so that the projections stay near unit scale
    return (torch.randn(n_out, n_in, generator=g) / np.sqrt(n_in)).to(torch.bfloat16)


QKV_CASES = [
    # (tokens, hidden, H, Hkv, D, rope)
    (200, 512, 8, 2, 128, True),    # ragged token count (two M tiles, the second partial)
    # 20 x 24 = 480 tiles: every CTA of the persistent grid takes three or four,
    # so both TMEM accumulator buffers are reused; 20 row tiles = one group of
    # 16 and a short group of 4, the last row tile ragged
    (2500, 256, 32, 8, 128, True),
    (130, 256, 4, 4, 64, True),     # head_dim 64: four heads per 256-column tile
    (1, 128, 8, 1, 128, True),      # one token, MQA
    (300, 1000, 4, 2, 128, False),  # no RoPE; hidden not a multiple of the 64-wide K block
]


def _qkv_expected(x, w, pos, H, Hkv, D, rope):
    y = x.double().numpy() @ w.double().numpy().T  # [T, (H + 2Hkv) D]
    T = y.shape[0]
    q = y[:, :H * D].reshape(T, H, D)
    k = y[:, H * D:(H + Hkv) * D].reshape(T, Hkv, D)
    v = y[:, (H + Hkv) * D:].reshape(T, Hkv, D)
    if rope:
        c, s = oracle.rope_cos_sin(pos.numpy(), D, THETA, 1.0)
        q = oracle.rope_rotate(q, c[:, None, :], s[:, None, :])
        k = oracle.rope_rotate(k, c[:, None, :], s[:, None, :])
    return q, k, v


@pytest.mark.parametrize("case", QKV_CASES, ids=lambda c: "T%d_h%d_H%d_KV%d_D%d" % c[:5])
def test_qkv_rope_matches_oracle(case):
    T, hidden, H, Hkv, D, rope = case
    g = torch.Generator().manual_seed(T + hidden)
    x = W.normal((T, hidden), torch.bfloat16, g)
    w = _weights((H + 2 * Hkv) * D, hidden, g)
    pos = torch.randint(0, 8192, (T,), generator=g)
    dev = torch.device("cuda")
    cos = sin = None
    if rope:
        cos, sin = api.rope_table(pos.view(1, -1).to(dev), D, THETA, 1.0)
        cos, sin = cos.view(T, D), sin.view(T, D)
    q, k, v = api.qkv_rope(x.to(dev), w.to(dev), H, Hkv, D, cos, sin)
    torch.cuda.synchronize()
    assert api.device_status() == api.LLAMA_OK
    eq, ek, ev = _qkv_expected(x, w, pos, H, Hkv, D, rope)
    _close(q, eq, f"{case} q")
    _close(k, ek, f"{case} k")
    _close(v, ev, f"{case} v")


@pytest.mark.parametrize("T,d_in,d_out", [(200, 512, 520), (1, 64, 256), (257, 1000, 768),
                                          (3000, 384, 4096)])  # 24 x 16 tiles
def test_out_proj_matches_oracle(T, d_in, d_out):
    g = torch.Generator().manual_seed(T + d_in + d_out)
    a = W.normal((T, d_in), torch.bfloat16, g)
    w = _weights(d_out, d_in, g)
    y = api.out_proj(a.cuda(), w.cuda())
    torch.cuda.synchronize()
    assert api.device_status() == api.LLAMA_OK
    _close(y, a.double().numpy() @ w.double().numpy().T, f"out_proj {T}x{d_in}x{d_out}")


def test_attention_block_matches_oracle_chain():
    # projections with RoPE in the GEMM epilogue -> causal GQA attention on the
    # pre-rotated q/k (no cos/sin) -> output projection
    T, hidden, H, Hkv, D = 300, 512, 8, 2, 128
    g = torch.Generator().manual_seed(31)
    x = W.normal((T, hidden), torch.bfloat16, g)
    w_qkv = _weights((H + 2 * Hkv) * D, hidden, g)
    w_o = _weights(hidden, H * D, g)
    pos = torch.arange(T)
    dev = torch.device("cuda")
    cos, sin = api.rope_table(pos.view(1, -1).to(dev), D, THETA, 1.0)
    q, k, v = api.qkv_rope(x.to(dev), w_qkv.to(dev), H, Hkv, D, cos.view(T, D), sin.view(T, D))
    attn = api.prefill(q.view(1, T, H, D), k.view(1, T, Hkv, D), v.view(1, T, Hkv, D),
                       causal=True, scale=1.0 / np.sqrt(D))
    y = api.out_proj(attn.view(T, H * D), w_o.to(dev))
    torch.cuda.synchronize()
    assert api.device_status() == api.LLAMA_OK
    eq, ek, ev = _qkv_expected(x, w_qkv, pos, H, Hkv, D, True)
    ref_attn = oracle.prefill(eq[None], ek[None], ev[None], None, scale=1.0 / np.sqrt(D),
                              causal=True)[0]
    ref_y = ref_attn @ w_o.double().numpy().T
    err = _close(y, ref_y, "attention block")
    PARITY_REPORT.append(("attention block (qkv+rope, prefill, o_proj)", "bfloat16",
                          float(err.max()), float(err.mean())))


def test_qkv_rope_70b_shape_sampled_rows():
    # the 70B projection at full size (8192 tokens, hidden 8192, 64 + 2 x 8 heads
    # of 128), the launch the projection benchmark times; rows sampled from every
    # group of row tiles and the last tile, all columns checked
    T, hidden, H, Hkv, D = 8192, 8192, 64, 8, 128
    g = torch.Generator().manual_seed(70)
    x = W.normal((T, hidden), torch.bfloat16, g)
    w = _weights((H + 2 * Hkv) * D, hidden, g)
    pos = torch.arange(T)
    dev = torch.device("cuda")
    cos, sin = api.rope_table(pos.view(1, -1).to(dev), D, THETA, 1.0)
    q, k, v = api.qkv_rope(x.to(dev), w.to(dev), H, Hkv, D, cos.view(T, D), sin.view(T, D))
    torch.cuda.synchronize()
    assert api.device_status() == api.LLAMA_OK
    rows = torch.tensor(sorted({0, 1, 127, 128, 2047, 2048, 4095, 4096, 6143, 6144, 8190, 8191}
                               | set(torch.randint(0, T, (20,), generator=g).tolist())))
    eq, ek, ev = _qkv_expected(x[rows], w, pos[rows], H, Hkv, D, True)
    errs = [_close(q.cpu()[rows], eq, "q"), _close(k.cpu()[rows], ek, "k"),
            _close(v.cpu()[rows], ev, "v")]
    err = np.concatenate([e.reshape(-1) for e in errs])
    PARITY_REPORT.append(("qkv+rope projection 70B shape (sampled rows)", "bfloat16",
                          float(err.max()), float(err.mean())))
