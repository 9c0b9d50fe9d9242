"""GPU parity of llama_attn_decode_append (marked gpu).

The decode step with the new token's own key and value: the key is rotated at
the new token's position p = min(max(len, 0), L - 1) (the query's position),
key and value are written into cache row p, and the query attends over rows
0..p.  The expected output is the fp64 oracle's decode over the cache with row
p replaced by the oracle's rotation of k_new and by v_new.  Also checked: the
rows written (the key to within the bf16 rounding of the rotation, the value
and every other row bit for bit), a closed form (an empty cache attends only
the new token, so the output is v_new), and that a plain decode over p + 1
rows of the updated cache gives bit-identical output.
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
    # (bsz, H, Hkv, D, L, lens)
    (4, 8, 2, 128, 300, [0, 1, 130, 299]),          # empty cache; the cache's last row
    (3, 16, 1, 64, 200, [63, 64, 500]),             # new row alone in its tile; full cache -> row L-1
    (2, 32, 2, 128, 256, [100, 255]),               # group 16: two head chunks share the new row
    (5, 12, 4, 128, 130, [-2, 65, 127, 128, 129]),  # negative length clamps to 0
]


def _inputs(b, H, Hkv, D, L, seed):
    g = torch.Generator().manual_seed(seed)
    q = W.normal((b, H, D), torch.bfloat16, g)
    k_new = W.normal((b, Hkv, D), torch.bfloat16, g)
    v_new = W.normal((b, Hkv, D), torch.bfloat16, g)
    k_cache = W.normal((b, Hkv, L, D), torch.bfloat16, g)
    v_cache = W.normal((b, Hkv, L, D), torch.bfloat16, g)
    return q, k_new, v_new, k_cache, v_cache


def _expected(q, k_new, v_new, k_cache, v_cache, pos, scale):
    b, Hkv, D = k_new.shape
    qpos = np.asarray(pos, dtype=np.int64)
    c, s = oracle.rope_cos_sin(qpos, D, THETA, 1.0)
    k_rot = oracle.rope_rotate(k_new.double().numpy(), c[:, None, :], s[:, None, :])
    k_ref = k_cache.double().numpy().copy()
    v_ref = v_cache.double().numpy().copy()
    for i, p in enumerate(pos):
        k_ref[i, :, p] = k_rot[i]
        v_ref[i, :, p] = v_new[i].double().numpy()
    # rows past p may hold anything: poison them so that a read of one shows
    for i, p in enumerate(pos):
        k_ref[i, :, p + 1:] = np.nan
        v_ref[i, :, p + 1:] = np.nan
    ref = oracle.decode(q, k_ref, v_ref, np.asarray(pos) + 1, qpos, theta=THETA, factor=1.0,
                        scale=scale)
    return ref, k_rot


def _run(b, H, Hkv, D, L, lens, seed):
    pos = [min(max(n, 0), L - 1) for n in lens]
    q, k_new, v_new, k_cache, v_cache = _inputs(b, H, Hkv, D, L, seed)
    scale = 1.0 / np.sqrt(D)
    dev = torch.device("cuda")
    kc, vc = k_cache.to(dev), v_cache.to(dev)
    qpos = torch.tensor(pos, dtype=torch.int64, device=dev)
    cos, sin = api.rope_table(qpos.view(-1, 1), D, THETA, 1.0)
    cos, sin = cos.view(b, D), sin.view(b, D)
    out = api.decode_append(q.to(dev), k_new.to(dev), v_new.to(dev), kc, vc,
                            torch.tensor(lens, dtype=torch.int32, device=dev), cos, sin,
                            scale=scale)
    torch.cuda.synchronize()
    assert api.device_status() == api.LLAMA_OK
    ref, k_rot = _expected(q, k_new, v_new, k_cache, v_cache, pos, scale)
    return dict(q=q, k_new=k_new, v_new=v_new, k_cache=k_cache, v_cache=v_cache, kc=kc, vc=vc,
                cos=cos, sin=sin, out=out, ref=ref, k_rot=k_rot, pos=pos, scale=scale)


def _check_out(out, ref, what, report=False):
    g = out.float().cpu().double().numpy()
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    assert err.max() <= BF16_MAX, f"{what}: max abs {err.max():.3e}"
    assert err.mean() <= BF16_MEAN, f"{what}: mean abs {err.mean():.3e}"
    if report:
        PARITY_REPORT.append((what, "bfloat16", float(err.max()), float(err.mean())))


def _check_cache_rows(r):
    kc, vc = r["kc"].cpu(), r["vc"].cpu()
    b = kc.shape[0]
    for i, p in enumerate(r["pos"]):
        got = kc[i, :, p].double().numpy()
        want = r["k_rot"][i]
        # the kernel rotates in fp32 and rounds to bf16 (relative 2^-8)
        assert np.all(np.abs(got - want) <= np.abs(want) * 2.0 ** -8 + 1e-6), f"k row b={i}"
        assert torch.equal(vc[i, :, p].view(torch.int16), r["v_new"][i].view(torch.int16))
    # every other row is untouched, bit for bit
    keep = torch.ones(kc.shape[:3], dtype=torch.bool)
    for i, p in enumerate(r["pos"]):
        keep[i, :, p] = False
    assert torch.equal(kc.view(torch.int16)[keep], r["k_cache"].view(torch.int16)[keep])
    assert torch.equal(vc.view(torch.int16)[keep], r["v_cache"].view(torch.int16)[keep])
    assert b == len(r["pos"])


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%dH%dKV%dD%dL%d" % c[:5])
def test_decode_append_matches_oracle(case):
    b, H, Hkv, D, L, lens = case
    r = _run(b, H, Hkv, D, L, lens, seed=sum(abs(n) for n in lens) + H)
    _check_out(r["out"], r["ref"], str(case))
    _check_cache_rows(r)


@pytest.mark.parametrize("case", CASES[:3], ids=lambda c: "b%dH%dKV%dD%dL%d" % c[:5])
def test_decode_append_equals_plain_decode_of_the_updated_cache(case):
    b, H, Hkv, D, L, lens = case
    r = _run(b, H, Hkv, D, L, lens, seed=7 + H)
    dev = torch.device("cuda")
    lens_after = torch.tensor([p + 1 for p in r["pos"]], dtype=torch.int32, device=dev)
    out2 = api.decode(r["q"].to(dev), r["kc"], r["vc"], lens_after, r["cos"], r["sin"],
                      scale=r["scale"])
    torch.cuda.synchronize()
    assert torch.equal(r["out"].view(torch.int16), out2.view(torch.int16))


def test_decode_append_on_an_empty_cache_returns_v_new():
    # one attended row: its weight is exactly 1, so out = v_new of the head's K/V head
    b, H, Hkv, D, L = 3, 16, 4, 128, 64
    r = _run(b, H, Hkv, D, L, [0, 0, -5], seed=11)
    group = H // Hkv
    out = r["out"].cpu().view(b, H, D)
    for h in range(H):
        assert torch.equal(out[:, h].view(torch.int16), r["v_new"][:, h // group].view(torch.int16))


def test_decode_append_decode70b_shape():
    # the decode workload's shape with lengths drawn from [512, 4095]
    cfg = W.DECODE70B
    g = torch.Generator().manual_seed(cfg.seed + 1)
    lens = torch.randint(cfg.min_len, cfg.max_cache_len, (cfg.bsz,), generator=g).tolist()
    r = _run(cfg.bsz, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.max_cache_len, lens, seed=5)
    _check_out(r["out"], r["ref"], "decode70b append", report=True)
    _check_cache_rows(r)
