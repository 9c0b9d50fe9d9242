"""Pins for the fp64 oracle: checks against facts that do not come from the oracle.

Each test names what fixes the expected value: a textbook closed form, a
library routine (torch SDPA, the HF LLaMA rotary embedding / attention the
pages walk through), an invariant the pages state, or the independent
pure-Python brute force.  Chosen so that a dropped term, a wrong sign, a wrong
index or a transposed operand in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from llama_gqa_causal_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64).to(dtype)


# ----------------------------------------------------------------------------- RoPE

def test_rope_d2_is_textbook_rotation():
    # D = 2: one pair, frequency theta**0 = 1, so position p rotates by angle p.
    for p in [0, 1, 2, 5, 17]:
        c, s = oracle.rope_cos_sin([p], 2, theta=10000.0)
        y = oracle.rope_rotate(np.array([[1.0, 0.0]]), c, s)
        np.testing.assert_allclose(y[0], [math.cos(p), math.sin(p)], atol=1e-15)
        y = oracle.rope_rotate(np.array([[0.0, 1.0]]), c, s)
        np.testing.assert_allclose(y[0], [-math.sin(p), math.cos(p)], atol=1e-15)


def test_rope_position_zero_is_identity():
    x = _rand((5, 128), 1).numpy()
    c, s = oracle.rope_cos_sin(np.zeros(5, np.int64), 128)
    np.testing.assert_array_equal(oracle.rope_rotate(x, c, s), x)


def test_rope_preserves_norm():
    x = _rand((64, 128), 2).numpy()
    pos = np.arange(64) * 131
    c, s = oracle.rope_cos_sin(pos, 128)
    y = oracle.rope_rotate(x, c, s)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


def test_rope_dot_depends_on_position_difference_only():
    q = _rand((1, 64), 3).numpy()
    k = _rand((1, 64), 4).numpy()
    def dot(m, n):
        cq, sq = oracle.rope_cos_sin([m], 64)
        ck, sk = oracle.rope_cos_sin([n], 64)
        return float((oracle.rope_rotate(q, cq, sq) @ oracle.rope_rotate(k, ck, sk).T)[0, 0])
    base = dot(7, 3)
    for t in [1, 10, 1000]:
        assert abs(dot(7 + t, 3 + t) - base) < 1e-10
    assert abs(dot(8, 3) - base) > 1e-6  # but it does depend on the difference


def test_rope_linear_scaling_divides_positions():
    facts = json.load(open(os.path.join(GOLDEN, "page_facts.json")))
    f = facts["linear_rope_scaling"]["factor"]
    pos = np.arange(0, 200, 2)
    c1, s1 = oracle.rope_cos_sin(pos, 128, factor=f)
    c2, s2 = oracle.rope_cos_sin(pos // 2, 128, factor=1.0)
    np.testing.assert_allclose(c1, c2, atol=1e-15)
    np.testing.assert_allclose(s1, s2, atol=1e-15)


@pytest.mark.parametrize("factor", [1.0, 2.0])
def test_rope_tables_match_hf_llama_rotary_embedding(factor):
    # Library pin: the HF LlamaRotaryEmbedding (fp32) that the LlamaAttention page calls.
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding
    rp = {"rope_theta": 10000.0, "rope_type": "default"}
    if factor != 1.0:
        rp = {"rope_theta": 10000.0, "rope_type": "linear", "factor": factor}
    cfg = LlamaConfig(hidden_size=4096, num_attention_heads=32, head_dim=128, rope_parameters=rp)
    emb = LlamaRotaryEmbedding(cfg)
    pos = torch.arange(0, 96).view(1, -1)
    cos, sin = emb(torch.zeros(1, dtype=torch.float32), pos)
    c, s = oracle.rope_cos_sin(pos.numpy(), 128, theta=10000.0, factor=factor)
    # HF rounds its frequencies and angles to fp32: |angle| <= 96 -> abs error ~1e-5
    np.testing.assert_allclose(c, cos[0].double().numpy(), atol=2e-5)
    np.testing.assert_allclose(s, sin[0].double().numpy(), atol=2e-5)


def test_rope_rotate_matches_hf_apply_rotary_pos_emb():
    # Library pin for the rotate-half form, with the oracle's own cos/sin in fp64.
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    b, H, S, D = 2, 3, 9, 64
    q = _rand((b, H, S, D), 5)
    k = _rand((b, H, S, D), 6)
    pos = np.arange(S) + 40
    c, s = oracle.rope_cos_sin(pos, D, factor=2.0)
    ct = torch.from_numpy(c).view(1, S, D).expand(b, S, D)
    st = torch.from_numpy(s).view(1, S, D).expand(b, S, D)
    qh, kh = apply_rotary_pos_emb(q, k, ct, st)
    qo = oracle.rope_rotate(q.numpy(), c[None, None], s[None, None])
    ko = oracle.rope_rotate(k.numpy(), c[None, None], s[None, None])
    np.testing.assert_allclose(qo, qh.numpy(), atol=1e-14)
    np.testing.assert_allclose(ko, kh.numpy(), atol=1e-14)


# ----------------------------------------------------------------------------- attention

def _sdpa_ref(q, k, v, causal, mask=None, scale=None):
    """torch SDPA in float64 with GQA (library routine). q [b,S,H,D] -> [b,S,H*D]."""
    qt, kt, vt = (x.double().permute(0, 2, 1, 3) for x in (q, k, v))
    am = None if mask is None else mask.double()
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=am, is_causal=causal and mask is None, scale=scale, enable_gqa=True)
    b, H, S, D = o.shape
    return o.permute(0, 2, 1, 3).reshape(b, S, H * D).numpy()


@pytest.mark.parametrize("H,Hkv", [(4, 4), (4, 2), (8, 1), (6, 3)])
@pytest.mark.parametrize("causal", [True, False])
def test_prefill_matches_torch_sdpa(H, Hkv, causal):
    b, S, D = 2, 37, 32
    q, k, v = _rand((b, S, H, D), 7), _rand((b, S, Hkv, D), 8), _rand((b, S, Hkv, D), 9)
    out = oracle.prefill(q, k, v, None, causal=causal)
    ref = _sdpa_ref(q.float(), k.float(), v.float(), causal)
    np.testing.assert_allclose(out, ref, atol=1e-6)  # inputs rounded to fp32 for the oracle
    # exact comparison on float32-representable inputs
    qf, kf, vf = q.float().double(), k.float().double(), v.float().double()
    np.testing.assert_allclose(out, _sdpa_ref(qf, kf, vf, causal), atol=1e-12)


def test_prefill_additive_mask_matches_torch_sdpa():
    b, S, H, Hkv, D = 2, 20, 4, 2, 16
    q, k, v = (_rand(s, 10 + i).float().double() for i, s in
               enumerate([(b, S, H, D), (b, S, Hkv, D), (b, S, Hkv, D)]))
    m = W.additive_mask(b, S, torch.Generator().manual_seed(3))
    out = oracle.prefill(q, k, v, None, causal=False, mask=m)
    np.testing.assert_allclose(out, _sdpa_ref(q, k, v, False, mask=m), atol=1e-12)
    # causal flag == additive -inf mask above the diagonal (added on top of m)
    tri = torch.full((S, S), float("-inf")).triu(1).view(1, 1, S, S)
    out_c = oracle.prefill(q, k, v, None, causal=True, mask=m)
    np.testing.assert_allclose(out_c, _sdpa_ref(q, k, v, False, mask=m + tri), atol=1e-12)


def test_prefill_with_rope_matches_hf_eager_attention():
    # Library pin: the HF eager attention + apply_rotary_pos_emb + repeat_kv the page walks through.
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb, eager_attention_forward
    b, S, H, Hkv, D = 1, 24, 8, 2, 32
    q, k, v = (_rand(s, 20 + i).float().double() for i, s in
               enumerate([(b, S, H, D), (b, S, Hkv, D), (b, S, Hkv, D)]))
    pos = np.arange(S).reshape(1, S) * 3
    c, s = oracle.rope_cos_sin(pos, D, factor=2.0)
    ct, st = torch.from_numpy(c).view(1, S, D), torch.from_numpy(s).view(1, S, D)
    qh, kh = apply_rotary_pos_emb(q.transpose(1, 2), k.transpose(1, 2), ct, st)
    causal = torch.full((S, S), float("-inf"), dtype=torch.float64).triu(1).view(1, 1, S, S)

    class _M(torch.nn.Module):
        num_key_value_groups = H // Hkv
        training = False
    o, _ = eager_attention_forward(_M(), qh, kh, v.transpose(1, 2), causal, scaling=D ** -0.5)
    ref = o.reshape(b, S, H * D).numpy()
    out = oracle.prefill(q, k, v, pos, factor=2.0, causal=True)
    # the page's eager path runs its softmax in fp32 (step 5.2), hence ~1e-7 differences
    np.testing.assert_allclose(out, ref, atol=1e-6)


def test_closed_form_two_tokens():
    # S=2, D=2, one head, scale 1, no RoPE.  q0=k0=(1,0), q1=k1=(0,1), v0=(1,2), v1=(3,4).
    # Row 0 scores (1, 0): weights (e, 1)/(e+1)  -> out0 = ((e+3)/(e+1), (2e+4)/(e+1)).
    # Row 1 scores (0, 1): weights (1, e)/(e+1)  -> out1 = ((1+3e)/(e+1), (2+4e)/(e+1)).
    # Causal: row 0 sees only key 0 -> out0 = v0.
    e = math.e
    q = torch.tensor([[[[1.0, 0.0]], [[0.0, 1.0]]]])
    k = q.clone()
    v = torch.tensor([[[[1.0, 2.0]], [[3.0, 4.0]]]])
    out = oracle.prefill(q, k, v, None, scale=1.0, causal=False)
    exp = [[(e + 3) / (e + 1), (2 * e + 4) / (e + 1)], [(1 + 3 * e) / (e + 1), (2 + 4 * e) / (e + 1)]]
    np.testing.assert_allclose(out[0], exp, atol=1e-15)
    out = oracle.prefill(q, k, v, None, scale=1.0, causal=True)
    np.testing.assert_allclose(out[0], [[1.0, 2.0], exp[1]], atol=1e-15)


def test_softmax_rows_are_distributions():
    cfg, x = W.small_prefill(1, 33, 4, 2, 32, torch.float32, causal=True, seed=5)
    _, probs = oracle.prefill(x["q"], x["k"], x["v"], x["pos"], return_probs=True)
    assert (probs >= 0).all()
    np.testing.assert_allclose(probs.sum(-1), 1.0, atol=1e-14)
    assert np.all(np.triu(probs[0, 0], 1) == 0)


def test_mask_constant_shift_invariance():
    cfg, x = W.small_prefill(2, 19, 4, 4, 16, torch.float32, causal=True, seed=6, with_mask=True)
    m = torch.round(x["mask"] * 1024) / 1024  # on a 2^-10 grid so that +3.25 is exact in fp32
    a = oracle.prefill(x["q"], x["k"], x["v"], x["pos"], mask=m)
    b = oracle.prefill(x["q"], x["k"], x["v"], x["pos"], mask=m + 3.25)
    np.testing.assert_allclose(a, b, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_scale_zero_gives_mean_of_visible_values(causal):
    # scale 0 -> uniform weights -> prefix mean (causal) or full mean of V.
    cfg, x = W.small_prefill(1, 15, 4, 2, 8, torch.float32, causal=causal, seed=7)
    out = oracle.prefill(x["q"], x["k"], x["v"], x["pos"], scale=0.0, causal=causal)
    v = x["v"].double().numpy()[0]  # [S, Hkv, D]
    S, Hkv, D = v.shape
    for i in range(S):
        vis = v[: i + 1] if causal else v
        mean = vis.mean(axis=0)  # [Hkv, D]
        for h in range(4):
            np.testing.assert_allclose(out[0, i, h * D:(h + 1) * D], mean[h // 2], atol=1e-14)


def test_gqa_equals_mha_on_repeated_kv():
    # repeat_kv: query head h reads K/V head h // group  ==  np.repeat along heads.
    facts = json.load(open(os.path.join(GOLDEN, "page_facts.json")))
    g = facts["gqa_group"]["queries_per_kv_head"]
    Hkv = 2
    H = g * Hkv
    cfg, x = W.small_prefill(1, 21, H, Hkv, 16, torch.float32, causal=True, seed=8)
    out = oracle.prefill(x["q"], x["k"], x["v"], x["pos"])
    k_rep = x["k"].repeat_interleave(g, dim=2)
    v_rep = x["v"].repeat_interleave(g, dim=2)
    out_mha = oracle.prefill(x["q"], k_rep, v_rep, x["pos"])
    np.testing.assert_allclose(out, out_mha, atol=1e-13)
    # the other plausible mapping (h % Hkv) gives a different answer
    out_tiled = oracle.prefill(x["q"], x["k"].repeat(1, 1, g, 1), x["v"].repeat(1, 1, g, 1), x["pos"])
    assert np.abs(out_tiled - out).max() > 1e-3


def test_mqa_equals_mha_with_kv_head_zero():
    cfg, x = W.small_prefill(1, 17, 6, 1, 16, torch.float32, causal=True, seed=9)
    out = oracle.prefill(x["q"], x["k"], x["v"], x["pos"])
    out_mha = oracle.prefill(x["q"], x["k"].expand(-1, -1, 6, -1), x["v"].expand(-1, -1, 6, -1), x["pos"])
    np.testing.assert_allclose(out, out_mha, atol=1e-13)


def test_head_group_concat_equals_full_attention():
    # Tensor-parallel demo: heads split into contiguous groups per card, outputs
    # concatenated on the last dim in card order == full attention.
    facts = json.load(open(os.path.join(GOLDEN, "page_facts.json")))["tp_demo"]
    world = facts["world"]
    cfg, x = W.small_prefill(2, 16, 8, 4, 16, torch.float32, causal=False, rope=False, seed=10)
    full = oracle.prefill(x["q"], x["k"], x["v"], None, causal=False)
    H, Hkv, D = 8, 4, 16
    parts = []
    for r in range(world):
        hs = slice(r * H // world, (r + 1) * H // world)
        ks = slice(r * Hkv // world, (r + 1) * Hkv // world)
        parts.append(oracle.prefill(x["q"][:, :, hs], x["k"][:, :, ks], x["v"][:, :, ks], None,
                                    causal=False))
    np.testing.assert_allclose(np.concatenate(parts, axis=-1), full, atol=1e-14)
    # wrong card order: right shape, wrong numbers
    wrong = np.concatenate(parts[::-1], axis=-1)
    assert wrong.shape == full.shape and np.abs(wrong - full).max() > 1e-3


def test_tp_demo_output_shape():
    f = json.load(open(os.path.join(GOLDEN, "page_facts.json")))["tp_demo"]
    hd = f["hidden"] // f["heads"]
    cfg, x = W.small_prefill(f["batch"], 4, f["heads"], f["heads"], hd, torch.float32,
                             causal=False, rope=False, seed=11)
    out = oracle.prefill(x["q"], x["k"], x["v"], None, causal=False, rows=(0, 1))
    assert list(out.shape) == [f["batch"], 4, f["hidden"]]
    assert f["expected_output_shape"][2] == out.shape[2]


def test_causal_row_ignores_future_keys():
    cfg, x = W.small_prefill(1, 24, 4, 2, 16, torch.float32, causal=True, seed=12)
    a = oracle.prefill(x["q"], x["k"], x["v"], x["pos"])
    k2, v2 = x["k"].clone(), x["v"].clone()
    k2[:, 10:] = torch.randn(k2[:, 10:].shape) * 5
    v2[:, 10:] = torch.randn(v2[:, 10:].shape) * 5
    b = oracle.prefill(x["q"], k2, v2, x["pos"])
    np.testing.assert_array_equal(a[:, :10], b[:, :10])
    assert np.abs(a[:, 10:] - b[:, 10:]).max() > 1e-3


def test_seq_one_returns_v():
    cfg, x = W.small_prefill(3, 1, 4, 2, 16, torch.float32, causal=True, seed=13)
    out = oracle.prefill(x["q"], x["k"], x["v"], x["pos"])
    v = x["v"].double().numpy()
    for h in range(4):
        np.testing.assert_allclose(out[:, 0, h * 16:(h + 1) * 16], v[:, 0, h // 2], atol=1e-15)


def test_fully_masked_row_is_zero():
    cfg, x = W.small_prefill(1, 6, 2, 2, 8, torch.float32, causal=False, rope=False, seed=14)
    m = torch.zeros(1, 1, 6, 6)
    m[0, 0, 2, :] = float("-inf")
    out = oracle.prefill(x["q"], x["k"], x["v"], None, causal=False, mask=m)
    assert np.all(out[0, 2] == 0.0)
    assert np.all(np.isfinite(out))


# ----------------------------------------------------------------------------- decode

def _rotated_cache(k, pos, theta, factor):
    """[b,S,Hkv,D] keys -> rotated cache [b,Hkv,S,D] via the brute-force rotation."""
    b, S, Hkv, D = k.shape
    kk = k.double().numpy()
    out = np.zeros((b, Hkv, S, D))
    for bi in range(b):
        for j in range(S):
            for g in range(Hkv):
                out[bi, g, j] = brute._rotate(list(kk[bi, j, g]), int(pos[bi][j]), theta, factor)
    return torch.from_numpy(out).float()


@pytest.mark.parametrize("H,Hkv", [(8, 2), (4, 4), (4, 1)])
def test_decode_equals_last_row_of_causal_prefill(H, Hkv):
    b, T, D = 2, 23, 16
    cfg, x = W.small_prefill(b, T, H, Hkv, D, torch.float32, causal=True, seed=15)
    # inputs exact in fp32 after rotation: compare in fp64 from the same rotated keys
    pre = oracle.prefill(x["q"], x["k"], x["v"], x["pos"])
    kc = _rotated_cache(x["k"], x["pos"], 10000.0, 1.0)
    vc = x["v"].permute(0, 2, 1, 3).contiguous()
    lens = np.full(b, T, np.int32)
    for i in [T - 1, 0, 7]:
        dec = oracle.decode(x["q"][:, i], kc, vc, np.full(b, i + 1, np.int32),
                            np.full(b, i, np.int64))
        # rotated keys were rounded to fp32 for the cache: tolerance from that rounding
        np.testing.assert_allclose(dec, pre[:, i], atol=2e-6)
    _ = lens


def test_decode_probs_are_distributions_and_ignore_tail():
    cfg, x = W.small_decode(3, 8, 2, 16, 40, torch.float32, min_len=5, max_len=40, seed=16)
    out, probs = oracle.decode(x["q"], x["k_cache"], x["v_cache"], x["lens"], x["qpos"],
                               return_probs=True)
    assert np.all(np.isfinite(out))  # NaN-poisoned tail never read
    np.testing.assert_allclose(probs.sum(-1), 1.0, atol=1e-14)
    for b in range(3):
        assert np.all(probs[b, :, int(x["lens"][b]):] == 0)


def test_decode_empty_cache_gives_zero():
    cfg, x = W.small_decode(2, 4, 2, 8, 6, torch.float32, lens=torch.tensor([0, 3]), seed=17)
    out = oracle.decode(x["q"], x["k_cache"], x["v_cache"], x["lens"], x["qpos"])
    assert np.all(out[0] == 0) and np.all(np.isfinite(out[1]))


# ----------------------------------------------------------------------------- brute force

@pytest.mark.parametrize("D", [2, 4, 8])
@pytest.mark.parametrize("causal", [True, False])
def test_brute_force_agrees_prefill(D, causal):
    for S in [1, 3, 8]:
        cfg, x = W.small_prefill(2, S, 4, 2, D, torch.float32, causal=causal,
                                 factor=2.0, seed=100 + S + D)
        m = W.additive_mask(2, S, torch.Generator().manual_seed(S)) if not causal else None
        out = oracle.prefill(x["q"], x["k"], x["v"], x["pos"], factor=2.0, causal=causal, mask=m)
        ref = brute.prefill(x["q"].double().tolist(), x["k"].double().tolist(),
                            x["v"].double().tolist(), x["pos"].tolist(), factor=2.0,
                            causal=causal, mask=None if m is None else m.double().tolist())
        np.testing.assert_allclose(out, np.array(ref), atol=1e-12)


def test_brute_force_agrees_decode():
    cfg, x = W.small_decode(2, 6, 3, 8, 7, torch.float32, min_len=1, max_len=7, seed=18,
                            poison=False)
    out = oracle.decode(x["q"], x["k_cache"], x["v_cache"], x["lens"], x["qpos"])
    ref = brute.decode(x["q"].double().tolist(), x["k_cache"].double().tolist(),
                       x["v_cache"].double().tolist(), x["lens"].tolist(), x["qpos"].tolist())
    np.testing.assert_allclose(out, np.array(ref), atol=1e-12)


MUTATIONS = {
    "rotate_half_sign": ("(d < half) ? -xr[d + half]", "(d < half) ? xr[d + half]"),
    "frequency_exponent": ("pow(theta, -2.0 * (double)i", "pow(theta, -1.0 * (double)i"),
    "linear_scaling": ("(double)pos[r] / factor", "(double)pos[r] * factor"),
    "kv_head_map": ("const int kh = h / group; /* repeat_kv", "const int kh = h % Hkv; /* repeat_kv"),
    "causal_diagonal": ("if (causal && j > i)", "if (causal && j >= i)"),
    "scale_dropped": ("double s = dot * scale;", "double s = dot;"),
    "mask_sign": ("s += (double)mask[", "s -= (double)mask["),
    "decode_value_row": ("v_cache + ((long)b * Hkv + kh) * (long)L * D,", "v_cache + ((long)b * Hkv) * (long)L * D,"),
}


def _pin_suite():
    """A fast subset of the pins above; returns the list of pins that failed."""
    failed = []
    checks = [
        ("rope_d2", test_rope_d2_is_textbook_rotation),
        ("rope_hf_tables", lambda: test_rope_tables_match_hf_llama_rotary_embedding(2.0)),
        ("rope_hf_rotate", test_rope_rotate_matches_hf_apply_rotary_pos_emb),
        ("sdpa_gqa_causal", lambda: test_prefill_matches_torch_sdpa(4, 2, True)),
        ("sdpa_mask", test_prefill_additive_mask_matches_torch_sdpa),
        ("hf_eager", test_prefill_with_rope_matches_hf_eager_attention),
        ("decode_last_row", lambda: test_decode_equals_last_row_of_causal_prefill(8, 2)),
        ("brute_decode", test_brute_force_agrees_decode),
    ]
    for name, fn in checks:
        try:
            fn()
        except AssertionError:
            failed.append(name)
    return failed


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_in_oracle_is_caught(mutation, tmp_path):
    """Plant one plausible mistake in a copy of the C oracle; the pins must catch it."""
    import subprocess
    src = open(oracle._SRC).read()
    old, new = MUTATIONS[mutation]
    assert src.count(old) == 1, f"mutation anchor not found: {old}"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(mut), "-lm"])
    saved = oracle._load()
    oracle._lib = oracle._bind(str(so))
    try:
        failed = _pin_suite()
    finally:
        oracle._lib = saved
    assert failed, f"planted mistake {mutation!r} slipped past every pin"


def test_unmutated_oracle_passes_pin_suite():
    assert _pin_suite() == []



# ----------------------------------------------------------------------------- NTK-aware scaling
# The pages name adjusting the RoPE base for longer contexts without a formula;
# the oracle takes the published NTK-aware rule.  What the rule is for fixes
# it: alpha = 1 is the plain table, the highest frequency (i = 0) never moves,
# and the lowest (i = D/2 - 1) is exactly linear position interpolation by alpha.

@pytest.mark.parametrize("D", [64, 128])
def test_ntk_alpha_one_is_the_plain_table(D):
    pos = np.arange(0, 5000, 7)
    c0, s0 = oracle.rope_cos_sin(pos, D, 10000.0, 1.0)
    c1, s1 = oracle.rope_cos_sin_ntk(pos, D, 10000.0, 1.0)
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1)


@pytest.mark.parametrize("D,alpha", [(64, 2.0), (128, 4.0), (128, 8.0)])
def test_ntk_keeps_the_highest_frequency(D, alpha):
    pos = np.arange(0, 40000, 13)
    c0, s0 = oracle.rope_cos_sin(pos, D, 10000.0, 1.0)
    c1, s1 = oracle.rope_cos_sin_ntk(pos, D, 10000.0, alpha)
    assert np.array_equal(c0[:, 0], c1[:, 0]) and np.array_equal(s0[:, 0], s1[:, 0])


@pytest.mark.parametrize("D,alpha", [(64, 2.0), (128, 4.0), (128, 8.0)])
def test_ntk_lowest_frequency_is_linear_interpolation(D, alpha):
    pos = np.arange(0, 40000, 13)
    lo = D // 2 - 1
    c_lin, s_lin = oracle.rope_cos_sin(pos, D, 10000.0, alpha)   # positions / alpha
    c_ntk, s_ntk = oracle.rope_cos_sin_ntk(pos, D, 10000.0, alpha)
    assert np.abs(c_ntk[:, lo] - c_lin[:, lo]).max() < 1e-9
    assert np.abs(s_ntk[:, lo] - s_lin[:, lo]).max() < 1e-9
    # and it is not plain interpolation elsewhere: a middle frequency moves less
    mid = D // 4
    assert np.abs(c_ntk[:, mid] - c_lin[:, mid]).max() > 1e-3


def test_oracle_thread_count_applies_to_one_call_only():
    # a one-core timing must not leave the process on one core for later calls
    before = oracle.max_threads()
    g = np.random.default_rng(5)
    q = g.standard_normal((1, 8, 2, 64)).astype(np.float32)
    k = g.standard_normal((1, 8, 1, 64)).astype(np.float32)
    a = oracle.prefill(q, k, k, None, nthreads=1)
    b = oracle.prefill(q, k, k, None)
    assert oracle.max_threads() == before
    assert np.array_equal(a, b)
