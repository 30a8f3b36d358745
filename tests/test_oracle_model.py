"""Pins of the oracle's decoder forward (CPU only).

The forward is compared with the HuggingFace ``transformers`` implementations
of OPT and Qwen3 (an independent library, float64 on CPU) on tiny random
models carrying the oracle's weights, and checked for the invariants the
method relies on: causality within a row and independence of rows (packing
changes layout, not results).
"""
import numpy as np
import pytest
import torch

from oracle import model as om
from zeroth_order_fine_b200 import workload as wl

TINY_Q3 = wl.ModelShape("tiny-qwen3", wl.ARCH_QWEN3, 2, 64, 4, 2, 16, 96, 256, 128,
                        1e-6, 1e6, wl.DTYPE_FP32, False)


def _rows(shape, lens, seed=0):
    rng = np.random.default_rng(seed)
    return [rng.integers(0, shape.vocab, size=L).astype(np.int32) for L in lens]


def _hf_opt(w: om.Weights):
    from transformers import OPTConfig, OPTForCausalLM
    sh = w.shape
    cfg = OPTConfig(vocab_size=sh.vocab, hidden_size=sh.d_model, num_hidden_layers=sh.n_layers,
                    ffn_dim=sh.d_ffn, num_attention_heads=sh.n_heads,
                    max_position_embeddings=sh.max_pos, do_layer_norm_before=True,
                    word_embed_proj_dim=sh.d_model, activation_function="relu",
                    enable_bias=True, dropout=0.0, attention_dropout=0.0,
                    layer_norm_elementwise_affine=True)
    cfg._attn_implementation = "eager"
    m = OPTForCausalLM(cfg).double().eval()
    dec = m.model.decoder
    with torch.no_grad():
        dec.embed_tokens.weight.copy_(w.tok_embed)
        dec.embed_positions.weight.zero_()
        dec.embed_positions.weight[2:2 + sh.max_pos].copy_(w.pos_embed)   # HF offset of 2
        dec.final_layer_norm.weight.copy_(w.final_w)
        dec.final_layer_norm.bias.copy_(w.final_b)
        for lay, p in zip(dec.layers, w.layers):
            at = lay.self_attn
            for name, m_id in (("q_proj", 0), ("k_proj", 1), ("v_proj", 2), ("out_proj", 3)):
                getattr(at, name).weight.copy_(p[f"W{m_id}"])
                getattr(at, name).bias.copy_(p[f"b{m_id}"])
            lay.fc1.weight.copy_(p["W5"]); lay.fc1.bias.copy_(p["b5"])
            lay.fc2.weight.copy_(p["W6"]); lay.fc2.bias.copy_(p["b6"])
            lay.self_attn_layer_norm.weight.copy_(p["ln1_w"])
            lay.self_attn_layer_norm.bias.copy_(p["ln1_b"])
            lay.final_layer_norm.weight.copy_(p["ln2_w"])
            lay.final_layer_norm.bias.copy_(p["ln2_b"])
        m.lm_head.weight.copy_(w.tok_embed)
    return m


def _hf_qwen3(w: om.Weights):
    from transformers import Qwen3Config, Qwen3ForCausalLM
    sh = w.shape
    cfg = Qwen3Config(vocab_size=sh.vocab, hidden_size=sh.d_model, intermediate_size=sh.d_ffn,
                      num_hidden_layers=sh.n_layers, num_attention_heads=sh.n_heads,
                      num_key_value_heads=sh.n_kv_heads, head_dim=sh.head_dim,
                      rms_norm_eps=sh.norm_eps, max_position_embeddings=sh.max_pos,
                      rope_parameters={"rope_theta": sh.rope_theta, "rope_type": "default"},
                      tie_word_embeddings=False, attention_bias=False)
    cfg._attn_implementation = "eager"
    m = Qwen3ForCausalLM(cfg).double().eval()
    with torch.no_grad():
        m.model.embed_tokens.weight.copy_(w.tok_embed)
        m.model.norm.weight.copy_(w.final_w)
        m.lm_head.weight.copy_(w.lm_head)
        for lay, p in zip(m.model.layers, w.layers):
            at = lay.self_attn
            for name, m_id in (("q_proj", 0), ("k_proj", 1), ("v_proj", 2), ("o_proj", 3)):
                getattr(at, name).weight.copy_(p[f"W{m_id}"])
            at.q_norm.weight.copy_(p["q_norm"])
            at.k_norm.weight.copy_(p["k_norm"])
            lay.mlp.gate_proj.weight.copy_(p["W4"])
            lay.mlp.up_proj.weight.copy_(p["W5"])
            lay.mlp.down_proj.weight.copy_(p["W6"])
            lay.input_layernorm.weight.copy_(p["ln1_w"])
            lay.post_attention_layernorm.weight.copy_(p["ln2_w"])
    return m


def _oracle_logprobs_all(w, rows):
    hs = om.hidden_states(w, rows, [0.0] * len(rows), 0.0, None)
    logits = hs @ w.lm_head.T
    return torch.log_softmax(logits, dim=-1)


@pytest.mark.parametrize("arch", ["opt", "qwen3"])
def test_forward_matches_transformers(arch):
    if arch == "opt":
        # HF's eager attention takes its softmax in fp32, hence 1e-6 and not 1e-12
        shape, tol = wl.TINY, 1e-6
        w = om.init_weights(shape)
        hf = _hf_opt(w)
    else:
        # HF's RMSNorm and rotary tables compute in fp32, hence the looser bound
        shape, tol = TINY_Q3, 2e-5
        w = om.init_weights(shape)
        hf = _hf_qwen3(w)
    rows = _rows(shape, [5, 17, 32])
    ours = _oracle_logprobs_all(w, rows)
    off = 0
    for r in rows:
        with torch.no_grad():
            out = hf(input_ids=torch.from_numpy(r.astype(np.int64))[None]).logits[0]
        ref = torch.log_softmax(out.double(), dim=-1)
        assert torch.max(torch.abs(ours[off:off + len(r)] - ref)) < tol
        off += len(r)


def test_objective_matches_cross_entropy():
    w = om.init_weights(wl.TINY)
    rows = _rows(wl.TINY, [9, 20])
    tls = [1, 3]
    hs = om.hidden_states(w, rows, [0.0, 0.0], 0.0, None)
    lps = om.token_logprobs(w, hs, rows, tls)
    off = 0
    for r, tl, lp in zip(rows, tls, lps):
        logits = hs[off:off + len(r)] @ w.lm_head.T
        L = len(r)
        ce = torch.nn.functional.cross_entropy(
            logits[L - tl - 1:L - 1], torch.from_numpy(r[L - tl:].astype(np.int64)),
            reduction="none")
        assert torch.allclose(-lp, ce, atol=1e-12, rtol=0)
        off += L


@pytest.mark.parametrize("shape", [wl.TINY, TINY_Q3], ids=["opt", "qwen3"])
def test_rows_independent_and_causal(shape):
    w = om.init_weights(shape)
    rows = _rows(shape, [7, 12, 3], seed=1)
    together = om.hidden_states(w, rows, [0.0] * 3, 0.0, None)
    off = 0
    for r in rows:
        alone = om.hidden_states(w, [r], [0.0], 0.0, None)
        assert torch.allclose(together[off:off + len(r)], alone, atol=1e-12, rtol=0)
        off += len(r)
    # changing the last token leaves every earlier position unchanged
    r = rows[1].copy()
    a = om.hidden_states(w, [r], [0.0], 0.0, None)
    r[-1] = (r[-1] + 1) % shape.vocab
    b = om.hidden_states(w, [r], [0.0], 0.0, None)
    assert torch.equal(a[:-1], b[:-1])
    assert not torch.equal(a[-1], b[-1])


def test_bf16_mode_rounds_weights():
    sh = wl.shrink_shape(wl.TINY, dtype=wl.DTYPE_BF16)
    w = om.init_weights(sh)
    W = w.layers[0]["W0"]
    assert torch.equal(W, W.to(torch.bfloat16).to(torch.float64))
    assert not torch.equal(w.layers[0]["b0"], w.layers[0]["b0"].to(torch.bfloat16).double())


@pytest.mark.parametrize("L,H,Hkv,hd", [(1, 4, 4, 8), (7, 8, 2, 16), (33, 6, 3, 32), (64, 4, 1, 128)])
def test_causal_attention_matches_library_attention_per_head(L, H, Hkv, hd):
    """The oracle's row attention against torch's scaled-dot-product attention (a library
    routine, causal), called once per query head h with kv head h // (H / Hkv): pins the
    1/sqrt(hd) scale, the causal mask, the softmax axis and the grouped-query head mapping
    (query heads sharing a kv head are consecutive)."""
    g = torch.Generator().manual_seed(L * 1000 + H)
    q = torch.randn(L, H, hd, generator=g, dtype=torch.float64)
    k = torch.randn(L, Hkv, hd, generator=g, dtype=torch.float64)
    v = torch.randn(L, Hkv, hd, generator=g, dtype=torch.float64)
    got = om.causal_attention(q, k, v, H // Hkv).reshape(L, H, hd)
    for h in range(H):
        kv = h // (H // Hkv)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[:, h][None, None], k[:, kv][None, None], v[:, kv][None, None], is_causal=True)[0, 0]
        assert torch.allclose(got[:, h], ref, atol=1e-12, rtol=1e-10), h


def test_rope_is_a_rotation_whose_dot_products_depend_on_the_offset_only():
    """Rotary positions (Qwen3's q/k) by their defining properties: position 0 is the
    identity, each (i, i + hd/2) pair keeps its length, and q(m).k(n) depends on m - n only;
    the lowest pair turns by exactly m radians at position m (frequency theta^0 = 1)."""
    hd, theta = 16, 1e6
    g = torch.Generator().manual_seed(3)
    q = torch.randn(1, 1, hd, generator=g, dtype=torch.float64)
    k = torch.randn(1, 1, hd, generator=g, dtype=torch.float64)
    at = lambda x, p: om.rope(x, torch.tensor([p]), theta)  # noqa: E731
    assert torch.equal(at(q, 0), q)
    half = hd // 2
    r = at(q, 37)
    assert torch.allclose(r[..., :half] ** 2 + r[..., half:] ** 2,
                          q[..., :half] ** 2 + q[..., half:] ** 2, atol=1e-12)
    dots = [float((at(q, m) * at(k, m - 5)).sum()) for m in (5, 11, 40, 300)]
    assert max(dots) - min(dots) < 1e-9, dots
    a0 = torch.atan2(q[0, 0, half], q[0, 0, 0])
    a1 = torch.atan2(r[0, 0, half], r[0, 0, 0])
    turn = float((a1 - a0) % (2 * np.pi))
    assert abs(turn - 37 % (2 * np.pi)) < 1e-9, turn


def test_norms_by_definition():
    """LayerNorm gives zero mean and unit variance before its affine terms; RMSNorm unit
    root-mean-square; both scale per feature by w (and LayerNorm shifts by b)."""
    g = torch.Generator().manual_seed(4)
    x = torch.randn(5, 24, generator=g, dtype=torch.float64) * 3 + 2
    one, zero = torch.ones(24, dtype=torch.float64), torch.zeros(24, dtype=torch.float64)
    y = om.layer_norm(x, one, zero, 0.0)
    assert torch.allclose(y.mean(-1), torch.zeros(5, dtype=torch.float64), atol=1e-12)
    assert torch.allclose((y * y).mean(-1), torch.ones(5, dtype=torch.float64), atol=1e-12)
    z = om.rms_norm(x, one, 0.0)
    assert torch.allclose((z * z).mean(-1), torch.ones(5, dtype=torch.float64), atol=1e-12)
    w = torch.randn(24, generator=g, dtype=torch.float64)
    b = torch.randn(24, generator=g, dtype=torch.float64)
    assert torch.allclose(om.layer_norm(x, w, b, 0.0), y * w + b, atol=1e-12)
    assert torch.allclose(om.rms_norm(x, w, 0.0), z * w, atol=1e-12)
