"""Whole-decoder pins for the CPU oracle on the 2-layer config: an fp64 brute
force, the transformers Llama model, special cases and invariants."""
import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, assume, given, settings, strategies as st

import oracle
from oracle.brute import Brute, bf16_bits_to_f64
from persistent_megakernel_interpreter_b200.inputs import make_kv_cache, make_tokens, make_weights
from strategies import shapes


def _np_cache(t):
    return oracle.bits(t).copy()


@pytest.fixture(scope="module")
def setup(tiny_cfg, tiny_weights):
    cfg = tiny_cfg
    om = oracle.Model(cfg, tiny_weights)
    k, v = make_kv_cache(cfg, batch=2, max_seq=160, past=[128, 40], seed=1)
    toks = make_tokens(cfg, 2, seed=2).numpy()
    return cfg, om, k, v, toks


def _brute_caches(cfg, k, v, b):
    K = [bf16_bits_to_f64(k[l, b]).copy() for l in range(cfg.n_layers)]
    V = [bf16_bits_to_f64(v[l, b]).copy() for l in range(cfg.n_layers)]
    return K, V


def test_oracle_vs_fp64_brute_same_rounding_points(setup, tiny_weights):
    """Brute force in fp64 with the same single rounding point (the KV write): the
    oracle's fp32 arithmetic differs only by fp32 accumulation error."""
    cfg, om, k, v, toks = setup
    kc, vc = _np_cache(k), _np_cache(v)
    pos = np.array([128, 40], np.int32)
    logits = om.decode_step(toks, pos, kc, vc)
    br = Brute(cfg, tiny_weights)
    for b in range(2):
        K, V = _brute_caches(cfg, k, v, b)
        ref = br.decode_step(int(toks[b]), int(pos[b]), K, V, rounding=True)
        assert np.max(np.abs(logits[b] - ref)) <= 1e-5 * np.max(np.abs(ref))
        assert int(np.argmax(logits[b])) == int(np.argmax(ref))
        for l in range(cfg.n_layers):   # the new KV slot: same bf16 value (or one ulp apart)
            for got, want in ((kc, K), (vc, V)):
                g = bf16_bits_to_f64(got[l, b, :, pos[b]])
                assert np.all(np.abs(g - want[l][:, pos[b]]) <= 2.0 ** -7 * np.abs(want[l][:, pos[b]]))


def test_oracle_vs_fp64_brute_exact(setup, tiny_weights):
    cfg, om, k, v, toks = setup
    kc, vc = _np_cache(k), _np_cache(v)
    pos = np.array([128, 40], np.int32)
    logits = om.decode_step(toks, pos, kc, vc)
    br = Brute(cfg, tiny_weights)
    for b in range(2):
        K, V = _brute_caches(cfg, k, v, b)
        ref = br.decode_step(int(toks[b]), int(pos[b]), K, V, rounding=False)
        # only the bf16 rounding of the new key/value separates the two
        assert np.max(np.abs(logits[b] - ref)) <= 1e-3 * np.max(np.abs(ref))


def hf_logits(cfg, w, k, v, b, pos, tok):
    """Logits of HF LlamaForCausalLM (fp64, eager attention, no rope scaling) for token
    `tok` at position `pos` of sequence `b`, with keys and values 0..pos-1 of the
    bf16 caches `k` / `v` ([L][B][nkv][S][d] torch tensors) as its past."""
    from transformers import LlamaConfig, LlamaForCausalLM
    from transformers.cache_utils import DynamicCache
    hc = LlamaConfig(vocab_size=cfg.vocab, hidden_size=cfg.hidden, intermediate_size=cfg.ffn,
                     num_hidden_layers=cfg.n_layers, num_attention_heads=cfg.n_heads,
                     num_key_value_heads=cfg.n_kv_heads, head_dim=cfg.head_dim,
                     rms_norm_eps=cfg.rms_eps, rope_theta=cfg.rope_theta,
                     tie_word_embeddings=True, max_position_embeddings=4096,
                     attention_bias=False, mlp_bias=False)
    hc._attn_implementation = "eager"
    model = LlamaForCausalLM(hc).to(torch.float64).eval()
    sd = {"model.embed_tokens.weight": w.embed, "model.norm.weight": w.final_norm,
          "lm_head.weight": w.embed}
    for l in range(cfg.n_layers):
        p = f"model.layers.{l}."
        sd.update({p + "self_attn.q_proj.weight": w.wq[l], p + "self_attn.k_proj.weight": w.wk[l],
                   p + "self_attn.v_proj.weight": w.wv[l], p + "self_attn.o_proj.weight": w.wo[l],
                   p + "mlp.gate_proj.weight": w.wgate[l], p + "mlp.up_proj.weight": w.wup[l],
                   p + "mlp.down_proj.weight": w.wdown[l], p + "input_layernorm.weight": w.attn_norm[l],
                   p + "post_attention_layernorm.weight": w.mlp_norm[l]})
    model.load_state_dict({n: t.to(torch.float64) for n, t in sd.items()}, strict=False)
    cache = DynamicCache()
    for l in range(cfg.n_layers):
        cache.update(k[l, b, :, :pos].to(torch.float64)[None], v[l, b, :, :pos].to(torch.float64)[None], l)
    with torch.no_grad():
        out = model(input_ids=torch.tensor([[int(tok)]]), position_ids=torch.tensor([[pos]]),
                    past_key_values=cache, use_cache=True)
    return out.logits[0, -1].numpy()


def test_oracle_vs_transformers_llama(setup, tiny_weights):
    """Library reduction: HF LlamaForCausalLM (fp32, eager, no rope scaling) fed the same
    weights and the same past K/V returns the same logits up to bf16 rounding."""
    cfg, om, k, v, toks = setup
    kc, vc = _np_cache(k), _np_cache(v)
    b, pos = 0, 128
    ours = om.decode_step(toks[:1], np.array([pos], np.int32), kc[:, :1].copy(), vc[:, :1].copy())
    ref = hf_logits(cfg, tiny_weights, k, v, b, pos, toks[0])
    assert np.max(np.abs(ours[0] - ref)) <= 1e-2 * np.max(np.abs(ref))
    assert int(np.argmax(ours[0])) == int(np.argmax(ref))


def test_zero_residual_branches_give_embedding_logits(tiny_cfg):
    """W_o = W_down = 0: every layer is the identity on x, so logits = E . rms(E[t]) and the
    largest logit is the token itself (its row aligns with itself)."""
    w = make_weights(tiny_cfg, seed=3)
    w.wo = [torch.zeros_like(t) for t in w.wo]
    w.wdown = [torch.zeros_like(t) for t in w.wdown]
    om = oracle.Model(tiny_cfg, w)
    k, v = make_kv_cache(tiny_cfg, 1, 64, past=20)
    kc, vc = _np_cache(k), _np_cache(v)
    E = oracle.bits(w.embed)
    for t in (0, 17, 4095):
        logits = om.decode_step(np.array([t]), np.array([20]), kc, vc)[0]
        y = oracle.rmsnorm(oracle.bf16_to_f32(E[t]), oracle.bits(w.final_norm), tiny_cfg.rms_eps)
        ref = bf16_bits_to_f64(E) @ y.astype(np.float64)
        assert np.max(np.abs(logits - ref)) <= 1e-5 * np.max(np.abs(ref))
        assert oracle.argmax(logits) == t


def test_incremental_decode_equals_causal_forward(tiny_cfg, tiny_weights):
    """Feeding a prefix one token at a time through the cache reproduces the exact
    cache-free causal forward at every position (up to bf16 rounding)."""
    cfg = tiny_cfg
    om = oracle.Model(cfg, tiny_weights)
    T = 12
    toks = make_tokens(cfg, T, seed=5).numpy()
    k, v = make_kv_cache(cfg, 1, 32, past=0)
    kc, vc = _np_cache(k), _np_cache(v)
    inc = np.stack([om.decode_step(toks[t:t + 1], np.array([t]), kc, vc)[0] for t in range(T)])
    full = Brute(cfg, tiny_weights).causal_forward(toks)
    for t in range(T):
        assert np.max(np.abs(inc[t] - full[t])) <= 1e-2 * np.max(np.abs(full[t]))


def test_kv_write_touches_only_slot_pos(setup):
    cfg, om, k, v, toks = setup
    kc, vc = _np_cache(k), _np_cache(v)
    k0, v0 = kc.copy(), vc.copy()
    pos = np.array([128, 40], np.int32)
    om.decode_step(toks, pos, kc, vc)
    for b in range(2):
        mask = np.ones(kc.shape[3], bool)
        mask[pos[b]] = False
        assert np.array_equal(kc[:, b][:, :, mask], k0[:, b][:, :, mask])
        assert np.array_equal(vc[:, b][:, :, mask], v0[:, b][:, :, mask])
        assert not np.array_equal(kc[:, b, :, pos[b]], k0[:, b, :, pos[b]])


def test_batch_rows_are_independent(setup):
    cfg, om, k, v, toks = setup
    pos = np.array([128, 40], np.int32)
    kc, vc = _np_cache(k), _np_cache(v)
    both = om.decode_step(toks, pos, kc, vc)
    for b in range(2):
        kb, vb = _np_cache(k)[:, b:b + 1].copy(), _np_cache(v)[:, b:b + 1].copy()
        one = om.decode_step(toks[b:b + 1], pos[b:b + 1], kb, vb)
        assert np.array_equal(one[0], both[b])
        assert np.array_equal(kb[:, 0], kc[:, b])


def test_bad_inputs_rejected_without_writes(setup):
    cfg, om, k, v, toks = setup
    kc, vc = _np_cache(k), _np_cache(v)
    k0 = kc.copy()
    with pytest.raises(ValueError):
        om.decode_step(np.array([cfg.vocab]), np.array([3]), kc[:, :1].copy(), vc[:, :1].copy())
    with pytest.raises(ValueError):
        om.decode_step(np.array([1]), np.array([160]), kc[:, :1].copy(), vc[:, :1].copy())
    assert np.array_equal(kc, k0)


# The 3B-style head layout (head_dim 128, 3 query heads per KV head) on a small model:
# the same pins as above for the shape the batch-8 workload uses.
def _small_3b_style():
    import dataclasses
    from persistent_megakernel_interpreter_b200.config import LLAMA_3B
    return dataclasses.replace(LLAMA_3B, name="3b-heads-small", n_layers=2, hidden=768, n_heads=6,
                               n_kv_heads=2, ffn=2048, vocab=4096)


@pytest.fixture(scope="module")
def setup_3b_heads():
    cfg = _small_3b_style()
    w = make_weights(cfg, seed=7, norm_jitter=0.1)
    k, v = make_kv_cache(cfg, batch=3, max_seq=96, past=[95, 0, 33], seed=8)
    toks = make_tokens(cfg, 3, seed=9).numpy()
    return cfg, w, k, v, toks


def test_oracle_vs_fp64_brute_3b_head_layout(setup_3b_heads):
    cfg, w, k, v, toks = setup_3b_heads
    assert cfg.head_dim == 128 and cfg.group == 3
    om = oracle.Model(cfg, w)
    kc, vc = _np_cache(k), _np_cache(v)
    pos = np.array([95, 0, 33], np.int32)
    logits = om.decode_step(toks, pos, kc, vc)
    br = Brute(cfg, w)
    for b in range(3):
        K, V = _brute_caches(cfg, k, v, b)
        ref = br.decode_step(int(toks[b]), int(pos[b]), K, V, rounding=True)
        assert np.max(np.abs(logits[b] - ref)) <= 1e-5 * np.max(np.abs(ref)), b
        assert int(np.argmax(logits[b])) == int(np.argmax(ref))


def test_oracle_vs_transformers_llama_3b_head_layout(setup_3b_heads):
    """The library reduction again, for head_dim 128 and 3 query heads per KV head
    (HF's repeat_kv maps query head h to KV head h // 3, as the oracle does)."""
    cfg, w, k, v, toks = setup_3b_heads
    om = oracle.Model(cfg, w)
    b, pos = 2, 33
    kc, vc = _np_cache(k)[:, b:b + 1].copy(), _np_cache(v)[:, b:b + 1].copy()
    ours = om.decode_step(toks[b:b + 1], np.array([pos], np.int32), kc, vc)
    ref = hf_logits(cfg, w, k, v, b, pos, toks[b])
    assert np.max(np.abs(ours[0] - ref)) <= 1e-2 * np.max(np.abs(ref))
    assert int(np.argmax(ours[0])) == int(np.argmax(ref))


@settings(max_examples=12, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])
@given(cfg=shapes(), pos=st.integers(0, 60), seed=st.integers(0, 1000))
def test_oracle_vs_transformers_llama_random_shapes(cfg, pos, seed):
    """The library reduction on drawn shapes (head_dim 64 / 128, 1-4 query heads per KV
    head, 1-3 layers, hidden 256-1024, ffn 1024-3072), norm weights 1 + N(0, 0.1)."""
    assume(cfg.hidden % cfg.n_heads == 0)  # LlamaConfig insists on it
    w = make_weights(cfg, seed=seed, norm_jitter=0.1)
    k, v = make_kv_cache(cfg, batch=1, max_seq=64, past=[pos], seed=seed + 1)
    tok = make_tokens(cfg, 1, seed=seed + 2).numpy()
    ours = oracle.Model(cfg, w).decode_step(tok, np.array([pos], np.int32), _np_cache(k), _np_cache(v))[0]
    ref = hf_logits(cfg, w, k, v, 0, pos, tok[0])
    err = np.max(np.abs(ours - ref))
    assert err <= 1e-2 * np.max(np.abs(ref))
    # random weights can leave the top logits closer than the two sides' rounding: the
    # oracle's choice must then be one of the logits HF cannot tell from its maximum
    assert ref[int(np.argmax(ours))] >= ref.max() - 2 * err
