"""The seeded input recipe: matrices bf16 N(0, 0.02), norm weights exactly 1 (or
1 + N(0, jitter)), KV slots below `past` N(0, 1) and zero above, tokens uniform in
[0, vocab); the same seed gives the same bytes whatever the thread count, and
different tensors get different streams."""
import numpy as np
import torch

from persistent_megakernel_interpreter_b200 import inputs
from persistent_megakernel_interpreter_b200.config import TINY


def test_weight_distributions_and_shapes():
    w = inputs.make_weights(TINY, seed=0)
    assert w.embed.shape == (TINY.vocab, TINY.hidden) and w.embed.dtype == torch.bfloat16
    assert w.wq[0].shape == (TINY.q_dim, TINY.hidden) and w.wk[0].shape == (TINY.kv_dim, TINY.hidden)
    assert w.wo[0].shape == (TINY.hidden, TINY.q_dim) and w.wdown[0].shape == (TINY.hidden, TINY.ffn)
    for t in (w.embed, w.wgate[1], w.wdown[0]):
        x = t.float().numpy().ravel()
        assert abs(x.mean()) < 3 * 0.02 / np.sqrt(x.size) + 1e-5
        assert abs(x.std() - 0.02) < 0.02 * 0.01
    for t in w.attn_norm + w.mlp_norm + [w.final_norm]:
        assert torch.all(t == 1.0)
    j = inputs.make_weights(TINY, seed=0, norm_jitter=0.1)
    x = torch.cat(j.attn_norm + j.mlp_norm).float().numpy()
    assert abs(x.mean() - 1.0) < 0.02 and abs(x.std() - 0.1) < 0.01
    # distinct tensors draw distinct numbers
    assert not torch.equal(w.wgate[0], w.wup[0]) and not torch.equal(w.wq[0][:64], w.wk[0][:64])


def test_kv_cache_slots_and_distribution():
    past = [100, 0, 37]
    k, v = inputs.make_kv_cache(TINY, 3, 128, past, seed=1)
    assert k.shape == (TINY.n_layers, 3, TINY.n_kv_heads, 128, TINY.head_dim)
    for b, p in enumerate(past):
        assert torch.all(k[:, b, :, p:] == 0) and torch.all(v[:, b, :, p:] == 0)
        if p:
            x = k[:, b, :, :p].float().numpy().ravel()
            assert abs(x.std() - 1.0) < 0.05 and np.count_nonzero(x) == x.size
    assert not torch.equal(k, v)


def test_tokens_are_uniform_in_range():
    t = inputs.make_tokens(TINY, 20000, seed=2).numpy()
    assert t.dtype == np.int32 and t.min() >= 0 and t.max() < TINY.vocab
    counts = np.bincount(t // 512, minlength=TINY.vocab // 512)
    assert counts.min() > 0.8 * counts.mean() and counts.max() < 1.2 * counts.mean()


def test_values_do_not_depend_on_thread_count_and_follow_the_seed():
    n = (1 << 22) * 2 + 1001          # three blocks, the last ragged
    a = inputs._normal_f32(n, 5, 9, threads=1)
    b = inputs._normal_f32(n, 5, 9, threads=3)
    assert np.array_equal(a, b)
    assert not np.array_equal(a[:1000], inputs._normal_f32(1000, 6, 9))
    assert not np.array_equal(a[:1000], inputs._normal_f32(1000, 5, 10))
    assert np.array_equal(inputs.make_tokens(TINY, 8, seed=3), inputs.make_tokens(TINY, 8, seed=3))
