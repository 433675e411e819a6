"""Hypothesis strategy for decoder shapes inside the ranges mk.h accepts: head_dim 64
or 128, 1-4 query heads per KV head (widened so that the query width is a multiple of
256), 1-3 layers, hidden 256-1024, ffn 1024-3072, vocab any multiple of 4 from 64.
Plain data: no arithmetic of the method."""
import dataclasses

from hypothesis import strategies as st

from persistent_megakernel_interpreter_b200.config import TINY


@st.composite
def shapes(draw):
    head_dim = draw(st.sampled_from([64, 128]))
    n_kv = draw(st.sampled_from([1, 2, 4]))
    group = draw(st.sampled_from([1, 2, 3, 4]))
    n_heads = group * n_kv
    if (n_heads * head_dim) % 256:
        n_heads = group * n_kv * (256 // head_dim)  # widen to the next legal head count
        n_kv = n_heads // group
    return dataclasses.replace(
        TINY, name="drawn", n_layers=draw(st.integers(1, 3)),
        hidden=draw(st.sampled_from([256, 512, 768, 1024])), n_heads=n_heads, n_kv_heads=n_kv,
        head_dim=head_dim, ffn=draw(st.sampled_from([1024, 2048, 3072])),
        vocab=4 * draw(st.integers(16, 600)))
