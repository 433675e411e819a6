"""Model shapes for the Llama-style decoder whose decode step the megakernel runs.

The three presets are the decoder shapes the megakernel write-ups measure
("Look Ma, No Bubbles" summaries: Llama-3.2-1B at batch 1), plus a 2-layer
model small enough for an exact CPU check and a 3B-style shape run at batch 8.
A config is plain data: it carries no arithmetic of the method.
"""
from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    name: str
    n_layers: int
    hidden: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float = 1e-5
    rope_theta: float = 500000.0
    tied_embeddings: bool = True

    @property
    def q_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def group(self) -> int:
        return self.n_heads // self.n_kv_heads

    def weight_bytes(self) -> int:
        """bf16 bytes of every matrix and norm vector, the tied table counted once."""
        per_layer = (self.hidden * (self.q_dim + 2 * self.kv_dim)  # W_q, W_k, W_v
                     + self.q_dim * self.hidden                     # W_o
                     + 3 * self.hidden * self.ffn                   # gate, up, down
                     + 2 * self.hidden)                             # two norms
        total = self.n_layers * per_layer + self.vocab * self.hidden + self.hidden
        if not self.tied_embeddings:
            total += self.vocab * self.hidden
        return 2 * total

    def step_bytes(self, batch: int, past: int) -> int:
        """Bytes one decode step must move from HBM at minimum.

        Every matrix once (the tied table once, as the LM head), the embedding
        row of each token, the norm vectors, the read of the ``past`` cached KV
        slots per sequence and layer, and the write of the new slot (whose read
        by attention in the same step is served from L2).
        """
        matrices = (self.n_layers * (self.hidden * (self.q_dim + 2 * self.kv_dim)
                                     + self.q_dim * self.hidden + 3 * self.hidden * self.ffn)
                    + self.vocab * self.hidden)
        if not self.tied_embeddings:
            matrices += self.vocab * self.hidden
        norms = (2 * self.n_layers + 1) * self.hidden
        embed_rows = batch * self.hidden
        kv_slot = 2 * self.n_layers * self.kv_dim            # K and V, all layers
        kv = batch * kv_slot * (past + 1)                     # past reads + 1 write
        return 2 * (matrices + norms + embed_rows + kv)


TINY = ModelConfig("tiny-2l-512", n_layers=2, hidden=512, n_heads=8, n_kv_heads=2,
                   head_dim=64, ffn=2048, vocab=4096)
LLAMA_1B = ModelConfig("llama-3.2-1b", n_layers=16, hidden=2048, n_heads=32, n_kv_heads=8,
                       head_dim=64, ffn=8192, vocab=128256)
LLAMA_3B = ModelConfig("llama-3.2-3b-style", n_layers=28, hidden=3072, n_heads=24,
                       n_kv_heads=8, head_dim=128, ffn=8192, vocab=128256)

PRESETS = {c.name: c for c in (TINY, LLAMA_1B, LLAMA_3B)}
