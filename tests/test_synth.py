"""The seeded generator is deterministic and follows its recipe's shapes (CPU only)."""
import numpy as np
import torch

from block_sparse_attention_tokens_b200 import synth


def test_generator_is_seeded_and_shaped():
    a = synth.generate(1, 3, 16, (2, 3, 4), seed=5, strength_range=(0.5, 3.0))
    b = synth.generate(1, 3, 16, (2, 3, 4), seed=5, strength_range=(0.5, 3.0))
    for x, y in zip(a[:3], b[:3]):
        assert x.dtype == torch.bfloat16 and x.shape == (1, 24, 3, 16)
        assert torch.equal(x, y)
    s = a[3]["strength"]
    assert s.shape == (3,) and np.all((s >= 0.5) & (s <= 3.0))


def test_query_subset_positions():
    q, k, v, _ = synth.generate(1, 2, 8, (4, 2, 3), seed=1, strength=1.5,
                                q_token_ids=np.arange(18, 24))
    assert q.shape == (1, 6, 2, 8) and k.shape == (1, 24, 2, 8)
