"""Host-side tensor checks of the Python binding (CPU only): the rule that decides
whether a tensor can serve as the token rows the C ABI reads or writes."""
import torch

from block_sparse_attention_tokens_b200 import binding as B

BF = torch.bfloat16


def test_exact_rows_pass():
    assert B._token_problem((2, 700, 3, 64), BF, 2, 700, 3, 64) is None


def test_padded_tail_is_allowed_for_one_batch_only():
    # one batch: a tile-order buffer of n_pad rows serves n tokens
    assert B._token_problem((1, 33280, 40, 128), BF, 1, 33276, 40, 128) is None
    # several batches: the library's batch stride is n rows, so padding would shift batch 1
    assert "exactly" in B._token_problem((2, 33280, 40, 128), BF, 2, 33276, 40, 128)


def test_too_few_rows_wrong_dtype_or_head_layout_are_refused():
    assert "rows" in B._token_problem((1, 256, 40, 128), BF, 1, 32768, 40, 128)
    assert "bfloat16" in B._token_problem((1, 256, 2, 64), torch.float16, 1, 256, 2, 64)
    assert "must be" in B._token_problem((1, 256, 64, 2), BF, 1, 256, 2, 64)
    assert "must be" in B._token_problem((2, 256, 2, 64), BF, 1, 256, 2, 64)
    assert "must be" in B._token_problem((256, 2, 64), BF, 1, 256, 2, 64)


def test_row_rule_of_the_permutes():
    # 3 x 256-byte rows per token (heads x head_dim bf16), 105 tokens
    assert B._row_problem((2, 105, 2, 64), 2, 2, 105, 256) is None
    assert B._row_problem((1, 128, 2, 64), 2, 1, 105, 256) is None        # padded, one batch
    assert "exactly" in B._row_problem((2, 128, 2, 64), 2, 2, 105, 256)
    assert "rows for" in B._row_problem((1, 100, 2, 64), 2, 1, 105, 256)
    assert "bytes" in B._row_problem((1, 105, 2, 32), 2, 1, 105, 256)
    assert "must be" in B._row_problem((3, 105, 2, 64), 2, 2, 105, 256)
