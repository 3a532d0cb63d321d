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


def test_row_stride_rule_of_strided_token_tensors():
    # head slice of a [2, 700, 8, 64] tensor: rows 512 elements apart, batches 700 rows apart
    full = torch.empty(2, 700, 8, 64, dtype=BF)
    sl = full[:, :, 2:5]
    assert B._stride_problem(tuple(sl.shape), tuple(sl.stride()), 700, 3 * 64, 8) is None
    # Q of a fused [1, 300, 3, 4, 64] projection: rows 768 elements apart
    qkv = torch.empty(1, 300, 3, 4, 64, dtype=BF)
    q = qkv[:, :, 0]
    assert B._stride_problem(tuple(q.shape), tuple(q.stride()), 300, 4 * 64, 8) is None
    # a padded batch stride (rows per batch != n) is refused for several batches
    pad = torch.empty(2, 704, 3, 64, dtype=BF)
    assert "batch stride" in B._stride_problem(tuple(pad.shape), tuple(pad.stride()), 700,
                                               3 * 64, 8)
    # transposed heads (head_dim not innermost-contiguous) and rows that do not fit
    tr = torch.empty(1, 100, 64, 4, dtype=BF).transpose(2, 3)
    assert "contiguous" in B._stride_problem(tuple(tr.shape), tuple(tr.stride()), 100, 256, 8)
    odd = torch.empty(1, 100, 260, dtype=BF)[:, :, :256].reshape(1, 100, 4, 64)
    assert "multiple of 8" in B._stride_problem(tuple(odd.shape), tuple(odd.stride()), 100,
                                                256, 8)


def test_device_status_must_be_one_int32_word_on_the_gpu():
    # refused before any argument reaches the library: a host tensor would be a
    # host pointer written by a kernel
    import pytest
    x = torch.zeros(1, 8, 1, 8, dtype=BF)
    choice = torch.zeros(1, 1, dtype=torch.int32)
    host_status = torch.zeros(1, dtype=torch.int32)
    with pytest.raises(ValueError, match="device_status"):
        B.bsa_scheme_permute(x, (2, 2, 2), [(1, 1, 1)], choice, 8, device_status=host_status)
    with pytest.raises(ValueError, match="device_status"):
        B.bsa_scheme_untile(x, (2, 2, 2), [(1, 1, 1)], choice, device_status=host_status)
    with pytest.raises(ValueError, match="device_status"):
        B._status(torch.zeros(1, dtype=torch.int64))
    B._status(None)
