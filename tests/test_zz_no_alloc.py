"""The allocation-free attention entry point (bsa_attn_fwd_noalloc).

Callers that may not allocate device memory -- a host framework that owns every
device byte through its own pre-reserved pool, or a serving loop where a
cudaMalloc (which can synchronise the device) is not allowed -- call this
variant, which keeps its workspace in a fixed 8 MiB array inside the library.
This file checks, through the C ABI, that two consecutive calls of it give the
same results as bsa_attn_fwd with a caller workspace (within the attention
tolerances used everywhere in the suite), and that a shape needing more than
the fixed scratch is refused before any work.  It is named so that pytest
collects it last.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_tokens_b200 import binding as B
from block_sparse_attention_tokens_b200 import synth
from tests._parity import assert_attention_close, to64

pytestmark = pytest.mark.gpu


def _inputs(Bn, H, nq, nk, D, bq, bk, list_heads, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Bn, nq, H, D, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(Bn, nk, H, D, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(Bn, nk, H, D, generator=g).to(torch.bfloat16).cuda()
    QB, KB = math.ceil(nq / bq), math.ceil(nk / bk)
    mask = synth.random_mask(list_heads * QB, KB, 0.4, seed=seed).reshape(list_heads, QB, KB)
    mask[0, 0] = 0                                    # one row without kept blocks
    rp, ci = B.bsa_mask_compact(torch.from_numpy(mask).cuda())
    return q, k, v, rp, ci


CASES = [  # (batch, heads, nq, nk, head_dim, block_q, block_k, list_heads, seed)
    (1, 2, 1000, 1100, 128, 128, 128, 2, 11),
    (2, 3, 700, 900, 64, 64, 64, 1, 12),
]


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for Bn, H, nq, nk, D, bq, bk, lh, seed in CASES:       # two calls in a row
        q, k, v, rp, ci = _inputs(Bn, H, nq, nk, D, bq, bk, lh, seed)
        o_ref, lse_ref, ws = B.bsa_attn_fwd(q, k, v, rp, ci, bq, bk, lh)
        o, lse = B.bsa_attn_fwd_noalloc(q, k, v, rp, ci, bq, bk, lh, device_status=status)
        torch.cuda.synchronize()
        assert B.bsa_read_status(ws) == 0
        assert int(status.item()) == 0
        D_ = q.shape[-1]
        assert_attention_close(to64(o).reshape(-1, D_), lse.cpu().numpy().astype(np.float64)
                               .transpose(0, 2, 1).reshape(-1),
                               to64(o_ref).reshape(-1, D_), lse_ref.cpu().numpy()
                               .astype(np.float64).transpose(0, 2, 1).reshape(-1),
                               what="noalloc vs workspace entry point")


def test_noalloc_refuses_shapes_beyond_its_scratch():
    # 40 heads with per-head lists over 512 x 512 blocks needs ~42 MB of workspace
    # (the library refuses on the workspace size before it touches any buffer)
    q = torch.zeros(1, 32768, 40, 128, dtype=torch.bfloat16, device="cuda")
    rp = torch.zeros(40 * 512 + 1, dtype=torch.int32, device="cuda")
    ci = torch.zeros(1, dtype=torch.int32, device="cuda")
    need = B.bsa_attn_workspace_size(1, 40, 32768, 32768, 64, 64, 40)
    assert need > 8 << 20
    with pytest.raises(B.BsaError) as e:
        B.bsa_attn_fwd_noalloc(q, q, q, rp, ci, 64, 64, 40)
    assert e.value.code == 3
