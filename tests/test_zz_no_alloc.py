"""The allocation-free attention entry point (bsa_attn_fwd_noalloc).

Some callers cannot allocate device memory for a workspace: a host framework
that owns every device byte through its own pre-reserved pool and forbids other
allocations, or a serving loop where a cudaMalloc (which can synchronise the
device) is not allowed.  They call this variant, which keeps its workspace in a
fixed 8 MiB array inside the library.  Through the C ABI this file checks that
  - calls of it in a row give exactly (bit for bit) what bsa_attn_fwd with a
    caller workspace gives on the same inputs -- the same kernels run, so any
    difference would come from the shared scratch -- and agree with the float64
    oracle within the suite's attention tolerances;
  - a call on the same shape with a sparser kept list than the call before it
    keeps nothing stale from that call;
  - a malformed kept list is reported through device_status, not faulted;
  - a shape needing more than the fixed scratch is refused before any work.
It is named so that pytest collects it last.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_tokens_b200 import binding as B
from block_sparse_attention_tokens_b200 import synth
from tests._parity import assert_attention_close, to64

pytestmark = pytest.mark.gpu


def _qkv(Bn, H, nq, nk, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Bn, nq, H, D, generator=g).to(torch.bfloat16)
    k = torch.randn(Bn, nk, H, D, generator=g).to(torch.bfloat16)
    v = torch.randn(Bn, nk, H, D, generator=g).to(torch.bfloat16)
    return q, k, v


def _mask(list_heads, nq, nk, bq, bk, density, seed):
    QB, KB = math.ceil(nq / bq), math.ceil(nk / bk)
    mask = synth.random_mask(list_heads * QB, KB, density, seed=seed).reshape(list_heads, QB, KB)
    mask[0, 0] = 0                                    # one row without kept blocks
    return mask


def _check_call(q, k, v, mask, bq, bk, lh, status, oracle_rows=None):
    """One no-alloc call against bsa_attn_fwd (bit-exact) and the oracle."""
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    rp, ci = B.bsa_mask_compact(torch.from_numpy(mask).cuda())
    o_ref, lse_ref, ws = B.bsa_attn_fwd(qc, kc, vc, rp, ci, bq, bk, lh)
    if status is not None:
        status.fill_(-1)
    o, lse = B.bsa_attn_fwd_noalloc(qc, kc, vc, rp, ci, bq, bk, lh, device_status=status)
    torch.cuda.synchronize()
    assert B.bsa_read_status(ws) == 0
    if status is not None:
        assert int(status.item()) == 0
    assert torch.equal(o, o_ref), "no-alloc O differs from the workspace entry point"
    assert torch.equal(lse, lse_ref), "no-alloc LSE differs from the workspace entry point"
    ro, rl = O.block_sparse_attention(to64(q), to64(k), to64(v), mask, bq, bk, rows=oracle_rows)
    rows = slice(None) if oracle_rows is None else oracle_rows
    D = q.shape[-1]
    assert_attention_close(to64(o)[:, rows].reshape(-1, D),
                           lse.cpu().numpy().astype(np.float64)[..., rows].transpose(0, 2, 1)
                           .reshape(-1),
                           ro[:, rows].reshape(-1, D),
                           rl[..., rows].transpose(0, 2, 1).reshape(-1), what="no-alloc vs oracle")


CASES = [  # (batch, heads, nq, nk, head_dim, block_q, block_k, list_heads, seed)
    (1, 2, 1000, 1100, 128, 128, 128, 2, 11),
    (2, 3, 700, 900, 64, 64, 64, 1, 12),
]


def test_noalloc_equals_workspace_entry_point_and_oracle_on_consecutive_calls():
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for Bn, H, nq, nk, D, bq, bk, lh, seed in CASES:       # two calls in a row
        q, k, v = _qkv(Bn, H, nq, nk, D, seed)
        _check_call(q, k, v, _mask(lh, nq, nk, bq, bk, 0.4, seed), bq, bk, lh, status)


def test_sparser_list_after_denser_on_the_same_shape_keeps_nothing_stale():
    Bn, H, nq, nk, D, bq, bk, lh = 1, 2, 1500, 1500, 128, 128, 128, 2
    q, k, v = _qkv(Bn, H, nq, nk, D, 21)
    dense = _mask(lh, nq, nk, bq, bk, 0.9, 22)
    sparse = _mask(lh, nq, nk, bq, bk, 0.15, 23)
    _check_call(q, k, v, dense, bq, bk, lh, None)          # device_status omitted
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    _check_call(q, k, v, sparse, bq, bk, lh, status)


def test_malformed_list_is_reported_through_device_status():
    q, k, v = (t.cuda() for t in _qkv(1, 1, 256, 256, 128, 31))
    rp = torch.tensor([0, 2, 3], dtype=torch.int32).cuda()
    ci = torch.tensor([0, 1, 9, 0], dtype=torch.int32).cuda()  # block 9 of 2: out of range
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    o, lse = B.bsa_attn_fwd_noalloc(q, k, v, rp, ci, 128, 128, 1, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1                          # BSA_ERR_INVALID_ARG
    # the next call starts from a cleared status word
    rp_ok = torch.tensor([0, 2, 4], dtype=torch.int32).cuda()
    ci_ok = torch.tensor([0, 1, 0, 1], dtype=torch.int32).cuda()
    B.bsa_attn_fwd_noalloc(q, k, v, rp_ok, ci_ok, 128, 128, 1, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_noalloc_refuses_shapes_beyond_its_scratch():
    # 40 heads with per-head lists over 512 x 512 blocks needs ~42 MB of workspace
    # (the library refuses on the workspace size before it touches any buffer)
    q = torch.zeros(1, 32768, 40, 128, dtype=torch.bfloat16, device="cuda")
    rp = torch.zeros(40 * 512 + 1, dtype=torch.int32, device="cuda")
    ci = torch.zeros(40 * 512 * 512, dtype=torch.int32, device="cuda")
    need = B.bsa_attn_workspace_size(1, 40, 32768, 32768, 64, 64, 40)
    assert need > 8 << 20
    with pytest.raises(B.BsaError) as e:
        B.bsa_attn_fwd_noalloc(q, q, q, rp, ci, 64, 64, 40)
    assert e.value.code == 3
