"""attn_fwd_splitkv_noalloc: the split-KV pass into the library's own static scratch
instead of a caller workspace (for callers that cannot allocate device memory per
call).  Compared, through the C ABI, with attn_fwd_splitkv on the same inputs and with
the fp64 oracle, within the parity tolerances, on two calls in a row; the cases cover
the D <= 128 kernel and, at D = 256, the wide kernel's split pass."""
import numpy as np
import pytest
import torch

import attention_forward_18_b200 as af
import oracle
from parity import LSE_TOL, O_TOL, compare
from workloads import make_qkv

FAKE = 0x10000000  # 16-byte aligned fake device addresses for argument checks


def test_oversize_is_rejected_before_any_cuda_call():
    # 1 x 32 heads x 1024 rows x 129 floats x 4 bytes is 16.9 MB per split: too big
    B, H, Sq, Sk, D, n = 1, 32, 1024, 8192, 128, 1
    assert af.splitkv_workspace_bytes(B, H, Sq, D, n) > af.SPLITKV_NOALLOC_SCRATCH_BYTES
    rc = af.attn_fwd_splitkv_noalloc(FAKE, FAKE + (1 << 28), FAKE + (2 << 28), FAKE + (3 << 28),
                                     None, B, H, Sq, Sk, D, 0, 0.1, af.ATTN_BF16, n, None)
    assert rc == af.ATTN_ERR_WORKSPACE
    rc = af.attn_fwd_splitkv_noalloc(FAKE, FAKE + (1 << 28), FAKE + (2 << 28), FAKE + (3 << 28),
                                     None, B, H, Sq, Sk, D, 0, 0.1, af.ATTN_BF16, 0, None)
    assert rc == af.ATTN_ERR_SHAPE


def _run_both(q, k, v, causal, n, stream):
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    scale = D ** -0.5
    dt = af.ATTN_BF16 if q.dtype == torch.bfloat16 else af.ATTN_F16
    o_ref = torch.empty_like(q)
    l_ref = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    nbytes = af.splitkv_workspace_bytes(B, H, Sq, D, n)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    rc = af.attn_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o_ref.data_ptr(),
                             l_ref.data_ptr(), B, H, Sq, Sk, D, int(causal), scale, dt, n,
                             ws.data_ptr(), nbytes, stream)
    assert rc == af.ATTN_OK
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    rc = af.attn_fwd_splitkv_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                     lse.data_ptr(), B, H, Sq, Sk, D, int(causal), scale, dt, n,
                                     stream)
    assert rc == af.ATTN_OK
    return o, lse, o_ref, l_ref


@pytest.mark.gpu
def test_two_calls_in_a_row_match_the_workspace_entry_point():
    stream = torch.cuda.current_stream().cuda_stream
    cases = [((2, 8, 4, 5000, 128, "bf16", 31), False, 6),
             ((3, 4, 16, 3000, 64, "f16", 32), True, 3),
             ((1, 4, 1, 3000, 256, "bf16", 33), False, 4)]
    for (B, H, Sq, Sk, D, dt, seed), causal, n in cases:
        qc, kc, vc = make_qkv(B, H, Sq, Sk, D, dt, seed)
        o_orc, l_orc = oracle.attn_ref(qc.double().numpy(), kc.double().numpy(),
                                       vc.double().numpy(), causal, D ** -0.5)
        q, k, v = (t.cuda() for t in (qc, kc, vc))
        o, lse, o_ref, l_ref = _run_both(q, k, v, causal, n, stream)
        torch.cuda.synchronize()
        assert af.attn_fwd_status() == 0
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
        assert (o.float() - o_ref.float()).abs().max().item() <= O_TOL
        assert (lse - l_ref).abs().max().item() <= LSE_TOL
        compare(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_orc, l_orc,
                f"noalloc B{B} H{H} Sq{Sq} Sk{Sk} D{D} splits {n}")
