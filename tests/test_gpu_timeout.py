"""Failure detection without a GPU fault: a pipeline wait that nothing will satisfy
must end with ATTN_ERR_TIMEOUT in the device status word after its bounded limit,
and the context must stay usable.

The test-only flag of attn_fwd_debug makes the TMA producer skip the Q loads, so
the MMA thread's first wait (for Q) is on a barrier nothing will complete: it gives
up after its 2 s limit, flags the CTA, and every role leaves its loop, drains its own
copies / MMAs, and the CTA frees its tensor memory and exits.  No trap, no fault."""
import time

import numpy as np
import pytest
import torch

import attention_forward_18_b200 as af
from parity import check_full
from workloads import make_qkv

pytestmark = pytest.mark.gpu


def test_unsatisfied_wait_reports_timeout_and_context_survives():
    q, k, v = (t.cuda() for t in make_qkv(1, 2, 256, 256, 64, "f16", 21))
    o = torch.zeros_like(q)
    lse = torch.zeros((1, 2, 256), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert af.attn_fwd_status() == 0
    t0 = time.monotonic()
    rc = af.attn_fwd_debug(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                           lse.data_ptr(), 1, 2, 256, 256, 64, 0, 0.125, af.ATTN_F16, stream, 1)
    assert rc == af.ATTN_OK                   # the launch itself succeeds
    status = af.attn_fwd_status()             # synchronises the stream
    elapsed = time.monotonic() - t0
    assert status == af.ATTN_ERR_TIMEOUT
    assert 1.0 < elapsed < 30.0               # the 2 s limit, not a hang
    assert af.attn_fwd_status() == 0          # reading cleared the word
    # the context is intact: a normal call still gives the oracle's answer
    check_full(1, 2, 200, 300, 64, "f16", True, seed=22)


def test_debug_entry_without_flags_is_the_normal_pass():
    q, k, v = (t.cuda() for t in make_qkv(1, 2, 130, 130, 128, "bf16", 23))
    o1, l1 = af.attention(q, k, v, causal=True)
    o2 = torch.empty_like(q)
    l2 = torch.empty_like(l1)
    rc = af.attn_fwd_debug(q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr(),
                           l2.data_ptr(), 1, 2, 130, 130, 128, 1, 1 / np.sqrt(128),
                           af.ATTN_BF16, torch.cuda.current_stream().cuda_stream, 0)
    assert rc == af.ATTN_OK
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert af.attn_fwd_status() == 0


@pytest.mark.parametrize("D,Sq", [(256, 300), (192, 300), (256, 64)])
def test_starved_pipeline_on_the_wide_head_dimensions(D, Sq):
    """The same starved pipeline on the CTA-pair kernel (D = 192 / 256 with more than 128
    rows: both CTAs of every pair skip their Q loads; rank 0's MMA thread gives up on Q,
    rank 1's softmax gives up on S, each CTA's other roles see its flag, and the two
    meet at the cluster barrier and leave) and on the wide kernel (a decode shape)."""
    q, k, v = (t.cuda() for t in make_qkv(1, 2, Sq, 500, D, "bf16", 24))
    o = torch.zeros_like(q)
    lse = torch.zeros((1, 2, Sq), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert af.attn_fwd_status() == 0
    t0 = time.monotonic()
    rc = af.attn_fwd_debug(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                           lse.data_ptr(), 1, 2, Sq, 500, D, 1, 0.07, af.ATTN_BF16, stream, 1)
    assert rc == af.ATTN_OK
    status = af.attn_fwd_status()
    elapsed = time.monotonic() - t0
    assert status == af.ATTN_ERR_TIMEOUT
    assert 1.0 < elapsed < 30.0
    assert af.attn_fwd_status() == 0
    check_full(1, 2, 300, 400, 64, "f16", False, seed=25)
    # and the kernel itself runs normally again
    o2, l2 = af.attention(q, k, v, causal=True, scale=0.07)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0 and torch.isfinite(o2.float()).all()


@pytest.mark.parametrize("D,Sq", [(64, 300), (128, 300), (256, 300), (256, 64)])
def test_failed_descriptor_encoding_returns_an_error_and_launches_nothing(D, Sq):
    """A TMA descriptor encoding that fails (forced by the host-side debug flag 2, on
    the D <= 128 kernel's, the CTA-pair kernel's and the wide kernel's maps) makes the
    call return ATTN_ERR_TENSORMAP before any launch: the outputs keep their sentinel
    values and the status word stays clear; the next normal call is unaffected."""
    q, k, v = (t.cuda() for t in make_qkv(1, 2, Sq, 400, D, "bf16", 26))
    o = torch.full_like(q, 7.0)
    lse = torch.full((1, 2, Sq), 7.0, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert af.attn_fwd_status() == 0
    rc = af.attn_fwd_debug(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                           lse.data_ptr(), 1, 2, Sq, 400, D, 1, 0.07, af.ATTN_BF16, stream, 2)
    assert rc == af.ATTN_ERR_TENSORMAP
    torch.cuda.synchronize()
    assert bool((o == 7.0).all()) and bool((lse == 7.0).all())
    assert af.attn_fwd_status() == 0
    o2, l2 = af.attention(q, k, v, causal=True, scale=0.07)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0 and torch.isfinite(o2.float()).all()
