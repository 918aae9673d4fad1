"""CUDA path vs the fp64 oracle on identical seeded inputs, element by element
(max |dO| <= 2e-2, max |dLSE| <= 1e-3), through the C ABI."""
import numpy as np
import pytest
import torch

import attention_forward_18_b200 as af
import oracle
from parity import O_TOL, LSE_TOL, check_full, compare, record, run_gpu
from workloads import WORKLOADS, make_inputs, make_qkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_workload_whole(causal):
    w = WORKLOADS["C1"]
    check_full(w.B, w.H, w.Sq, w.Sk, w.D, w.dtype, causal, w.seed)


RAGGED = [(1, 1), (17, 17), (127, 127), (129, 129), (1000, 1000), (17, 300),
          (300, 17), (129, 1000), (1000, 129), (255, 256), (256, 255), (384, 384)]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", RAGGED)
def test_ragged_shapes(Sq, Sk, causal, dtype, D):
    check_full(2, 3, Sq, Sk, D, dtype, causal, seed=Sq * 7 + Sk)


@pytest.mark.parametrize("causal", [False, True])
def test_bench_workload_whole(causal):
    """C2 (B=4, H=16, S=1024, D=64, fp16), every element, both passes."""
    w = WORKLOADS["C2"]
    rep = check_full(w.B, w.H, w.Sq, w.Sk, w.D, w.dtype, causal, w.seed)
    record(f"C2 causal={causal}", rep)


@pytest.mark.parametrize("name", ["C3", "C4", "C5"])
def test_large_workloads_every_element(name):
    """The full-size workloads of the benchmark step, launched as the benchmark launches
    them, every element of O and LSE against the oracle: its row entry point (each
    row's scores materialised in fp64, masked, softmaxed, times V) over every (b, h, i),
    a few heads per call to bound host memory."""
    w = WORKLOADS[name]
    q, k, v = make_inputs(w)
    qd, kd, vd = q.double().numpy(), k.double().numpy(), v.double().numpy()
    for causal in w.causal:
        o, lse = run_gpu(q, k, v, causal, w.scale)
        o = o.reshape(w.B * w.H, w.Sq, w.D)
        lse = lse.reshape(w.B * w.H, w.Sq)
        per_call = max(1, (1 << 16) // w.Sq)       # heads per oracle call
        total = {"max_dO": 0.0, "max_dLSE": 0.0, "rows": 0}
        for h0 in range(0, w.B * w.H, per_call):
            hs = np.arange(h0, min(h0 + per_call, w.B * w.H))
            bh = np.repeat(hs, w.Sq)
            rows = np.stack([bh // w.H, bh % w.H, np.tile(np.arange(w.Sq), len(hs))], axis=1)
            ro, rl = oracle.attn_ref_rows(qd, kd, vd, rows, causal, w.scale)
            rep = compare(o[hs].reshape(-1, w.D), lse[hs].reshape(-1), ro, rl,
                          f"{name} causal={causal} heads {h0}..{hs[-1]}")
            total["rows"] += len(rows)
            if rep["max_dO"] >= total["max_dO"]:
                r = rows[rep["worst"][0]]
                total.update(max_dO=rep["max_dO"], worst_bhid=[int(r[0]), int(r[1]), int(r[2]),
                                                               int(rep["worst"][1])],
                             abs_O_at_worst=rep["|O| at worst"])
            total["max_dLSE"] = max(total["max_dLSE"], rep["max_dLSE"])
        assert total["rows"] == w.B * w.H * w.Sq
        record(f"{name} causal={causal} (every element)", total)


def test_lse_pointer_may_be_null():
    q, k, v = make_qkv(1, 2, 200, 200, 64, "f16", 11)
    o, lse = run_gpu(q, k, v, True, 0.125, with_lse=False)
    assert lse is None
    o_ref, _ = oracle.attn_ref(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                               True, 0.125)
    assert np.abs(o - o_ref).max() <= O_TOL


@pytest.mark.parametrize("scale", [0.0, -0.3, 1.7])
def test_unusual_scales(scale):
    check_full(1, 2, 130, 260, 64, "bf16", True, seed=5, scale=scale)
    check_full(1, 2, 130, 260, 128, "f16", False, seed=6, scale=scale)


@pytest.mark.parametrize("causal", [False, True])
def test_near_one_hot_rows_in_bf16(causal):
    """Scale 0.5 at D = 128 in bf16: scores spread over tens of log2 units, the row max
    jumps by more than the lazy threshold on later tiles, and |O| reaches max |v|
    (about 4.5), where bf16's own rounding of O is 1/64: the error budget left for the
    rounding of P is small."""
    rep = check_full(2, 4, 300, 1500, 128, "bf16", causal, seed=19 + causal, scale=0.5)
    record(f"near one-hot D128 bf16 causal={causal}", rep)


def test_deterministic_and_stream():
    """Bitwise-identical results over repeated runs, also on a non-default stream."""
    q, k, v = (t.cuda() for t in make_qkv(2, 4, 700, 900, 128, "bf16", 12))
    o1, l1 = af.attention(q, k, v, causal=True)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o2, l2 = af.attention(q, k, v, causal=True, stream=s)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for _ in range(3):
        o3, l3 = af.attention(q, k, v, causal=True)
        assert torch.equal(o1, o3) and torch.equal(l1, l3)
    assert af.attn_fwd_status() == 0


def test_single_head_and_constant_value():
    """B*H = 1; a constant V returns that constant (exactly representable)."""
    q, k, _ = make_qkv(1, 1, 333, 333, 64, "f16", 13)
    v = torch.full((1, 1, 333, 64), 0.75, dtype=torch.float16)
    o, lse = run_gpu(q, k, v, False, 0.125)
    assert np.abs(o - 0.75).max() <= 1e-3


def test_host_buffers_entry_point():
    """attn_fwd_host: pinned host in, host out, same numbers as the device call."""
    B, H, S, D = 2, 2, 300, 128
    q, k, v = make_qkv(B, H, S, S, D, "bf16", 14)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((B, H, S), dtype=torch.float32).pin_memory()
    staging = (torch.empty_like(q, device="cuda"), torch.empty_like(k, device="cuda"),
               torch.empty_like(v, device="cuda"), torch.empty_like(q, device="cuda"),
               torch.empty((B, H, S), dtype=torch.float32, device="cuda"))
    af.attention_host(qh, kh, vh, staging, causal=True, out=oh, lse=lh)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attn_ref(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                   True, 1 / np.sqrt(D))
    compare(oh.double().numpy(), lh.double().numpy(), o_ref, l_ref, "host entry")


HOST_CHUNKED = [
    # (B, H, Sq, Sk, D, dtype, causal, with_lse): Q + K + V of 16 MB or more, which
    # attn_fwd_host pipelines in chunks of whole heads (here 2-8 chunks, the last one
    # shorter where B*H does not divide)
    (1, 7, 4096, 4096, 128, "bf16", True, True),      # 2 chunks: 4 + 3 heads
    (3, 5, 1000, 5000, 64, "f16", False, True),       # 2 chunks: 8 + 7
    (2, 9, 2048, 2048, 128, "bf16", False, False),    # 3 chunks of 6
    (1, 11, 300, 9000, 96, "f16", True, True),        # 4 chunks: 3 + 3 + 3 + 2
    (2, 8, 4096, 4096, 128, "bf16", True, True),      # 6 chunks: 5 x 3 + 1
]


@pytest.mark.parametrize("B,H,Sq,Sk,D,dtype,causal,with_lse", HOST_CHUNKED)
def test_host_buffers_pipelined_chunks(B, H, Sq, Sk, D, dtype, causal, with_lse):
    """attn_fwd_host on passes large enough to run as a pipeline of head chunks: O and
    LSE equal the device entry's bit for bit (a head's arithmetic does not depend on
    which launch runs it), and oracle rows of the first and last head of every possible
    chunk boundary match within the tolerances."""
    q, k, v = make_qkv(B, H, Sq, Sk, D, dtype, 40 + H)
    scale = 1 / np.sqrt(D)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.full((B, H, Sq), 7.0, dtype=torch.float32).pin_memory()
    staging = (torch.empty_like(q, device="cuda"), torch.empty_like(k, device="cuda"),
               torch.empty_like(v, device="cuda"), torch.empty_like(q, device="cuda"),
               torch.empty((B, H, Sq), dtype=torch.float32, device="cuda"))
    side = torch.cuda.Stream()
    af.attention_host(qh, kh, vh, staging, causal=causal, scale=scale, out=oh,
                      lse=lh if with_lse else None, stream=side)
    side.synchronize()
    assert af.attn_fwd_status() == 0
    o_dev, l_dev = af.attention(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert torch.equal(oh, o_dev.cpu())
    if with_lse:
        assert torch.equal(lh, l_dev.cpu())
    else:
        assert bool((lh == 7.0).all())  # no LSE pointer: the host buffer is untouched
    heads = sorted({0, B * H - 1} | {x for c in range(1, 9) for x in
                                     (c * -(-B * H // c) - 1, c * -(-B * H // c))
                                     if 0 <= x < B * H})
    rng = np.random.default_rng(B * H)
    rows = [(bh // H, bh % H, int(i)) for bh in heads
            for i in {0, Sq - 1, *rng.integers(0, Sq, 3).tolist()}]
    o_ref, l_ref = oracle.attn_ref_rows(q.double().numpy(), k.double().numpy(),
                                        v.double().numpy(), np.array(rows), causal, scale)
    o_got = np.stack([oh[b, h, i].double().numpy() for b, h, i in rows])
    l_got = np.array([lh[b, h, i].item() for b, h, i in rows]) if with_lse else None
    compare(o_got, l_got, o_ref, l_ref, "pipelined host entry")


def test_host_buffers_back_to_back_calls_on_one_stream():
    """Two pipelined attn_fwd_host calls queued on one stream without a synchronise in
    between, the second on other inputs but the same staging and host output buffers:
    the host output holds the second call's result (the calls are ordered on the
    stream, copy streams included)."""
    B, H, S, D = 1, 6, 4096, 128
    q1, k1, v1 = make_qkv(B, H, S, S, D, "bf16", 71)
    q2, k2, v2 = make_qkv(B, H, S, S, D, "bf16", 72)
    pinned1 = [t.pin_memory() for t in (q1, k1, v1)]
    pinned2 = [t.pin_memory() for t in (q2, k2, v2)]
    oh = torch.empty_like(q1).pin_memory()
    lh = torch.empty((B, H, S), dtype=torch.float32).pin_memory()
    staging = (torch.empty_like(q1, device="cuda"), torch.empty_like(k1, device="cuda"),
               torch.empty_like(v1, device="cuda"), torch.empty_like(q1, device="cuda"),
               torch.empty((B, H, S), dtype=torch.float32, device="cuda"))
    s = torch.cuda.current_stream()
    af.attention_host(*pinned1, staging, causal=True, out=oh, lse=lh, stream=s)
    af.attention_host(*pinned2, staging, causal=False, out=oh, lse=lh, stream=s)
    s.synchronize()
    o_dev, l_dev = af.attention(q2.cuda(), k2.cuda(), v2.cuda(), causal=False)
    torch.cuda.synchronize()
    assert torch.equal(oh, o_dev.cpu())
    assert torch.equal(lh, l_dev.cpu())


def _host_case(B, H, S, D, seed):
    q, k, v = make_qkv(B, H, S, S, D, "bf16", seed)
    pinned = [t.pin_memory() for t in (q, k, v)]
    oh = torch.zeros_like(q).pin_memory()
    lh = torch.zeros((B, H, S), dtype=torch.float32).pin_memory()
    staging = (torch.empty_like(q, device="cuda"), torch.empty_like(k, device="cuda"),
               torch.empty_like(v, device="cuda"), torch.empty_like(q, device="cuda"),
               torch.empty((B, H, S), dtype=torch.float32, device="cuda"))
    return (q, k, v), pinned, oh, lh, staging


def test_host_buffers_pipeline_in_a_cuda_graph():
    """A pipelined attn_fwd_host call captured into a CUDA graph (its copy streams join
    the capture and rejoin the captured stream), replayed on new host inputs written
    into the same pinned buffers: each replay's host output equals the device entry's."""
    B, H, S, D = 1, 6, 4096, 128
    (q, k, v), pinned, oh, lh, staging = _host_case(B, H, S, D, 81)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        af.attention_host(*pinned, staging, causal=True, out=oh, lse=lh, stream=side)  # warm-up
    side.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        af.attention_host(*pinned, staging, causal=True, out=oh, lse=lh,
                          stream=torch.cuda.current_stream())
    for seed in (82, 83):
        q2, k2, v2 = make_qkv(B, H, S, S, D, "bf16", seed)
        for dst, src in zip(pinned, (q2, k2, v2)):
            dst.copy_(src)
        graph.replay()
        torch.cuda.synchronize()
        assert af.attn_fwd_status() == 0
        o_dev, l_dev = af.attention(q2.cuda(), k2.cuda(), v2.cuda(), causal=True)
        torch.cuda.synchronize()
        assert torch.equal(oh, o_dev.cpu()) and torch.equal(lh, l_dev.cpu())
    del graph


def test_host_buffers_pipeline_from_two_threads():
    """Two host threads calling the pipelined attn_fwd_host at once, each on its own
    stream and buffers (the calls on one device queue one after the other): both host
    outputs equal the device entry's."""
    import threading
    cases = [_host_case(1, 6, 4096, 128, 91), _host_case(2, 3, 4096, 128, 92)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    errors = []

    def worker(i):
        try:
            _, pinned, oh, lh, staging = cases[i]
            for _ in range(3):
                af.attention_host(*pinned, staging, causal=bool(i), out=oh, lse=lh,
                                  stream=streams[i])
            streams[i].synchronize()
        except Exception as e:  # reported in the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    assert af.attn_fwd_status() == 0
    for i, ((q, k, v), _, oh, lh, _) in enumerate(cases):
        o_dev, l_dev = af.attention(q.cuda(), k.cuda(), v.cuda(), causal=bool(i))
        torch.cuda.synchronize()
        assert torch.equal(oh, o_dev.cpu()) and torch.equal(lh, l_dev.cpu())


def test_concurrent_streams_do_not_interfere():
    """The library keeps no per-call state on the device: four passes of different
    shapes, masks and paths (whole, split, grouped heads) in flight at once on four
    streams each match the oracle."""
    cases = [
        (dict(B=2, H=4, Sq=700, Sk=900, D=128, dtype="bf16", seed=91), af.ATTN_MASK_CAUSAL, 0, 4),
        (dict(B=1, H=8, Sq=1, Sk=20000, D=64, dtype="f16", seed=92), af.ATTN_MASK_NONE, None, 8),
        (dict(B=3, H=2, Sq=300, Sk=300, D=64, dtype="f16", seed=93), af.ATTN_MASK_NONE, 0, 2),
        (dict(B=1, H=8, Sq=33, Sk=5000, D=128, dtype="bf16", seed=94),
         af.ATTN_MASK_CAUSAL_BOTTOM_RIGHT, 3, 2),
    ]
    streams = [torch.cuda.Stream() for _ in cases]
    runs = []
    for (kw, mask, n_splits, Hkv), st in zip(cases, streams):
        q, _, _ = make_qkv(kw["B"], kw["H"], kw["Sq"], 1, kw["D"], kw["dtype"], kw["seed"])
        _, k, v = make_qkv(kw["B"], Hkv, 1, kw["Sk"], kw["D"], kw["dtype"], kw["seed"] + 1)
        with torch.cuda.stream(st):
            dq, dk, dv = (t.cuda(non_blocking=False) for t in (q, k, v))
            o, lse = af.attention_ex(dq, dk, dv, mask=mask, scale=0.1, n_splits=n_splits,
                                     stream=st)
        runs.append((q, k, v, mask, o, lse))
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    for (q, k, v, mask, o, lse) in runs:
        o_ref, lse_ref = oracle.attn_ref_ex(q.double().numpy(), k.double().numpy(),
                                            v.double().numpy(), mask, 0.1)
        compare(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref,
                f"stream case mask={mask}")
