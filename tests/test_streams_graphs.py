"""The library as a framework uses it: CUDA-graph capture, several streams at
once, and calls from several host threads. Every call is asynchronous on the
stream it is given and keeps no state between calls (besides the device
status word), so each of these must give the same bits as plain calls."""
import threading

import pytest
import torch

import exact_attention_105_b200 as ea
import workloads

pytestmark = pytest.mark.gpu


def _problem(seed, B=2, Hq=4, Hkv=2, N=700, d=128):
    q, k, v, do = (t.cuda() for t in workloads.make_inputs_qk(B, Hq, Hkv, N, N, d, seed=seed))
    return q, k, v, do


def _eager(q, k, v, do, stream=None):
    o, lse = ea.attn_fwd(q, k, v, causal=True, stream=stream)
    dq, dk, dv = ea.attn_bwd(q, k, v, o, lse, do, causal=True, stream=stream)
    return o, lse, dq, dk, dv


def test_cuda_graph_replay_matches_eager_calls():
    q, k, v, do = _problem(1)
    ref = _eager(q, k, v, do)
    torch.cuda.synchronize()
    o, lse = torch.empty_like(q), torch.empty(q.shape[:3], device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(ea.attn_bwd_workspace_size(2, 4, 700, 128), dtype=torch.uint8, device="cuda")

    def step():
        ea.attn_fwd(q, k, v, o, lse, causal=True)
        ea.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, causal=True)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()                                  # first launches outside the capture
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        step()
    for t in (o, lse, dq, dk, dv):
        t.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    ea.attn_check_status()
    for got, want in zip((o, lse, dq, dk, dv), ref):
        assert torch.equal(got, want)


def test_two_streams_at_once():
    a, b = _problem(2), _problem(3, N=1500)
    ref_a, ref_b = _eager(*a), _eager(*b)
    torch.cuda.synchronize()
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    sa.wait_stream(torch.cuda.current_stream())
    sb.wait_stream(torch.cuda.current_stream())
    outs = {}
    for _ in range(3):
        outs["a"] = _eager(*a, stream=sa)
        outs["b"] = _eager(*b, stream=sb)
    torch.cuda.synchronize()
    ea.attn_check_status()
    for got, want in zip(outs["a"], ref_a):
        assert torch.equal(got, want)
    for got, want in zip(outs["b"], ref_b):
        assert torch.equal(got, want)


def test_calls_from_several_host_threads():
    problems = [_problem(10 + i, N=300 + 200 * i) for i in range(4)]
    refs = [_eager(*p) for p in problems]
    torch.cuda.synchronize()
    results, errors = [None] * 4, []

    def worker(i):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for _ in range(3):
                    results[i] = _eager(*problems[i])
            s.synchronize()
        except Exception as e:     # reported below, on the main thread
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(4)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not errors, errors
    torch.cuda.synchronize()
    ea.attn_check_status()
    for res, ref in zip(results, refs):
        for got, want in zip(res, ref):
            assert torch.equal(got, want)
