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


def test_fast_and_checked_paths_agree():
    """Calls with their outputs passed in take the per-step path once a fully
    checked call has run. Its results are bitwise those of the checked path,
    on the current stream and on a given one, and arguments it cannot vouch
    for still get the checked path's errors."""
    q, k, v, do = _problem(7)
    shape_lse = q.shape[:3]
    ws = torch.empty(ea.attn_bwd_workspace_size(2, 4, 700, 128), dtype=torch.uint8, device="cuda")

    def outputs():
        return (torch.empty_like(q), torch.empty(shape_lse, device="cuda"), torch.empty_like(q),
                torch.empty_like(k), torch.empty_like(v))

    o1, lse1, dq1, dk1, dv1 = outputs()
    ea._attn_fwd_checked(q, k, v, o1, lse1, None, True, None)
    ea._attn_bwd_checked(q, k, v, o1, lse1, do, dq1, dk1, dv1, ws, None, True, None)
    assert ea._FAST is not None and ea._FAST[0] is ea.load_library()
    o2, lse2, dq2, dk2, dv2 = outputs()
    ea.attn_fwd(q, k, v, o2, lse2, causal=True)
    ea.attn_bwd(q, k, v, o2, lse2, do, dq2, dk2, dv2, ws, causal=True)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    o3, lse3, dq3, dk3, dv3 = outputs()
    ea.attn_fwd(q, k, v, o3, lse3, causal=True, stream=s)
    ea.attn_bwd(q, k, v, o3, lse3, do, dq3, dk3, dv3, ws, causal=True, stream=s)
    s.synchronize()
    torch.cuda.synchronize()
    ea.attn_check_status()
    for got2, got3, want in zip((o2, lse2, dq2, dk2, dv2), (o3, lse3, dq3, dk3, dv3),
                                (o1, lse1, dq1, dk1, dv1)):
        assert torch.equal(got2, want)
        assert torch.equal(got3, want)
    o_t = torch.empty(q.shape[0], q.shape[2], q.shape[1], q.shape[3], dtype=q.dtype,
                      device="cuda").transpose(1, 2)
    with pytest.raises(ValueError, match="contiguous"):
        ea.attn_fwd(q, k, v, o_t, lse2, causal=True)
    with pytest.raises(TypeError, match="lse must be"):
        ea.attn_fwd(q, k, v, o2, lse2.double(), causal=True)
    with pytest.raises(ValueError, match="shape"):
        ea.attn_fwd(q, k, v[:, :, :600], o2, lse2, causal=True)
    with pytest.raises(TypeError, match="dq must be"):
        ea.attn_bwd(q, k, v, o2, lse2, do, dq2.float(), dk2, dv2, ws, causal=True)


# Causal shapes whose block count makes the host build a block plan (more
# distinct shapes than the plan cache holds, so entries are evicted while other
# threads launch with them).
PLAN_SHAPES = [(3, 16, 1700, 64), (4, 12, 1700, 64), (3, 12, 2300, 64), (2, 20, 2300, 64),
               (2, 16, 2900, 64), (4, 8, 2900, 64), (3, 16, 1700, 128), (4, 12, 1700, 128),
               (2, 12, 3500, 64), (3, 8, 3500, 64)]


def test_causal_plans_from_several_host_threads():
    problems = []
    for i, (B, H, N, d) in enumerate(PLAN_SHAPES):
        q, k, v, _ = workloads.make_inputs_qk(B, H, H, N, N, d, seed=100 + i)
        problems.append(tuple(t.cuda() for t in (q, k, v)))
    refs = [ea.attn_fwd(q, k, v, causal=True) for q, k, v in problems]
    torch.cuda.synchronize()
    results, errors = {}, []

    def worker(w):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                n = len(problems)
                order = [(i + 3 * w) % n for i in range(n)]
                for _ in range(2):
                    for i in (order[::-1] if w % 2 else order):
                        results[(w, i)] = ea.attn_fwd(*problems[i], causal=True)
            s.synchronize()
        except Exception as e:     # reported below, on the main thread
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(w,)) for w in range(3)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not errors, errors
    torch.cuda.synchronize()
    ea.attn_check_status()
    assert results
    for (w, i), (o, lse) in results.items():
        assert torch.equal(o, refs[i][0]) and torch.equal(lse, refs[i][1]), (w, PLAN_SHAPES[i])


def test_dependent_calls_back_to_back():
    """Each forward reads the previous one's output (and a torch kernel sits
    between some of them), with no synchronisation in between: the kernels are
    launched with programmatic stream serialization and may start early, so
    this checks that each one waits for its predecessor's results. Compared
    bit for bit with the same chain synchronised after every call."""
    q, k, v, do = _problem(21, N=900)
    scale = 1.0 / 128 ** 0.5

    def chain(sync):
        x = q
        outs = []
        for i in range(6):
            o, lse = ea.attn_fwd(x, k, v, causal=True, scale=scale)
            if sync:
                torch.cuda.synchronize()
            outs.append((o, lse))
            x = (o * 2.0) if i % 2 else o      # every other link through a torch kernel
        dq, dk, dv = ea.attn_bwd(x, k, v, *ea.attn_fwd(x, k, v, causal=True, scale=scale), do,
                                 causal=True, scale=scale)
        outs.append((dq, dk, dv))
        return outs

    ref = chain(True)
    got = chain(False)
    torch.cuda.synchronize()
    ea.attn_check_status()
    for a, b in zip(got, ref):
        for x, y in zip(a, b):
            assert torch.equal(x, y)


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
