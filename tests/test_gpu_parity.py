"""Parity of the CUDA layer (through the C ABI) with the fp64 oracle, and the layer's
GPU-side contracts (state untouched by queries, determinism, constant memory, bounded waits).
"""
import numpy as np
import pytest
import torch

import oracle
from arl2_cases import O_TOL, S_TOL, Case, dev_bf16, dev_f32, host_f64, o_errors, s_error, sample_rows
from softmax_attention_ar_b200 import arl2, synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the gpu marker deselects these on CPU-only machines
    pytest.skip("needs a CUDA device", allow_module_level=True)


# ------------------------------------------------------------------ parity over frames
def test_tiny_config_every_call():
    # Tiny oracle check: B=1, H=2, T=64, d=32, 4 frames of 2 queries + 1 commit.
    w = synth.WORKLOADS["tiny"]
    c = Case(w["B"], w["T"], w["H"], w["d"], config=w["config"])
    c.run(w["frames"], w["queries"])


def test_several_tiles_ragged_tail_batched():
    c = Case(B=2, T=300, H=3, d=128, config=101)
    c.run(frames=3, queries=2)


@pytest.mark.parametrize("d", [32, 64])
def test_smaller_head_dims(d):
    c = Case(B=1, T=200, H=2, d=d, config=102)
    c.run(frames=2, queries=2)


@pytest.mark.parametrize("T", [1, 2, 127, 128, 129, 255])
def test_edge_token_counts(T):
    c = Case(B=1, T=T, H=2, d=128, config=103)
    c.run(frames=2, queries=2)


def test_480p_21_frames_every_row_at_first_and_last_frame():
    # 480p single layer: B=1, H=12, d=128, T=1560, 21 frames of 4 queries + 1 commit. Every
    # row of O is compared on the first query of frames 0 and 20 (every query tile, every
    # stream-K split of this launch shape), sampled rows on the other queries; S after
    # every commit. The worst state error over the 21 commits is printed for the record.
    w = synth.WORKLOADS["480p"]
    c = Case(w["B"], w["T"], w["H"], w["d"], config=w["config"])
    errs = []
    worst_o, worst_s = c.run(w["frames"], w["queries"], rows=sample_rows(w["T"]),
                             full_rows_at=(0, w["frames"] - 1), s_errors=errs)
    print(f"\n480p: worst O error {worst_o:.3e}; worst per-(b,h) S error {worst_s:.3e} "
          f"(after frame {int(np.argmax(errs)) + 1}), after frame 21 {errs[-1]:.3e}")
    assert worst_o <= O_TOL and worst_s <= S_TOL


@pytest.mark.parametrize("B,H,T", [(1, 1, 2048), (1, 2, 200), (2, 3, 300)])
def test_query_tiles_split_across_many_ctas(B, H, T):
    # Few query tiles: the persistent split gives each tile to several CTAs (up to its cap
    # of 8), which merge partial softmax records.
    c = Case(B=B, T=T, H=H, d=128, config=115)
    c.run(frames=2, queries=2)


def test_maximum_tokens_per_frame():
    c = Case(B=1, T=4096, H=2, d=128, config=104)
    c.run(frames=2, queries=1, rows=sample_rows(4096))


@pytest.mark.parametrize("B,T", [(1, 390), (4, 390), (4, 1560), (1, 3600), (4, 3600)])
def test_sweep_shapes(B, T):
    # Token/batch sweep shapes, H=12, d=128 (T=1560 at B=1 is the 480p test). Every row of
    # the first frame's first query is compared; shapes above 400 tokens are checked on
    # sampled rows after that.
    c = Case(B=B, T=T, H=12, d=128, config=3)
    rows = None if T <= 400 else sample_rows(T, n=24)
    c.run(frames=2, queries=2, rows=rows, full_rows_at=(0,))


@pytest.mark.parametrize("T", [1560, 3600])
def test_split_tiles_stay_correct_over_many_launches(T):
    # B=4, H=12: every launch splits query tiles across CTAs that merge partial records. A
    # CTA that stalls at start-up gives up after its bounded wait and reports a time-out, so
    # each launch checks itself: 20 repeats of (query, pause, commit, pause, query), every
    # call ARL2_OK and every repeat bit-identical to the first. The first repeat is also
    # compared with the oracle on sampled rows.
    import time
    B, H, d, cfg = 4, 12, 128, 117
    c = Case(B=B, T=T, H=H, d=d, config=cfg)
    q0, k0, v0 = (dev_bf16(x) for x in c.inputs(0, 0))
    q1, k1, v1 = (dev_bf16(x) for x in c.inputs(1, 0))
    _, kc, vc = (dev_bf16(x) for x in c.inputs(0, synth.CLEAN_PASS))
    a, b = (dev_f32(x) for x in c.gates(0))
    rows = sample_rows(T, 16, seed=3)
    first = None
    for rep in range(20):
        c.gpu.reset()
        o0 = c.gpu.query(q0, k0, v0)
        assert c.gpu.status() == arl2.ARL2_OK, f"rep {rep}: a bounded wait ran out in query 0"
        time.sleep(0.05 if rep % 4 else 0.4)
        c.gpu.commit(kc, vc, a, b)
        assert c.gpu.status() == arl2.ARL2_OK, f"rep {rep}: a bounded wait ran out in the commit"
        time.sleep(0.05 if rep % 4 else 0.4)
        o1 = c.gpu.query(q1, k1, v1)
        assert c.gpu.status() == arl2.ARL2_OK, f"rep {rep}: a bounded wait ran out in query 1"
        outs = (o0.clone(), o1.clone(), c.gpu.get_state().clone())
        if first is None:
            first = outs
            ref0 = c.ref.query(*(synth.bf16_to_f64(x) for x in c.inputs(0, 0)), rows=rows)
            assert max(o_errors(host_f64(o0)[:, rows], ref0)) <= O_TOL
            c.ref.commit(*(synth.bf16_to_f64(x) for x in c.inputs(0, synth.CLEAN_PASS)[1:]), *c.gates(0))
            ref1 = c.ref.query(*(synth.bf16_to_f64(x) for x in c.inputs(1, 0)), rows=rows)
            assert max(o_errors(host_f64(o1)[:, rows], ref1)) <= O_TOL
        else:
            for name, x, y in zip(("query 0", "query 1", "state"), outs, first):
                assert torch.equal(x, y), f"rep {rep}: {name} differs from the first repeat"


def test_calls_after_idle_pauses_on_split_tiles():
    # Each launch follows a pause and fresh uploads, so the kernel's code is often cold when
    # its first CTAs start. A start-up wait that could pass a barrier phase unseen stalled
    # such CTAs until their wait limit ran out; their tiles, and the tiles whose records they
    # owe, were then never written. Every call must report no timeout, and repeats must match
    # bit for bit.
    import time
    B, T, H, d = 4, 1560, 12, 128
    wq, wk, wv = synth.feature_maps(0, 116, H, d)
    first = None
    for rep in range(3):
        layer = arl2.ARL2Layer(H, T, d, B)
        layer.set_feature_maps(dev_bf16(wq), dev_bf16(wk), dev_bf16(wv))
        outs = []
        for f in range(2):
            q, k, v = (dev_bf16(x) for x in synth.qkv(0, 116, f, 0, B, T, H, d))
            outs.append(layer.query(q, k, v).float().cpu())
            assert layer.status() == arl2.ARL2_OK, f"rep {rep} frame {f}: a bounded wait ran out in the query"
            time.sleep(0.5)
            _, k, v = (dev_bf16(x) for x in synth.qkv(0, 116, f, synth.CLEAN_PASS, B, T, H, d))
            a, b = (dev_f32(x) for x in synth.gates(0, 116, f, B, H, T))
            layer.commit(k, v, a, b)
            assert layer.status() == arl2.ARL2_OK, f"rep {rep} frame {f}: a bounded wait ran out in the commit"
            time.sleep(0.5)
        layer.close()
        if first is None:
            first = outs
        else:
            for f, (x, y) in enumerate(zip(outs, first)):
                assert torch.equal(x, y), f"rep {rep} frame {f}: output differs from the first repeat"


# ------------------------------------------------------------------ closed forms on the GPU
def test_queries_leave_the_state_bit_identical():
    c = Case(B=1, T=300, H=2, d=128, config=105)
    c.commit(0)
    before = c.gpu.get_state().clone()
    for p in range(4):
        c.query(1, p)
    torch.cuda.synchronize()
    assert torch.equal(c.gpu.get_state(), before)


def test_alpha_one_beta_zero_keeps_the_state_bit_identical():
    c = Case(B=1, T=300, H=2, d=128, config=106)
    c.gpu.set_state(dev_f32(synth.state(0, 106, 1, 2, 128)))
    before = c.gpu.get_state().clone()
    _, k, v = c.inputs(0, synth.CLEAN_PASS)
    ones = torch.ones((1, 2, 300), device="cuda")
    c.gpu.commit(dev_bf16(k), dev_bf16(v), ones, torch.zeros_like(ones))
    assert torch.equal(c.gpu.get_state(), before)


def test_readout_branch_with_a_set_state():
    # A unit-variance state makes the readout dominate O, which isolates phi_q and Q'S.
    B, T, H, d = 1, 260, 3, 128
    c = Case(B, T, H, d, config=107)
    S0 = synth.state(0, 107, B, H, d)
    c.gpu.set_state(dev_f32(S0))
    c.ref.S = S0.astype(np.float64)
    o_gpu, o_ref = c.query(0, 0)
    assert max(o_errors(o_gpu, o_ref)) <= O_TOL
    q, k, v = c.inputs(0, 0)
    o_inter = oracle.readout(synth.bf16_to_f64(q), c.ref.Wq, c.ref.S)
    assert np.abs(o_inter).max() > 5 * np.abs(o_ref - o_inter).max()  # readout-dominated


def test_pure_decay_over_many_frames():
    # beta = 0 and alpha = c for N frames: S_N = c^N S_0.
    B, T, H, d = 1, 130, 2, 64
    c = Case(B, T, H, d, config=108)
    S0 = synth.state(0, 108, B, H, d)
    c.gpu.set_state(dev_f32(S0))
    _, k, v = c.inputs(0, synth.CLEAN_PASS)
    kk, vv = dev_bf16(k), dev_bf16(v)
    cst = 0.97
    alpha = torch.full((B, H, T), cst, device="cuda")
    beta = torch.zeros_like(alpha)
    for n in range(1, 61):
        c.gpu.commit(kk, vv, alpha, beta)
        if n in (1, 60):
            S = host_f64(c.gpu.get_state())
            np.testing.assert_allclose(S, float(np.float32(cst)) ** n * S0, rtol=1e-4, atol=1e-6)


def test_single_unit_key_writes_its_value():
    # T=1, unit key (phi_k = I), beta/T = 1, alpha = 1: K' S_N = V' (= v @ Wv).
    B, T, H, d = 1, 1, 1, 128
    layer = arl2.ARL2Layer(H, T, d, B)
    eye = dev_bf16(synth.bf16_bits(np.eye(d, dtype=np.float32)[None]))
    _, _, wv = synth.feature_maps(0, 109, H, d)
    layer.set_feature_maps(eye, eye, dev_bf16(wv))
    layer.set_state(dev_f32(synth.state(0, 109, B, H, d, scale=0.1)))
    k = np.zeros((B, T, H, d), np.float32); k[..., 5] = 1.0
    v = np.random.default_rng(0).standard_normal((B, T, H, d)).astype(np.float32)
    kb, vb = synth.bf16_bits(k), synth.bf16_bits(v)
    one = torch.ones((B, H, T), device="cuda")
    layer.commit(dev_bf16(kb), dev_bf16(vb), one, one)
    S = host_f64(layer.get_state())
    vp = synth.bf16_to_f64(vb)[0, 0, 0] @ synth.bf16_to_f64(wv)[0]
    np.testing.assert_allclose(S[0, 0, 5], vp, rtol=0, atol=2e-2 * np.abs(vp).max())


# ------------------------------------------------------------------ contracts
def test_deterministic_outputs_and_state():
    results = []
    for _ in range(2):
        c = Case(B=1, T=520, H=4, d=128, config=110)
        outs = []
        for f in range(2):
            q, k, v = c.inputs(f, 0)
            outs.append(c.gpu.query(dev_bf16(q), dev_bf16(k), dev_bf16(v)).clone())
            c.commit(f)
        outs.append(c.gpu.get_state().clone())
        results.append(outs)
        c.gpu.close()
    for x, y in zip(*results):
        assert torch.equal(x, y)


def test_long_stream_constant_memory_and_state_parity():
    # Long streaming: 480p shapes over 240 frames; memory constant; S checked at 1, 60, 240.
    w = synth.WORKLOADS["stream240"]
    B, T, H, d = w["B"], w["T"], w["H"], w["d"]
    c = Case(B, T, H, d, config=w["config"])
    q, k, v = (dev_bf16(x) for x in c.inputs(0, 0))
    o = torch.empty_like(q)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    held0 = c.gpu.memory_bytes
    errs = {}
    for f in range(w["frames"]):
        for _ in range(w["queries"]):
            c.gpu.query(q, k, v, out=o)
        s_gpu, s_ref = c.commit(f)   # the oracle replays only the commits
        errs[f + 1] = s_error(s_gpu, s_ref)
        if f + 1 in (1, 60, 240):
            assert errs[f + 1] <= S_TOL, f"frame {f + 1}"
    worst = max(errs, key=errs.get)
    print(f"\n240 frames: S error at frames 1/60/240 {errs[1]:.3e} / {errs[60]:.3e} / {errs[240]:.3e}; "
          f"worst {errs[worst]:.3e} after frame {worst}")
    assert errs[worst] <= S_TOL
    torch.cuda.synchronize()
    assert c.gpu.memory_bytes == held0
    assert torch.cuda.mem_get_info()[0] == free0
    assert c.gpu.frame_index == 240
    assert c.gpu.status() == arl2.ARL2_OK


def test_host_buffer_calls_match_device_calls():
    B, T, H, d = 1, 300, 2, 128
    a = Case(B, T, H, d, config=111)
    b = Case(B, T, H, d, config=111)
    q, k, v = a.inputs(0, 0)
    o_dev = a.gpu.query(dev_bf16(q), dev_bf16(k), dev_bf16(v))
    pin = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    o_host = torch.empty((B, T, H, d), dtype=torch.bfloat16).pin_memory()
    b.gpu.query_host(pin(q), pin(k), pin(v), o_host)
    torch.cuda.synchronize()
    assert torch.equal(o_dev.cpu(), o_host)
    _, k, v = a.inputs(0, synth.CLEAN_PASS)
    al, be = a.gates(0)
    a.gpu.commit(dev_bf16(k), dev_bf16(v), dev_f32(al), dev_f32(be))
    b.gpu.commit_host(pin(k), pin(v), torch.from_numpy(al).pin_memory(), torch.from_numpy(be).pin_memory())
    torch.cuda.synchronize()
    assert torch.equal(a.gpu.get_state(), b.gpu.get_state())


def test_reset_and_out_of_order_calls():
    layer = arl2.ARL2Layer(2, 64, 32, 1)
    x = torch.zeros((1, 64, 2, 32), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(arl2.Arl2Error) as e:
        layer.query(x, x, x)
    assert e.value.status == arl2.ARL2_ERR_STATE
    c = Case(B=1, T=64, H=2, d=32, config=112)
    c.commit(0)
    assert c.gpu.frame_index == 1 and torch.any(c.gpu.get_state() != 0)
    c.gpu.reset()
    assert c.gpu.frame_index == 0 and torch.all(c.gpu.get_state() == 0)


def test_bounded_waits_report_a_timeout_and_leave_the_context_usable():
    # The test hook makes one launch wait on a barrier nothing signals: its bounded wait
    # runs out (1 ms limit), every role stops, and the status says so. The context (TMEM,
    # counters, barriers of later launches) stays usable.
    c = Case(B=1, T=300, H=2, d=128, config=113)
    q, k, v = (dev_bf16(x) for x in c.inputs(0, 0))
    c.gpu.set_wait_timeout_ns(1_000_000)
    c.gpu.test_stall_next_query()
    c.gpu.query(q, k, v)
    assert c.gpu.status() == arl2.ARL2_ERR_TIMEOUT
    c.gpu.set_wait_timeout_ns(1_000_000_000)
    assert c.gpu.status() == arl2.ARL2_OK
    o_gpu, o_ref = c.query(0, 0)
    assert max(o_errors(o_gpu, o_ref)) <= O_TOL
    # Several stalled launches in a row, on a split plan (partial records and counters).
    big = Case(B=1, T=1560, H=4, d=128, config=115)
    q, k, v = (dev_bf16(x) for x in big.inputs(0, 0))
    big.gpu.set_wait_timeout_ns(1_000_000)
    for _ in range(3):
        big.gpu.test_stall_next_query()
        big.gpu.query(q, k, v)
        assert big.gpu.status() == arl2.ARL2_ERR_TIMEOUT
    big.gpu.set_wait_timeout_ns(1_000_000_000)
    o_gpu, o_ref = big.query(0, 0, rows=sample_rows(1560, 64, seed=5))
    assert max(o_errors(o_gpu, o_ref)) <= O_TOL


def test_back_to_back_calls_overlapping_the_previous_kernel():
    # With overlap on, each call is launched as a programmatic dependent of the kernel before
    # it (its CTAs start while the previous query's last CTAs still run). Checked: four
    # queries into one output buffer (the last one must win), four into separate buffers,
    # a query whose q is the previous query's output (the guard launches it normally), and
    # a commit right behind a query, followed by a query that reads the new state.
    B, T, H, d = 1, 1560, 4, 128
    c = Case(B, T, H, d, config=116)
    c.gpu.set_launch_overlap(True)
    host = [c.inputs(0, p) for p in range(4)]
    dev = [tuple(dev_bf16(x) for x in qkv) for qkv in host]
    rows = sample_rows(T, 32, seed=7)
    refs = [c.ref.query(*(synth.bf16_to_f64(x) for x in qkv), rows=rows) for qkv in host]
    shared = torch.empty_like(dev[0][0])
    for p in range(4):
        c.gpu.query(*dev[p], out=shared)
    assert max(o_errors(host_f64(shared)[:, rows], refs[3])) <= O_TOL
    outs = [torch.empty_like(dev[0][0]) for _ in range(4)]
    for p in range(4):
        c.gpu.query(*dev[p], out=outs[p])
    for p in range(4):
        assert max(o_errors(host_f64(outs[p])[:, rows], refs[p])) <= O_TOL, f"query {p}"
    o1, o2 = torch.empty_like(dev[0][0]), torch.empty_like(dev[0][0])
    c.gpu.query(*dev[0], out=o1)
    c.gpu.query(o1, dev[1][1], dev[1][2], out=o2)
    q2 = o1.view(torch.int16).cpu().numpy().view(np.uint16)
    ref2 = c.ref.query(synth.bf16_to_f64(q2), synth.bf16_to_f64(host[1][1]), synth.bf16_to_f64(host[1][2]), rows=rows)
    assert max(o_errors(host_f64(o2)[:, rows], ref2)) <= O_TOL
    # A commit right behind a query also overlaps it; then a query must see the new state.
    c.gpu.query(*dev[2], out=outs[0])
    s_gpu, s_ref = c.commit(0)
    assert s_error(s_gpu, s_ref) <= S_TOL
    o_gpu, o_ref = c.query(1, 0, rows=rows)
    assert max(o_errors(o_gpu, o_ref)) <= O_TOL
    assert c.gpu.status() == arl2.ARL2_OK


# ------------------------------------------------------------------ growing-KV baseline
def test_kv_cache_baseline_parity():
    B, T, H, d, frames = 1, 200, 2, 128, 3
    base = arl2.KVCacheBaseline(H, T, d, B, max_frames=frames)
    kc, vc = [], []
    for f in range(frames):
        for p in range(2):
            q, k, v = synth.qkv(0, 114, f, p, B, T, H, d)
            o = host_f64(base.query(dev_bf16(q), dev_bf16(k), dev_bf16(v)))
            keys = np.concatenate(kc + [synth.bf16_to_f64(k)], axis=1)
            vals = np.concatenate(vc + [synth.bf16_to_f64(v)], axis=1)
            ref = oracle.kv_cache_attention(synth.bf16_to_f64(q), keys, vals, (f + 1) * T)
            assert max(o_errors(o, ref)) <= O_TOL
        _, k, v = synth.qkv(0, 114, f, synth.CLEAN_PASS, B, T, H, d)
        base.commit(dev_bf16(k), dev_bf16(v))
        kc.append(synth.bf16_to_f64(k))
        vc.append(synth.bf16_to_f64(v))
    assert base.frames == frames
    assert base.status() == arl2.ARL2_OK
