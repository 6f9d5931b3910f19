"""The fused clean pass (query and commit of the clean pass in one launch) on the GPU through
the C ABI, against the fp64 oracle's query then commit on the same inputs.

The query CTAs of the launch run the query's stream-K split on part of the SMs; the commit CTAs
run the commit as a stream of chunk units, and a head split between commit CTAs is reduced by
its last-arriving segment. The tests cover whole and split heads (the split is forced up to
every chunk its own segment), ragged tails, d < 128, several frames in a row and bit-identical
results across runs with the same split.
"""
import pytest
import torch

from arl2_cases import O_TOL, S_TOL, Case, dev_bf16, dev_f32, host_f64, o_errors, s_error
from softmax_attention_ar_b200 import arl2, synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the gpu marker deselects these on CPU-only machines
    pytest.skip("needs a CUDA device", allow_module_level=True)


def clean_pass(c: Case, frame: int):
    """One clean pass on both sides: returns (o_gpu, o_ref, S_gpu, S_ref) in fp64."""
    q, k, v = c.inputs(frame, synth.CLEAN_PASS)
    a, b = c.gates(frame)
    o = c.gpu.clean_pass(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_f32(a), dev_f32(b))
    st = c.gpu.status()
    assert st == arl2.ARL2_OK, f"frame {frame}: device status {st} after the clean pass"
    qf, kf, vf = (synth.bf16_to_f64(x) for x in (q, k, v))
    o_ref = c.ref.query(qf, kf, vf)
    s_ref = c.ref.commit(kf, vf, a, b)
    return host_f64(o), o_ref, host_f64(c.gpu.get_state()), s_ref


def check(c: Case, frame: int):
    o_gpu, o_ref, s_gpu, s_ref = clean_pass(c, frame)
    g, per = o_errors(o_gpu, o_ref)
    assert g <= O_TOL and per <= O_TOL, f"frame {frame}: O error {g:.3e} / {per:.3e}"
    e = s_error(s_gpu, s_ref)
    assert e <= S_TOL, f"frame {frame}: S error {e:.3e}"
    return per, e


@pytest.mark.parametrize("B,T,H,d", [(1, 1, 2, 32), (1, 64, 2, 32), (2, 300, 4, 64), (3, 129, 4, 64),
                                     (1, 1000, 3, 128), (4, 390, 12, 128)])
def test_clean_pass_matches_the_oracle(B, T, H, d):
    c = Case(B, T, H, d, config=300 + T)
    for f in range(2):
        check(c, f)
    assert c.gpu.frame_index == 2


def test_clean_pass_480p_every_row_over_frames():
    # 480p shapes; the first frame starts from S = 0, the next two read a committed state.
    c = Case(1, 1560, 12, 128, config=301)
    worst_o, worst_s = 0.0, 0.0
    for f in range(3):
        o, s = check(c, f)
        worst_o, worst_s = max(worst_o, o), max(worst_s, s)
    print(f"clean pass 480p: worst O error {worst_o:.3e}, worst S error {worst_s:.3e}")


@pytest.mark.parametrize("commit_sms", [1, 5, 40, 147])
def test_forced_splits_reduce_split_heads_correctly(commit_sms):
    # 12 heads of 13 chunks on commit_sms CTAs: from one CTA walking every head to every chunk
    # its own segment (up to 13 segments per head, reduced by the last arrival).
    c = Case(1, 1560, 12, 128, config=302)
    c.gpu.set_clean_split(commit_sms)
    for f in range(2):
        check(c, f)


def test_clean_pass_is_deterministic():
    # Two layers, same split and inputs: bit-identical outputs and states, whichever segment of
    # a split head arrives last.
    runs = []
    for _ in range(2):
        c = Case(2, 1560, 12, 128, config=303)
        c.gpu.set_clean_split(37)
        outs = []
        for f in range(2):
            q, k, v = c.inputs(f, synth.CLEAN_PASS)
            a, b = c.gates(f)
            outs.append(c.gpu.clean_pass(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_f32(a), dev_f32(b)).clone())
        assert c.gpu.status() == arl2.ARL2_OK
        runs.append((outs, c.gpu.get_state().clone()))
    for o0, o1 in zip(runs[0][0], runs[1][0]):
        assert torch.equal(o0, o1)
    assert torch.equal(runs[0][1], runs[1][1])


def test_frames_of_queries_and_clean_passes():
    # The per-frame schedule with the fused clean pass: 4 denoising queries, then the clean
    # pass, over 6 frames with launch overlap on; every query and every state checked.
    c = Case(1, 1560, 12, 128, config=304)
    c.gpu.set_launch_overlap(True)
    for f in range(6):
        for p in range(4):
            o_gpu, o_ref = c.query(f, p)
            g, per = o_errors(o_gpu, o_ref)
            assert g <= O_TOL and per <= O_TOL, f"frame {f} pass {p}: O error {g:.3e}"
        check(c, f)


def test_clean_pass_agrees_with_query_then_commit():
    # Against the two separate calls on the same inputs: the same results up to the order of
    # floating-point sums.
    B, T, H, d = 2, 777, 6, 128
    a_case, b_case = Case(B, T, H, d, config=305), Case(B, T, H, d, config=305)
    for f in range(2):
        q, k, v = (dev_bf16(x) for x in a_case.inputs(f, synth.CLEAN_PASS))
        al, be = (dev_f32(x) for x in a_case.gates(f))
        o_fused = a_case.gpu.clean_pass(q, k, v, al, be)
        o_sep = b_case.gpu.query(q, k, v)
        b_case.gpu.commit(k, v, al, be)
        torch.cuda.synchronize()
        g, per = o_errors(host_f64(o_fused), host_f64(o_sep))
        assert per <= 1e-2
        assert s_error(host_f64(a_case.gpu.get_state()), host_f64(b_case.gpu.get_state())) <= 2e-3
    assert a_case.gpu.status() == arl2.ARL2_OK and b_case.gpu.status() == arl2.ARL2_OK


def test_clean_pass_checks_its_arguments():
    layer = arl2.ARL2Layer(2, 64, 32, 1)
    x = torch.zeros((1, 64, 2, 32), dtype=torch.bfloat16, device="cuda")
    g = torch.zeros((1, 2, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(arl2.Arl2Error) as e:   # feature maps not set yet
        layer.clean_pass(x, x, x, g, g)
    assert e.value.status == arl2.ARL2_ERR_STATE
    with pytest.raises(arl2.Arl2Error) as e:
        layer.set_clean_split(-1)
    assert e.value.status == arl2.ARL2_ERR_INVALID_ARG
    layer.close()
