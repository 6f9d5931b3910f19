"""Gates produced from the hidden state, on the GPU through the C ABI, against the fp64 oracle.

The gate kernel computes alpha = sigmoid(x Wa^T + ba) and beta = sigmoid(x Wb^T + bb) per head
from bf16 hidden states (fp32 accumulation on the tensor cores, split over the model width
across a cluster and reduced in a fixed order). The gates themselves are compared element by
element; the gated commit is compared with the oracle's commit on the oracle's gates.
"""
import numpy as np
import pytest
import torch

import oracle
from arl2_cases import S_TOL, Case, dev_bf16, dev_f32, host_f64, s_error
from softmax_attention_ar_b200 import arl2, synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the gpu marker deselects these on CPU-only machines
    pytest.skip("needs a CUDA device", allow_module_level=True)

# fp32 accumulation of up to D = 1536 bf16 products, then an fp32 sigmoid: the gates agree with
# the fp64 oracle far inside this absolute bound (they lie in (0, 1)).
GATE_TOL = 1e-4


def _gate_setup(layer, cfg, H, D):
    wa, ba, wb, bb = synth.gate_weights(0, cfg, H, D)
    layer.set_gate_weights(dev_bf16(wa), dev_bf16(wb), dev_f32(ba), dev_f32(bb))
    return tuple(synth.bf16_to_f64(w) if w.dtype == np.uint16 else w.astype(np.float64) for w in (wa, ba, wb, bb))


@pytest.mark.parametrize("B,T,H,d", [(1, 1560, 12, 128), (2, 300, 12, 128), (1, 1, 2, 32), (3, 129, 4, 64),
                                     (1, 200, 32, 32)])
def test_gates_match_the_oracle(B, T, H, d):
    cfg = 200 + T
    D = H * d
    layer = arl2.ARL2Layer(H, T, d, B)
    wa, ba, wb, bb = _gate_setup(layer, cfg, H, D)
    x = synth.hidden(0, cfg, 0, B, T, D)
    a_gpu, b_gpu = layer.gates(dev_bf16(x))
    a_ref, b_ref = oracle.gates_from_hidden(synth.bf16_to_f64(x), wa, ba, wb, bb)
    assert layer.status() == arl2.ARL2_OK
    assert np.abs(host_f64(a_gpu) - a_ref).max() <= GATE_TOL
    assert np.abs(host_f64(b_gpu) - b_ref).max() <= GATE_TOL
    layer.close()


def test_gated_commit_matches_the_oracle_over_frames():
    # 480p shapes, three frames: the state after every gated commit, against the oracle's
    # commit on the oracle's gates from the same hidden states.
    B, T, H, d, cfg = 1, 1560, 12, 128, 210
    D = H * d
    c = Case(B, T, H, d, config=cfg)
    wa, ba, wb, bb = _gate_setup(c.gpu, cfg, H, D)
    for f in range(3):
        _, k, v = c.inputs(f, synth.CLEAN_PASS)
        x = synth.hidden(0, cfg, f, B, T, D)
        c.gpu.commit_gated(dev_bf16(x), dev_bf16(k), dev_bf16(v))
        assert c.gpu.status() == arl2.ARL2_OK
        s_ref = c.ref.commit(synth.bf16_to_f64(k), synth.bf16_to_f64(v),
                             *oracle.gates_from_hidden(synth.bf16_to_f64(x), wa, ba, wb, bb))
        assert s_error(host_f64(c.gpu.get_state()), s_ref) <= S_TOL, f"frame {f}"


def test_gated_commit_equals_the_commit_on_the_produced_gates():
    B, T, H, d, cfg = 2, 300, 4, 64, 211
    D = H * d
    a_case, b_case = Case(B, T, H, d, config=cfg), Case(B, T, H, d, config=cfg)
    for c in (a_case, b_case):
        _gate_setup(c.gpu, cfg, H, D)
    _, k, v = a_case.inputs(0, synth.CLEAN_PASS)
    x = dev_bf16(synth.hidden(0, cfg, 0, B, T, D))
    a_case.gpu.commit_gated(x, dev_bf16(k), dev_bf16(v))
    alpha, beta = b_case.gpu.gates(x)
    b_case.gpu.commit(dev_bf16(k), dev_bf16(v), alpha, beta)
    torch.cuda.synchronize()
    assert torch.equal(a_case.gpu.get_state(), b_case.gpu.get_state())


def test_gate_calls_check_their_state():
    layer = arl2.ARL2Layer(2, 64, 32, 1)
    x = torch.zeros((1, 64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(arl2.Arl2Error) as e:
        layer.gates(x)
    assert e.value.status == arl2.ARL2_ERR_STATE
    big = arl2.ARL2Layer(33, 64, 32, 1)   # 2H = 66 > 64: gates from x unsupported
    w = torch.zeros((33, 33 * 32), dtype=torch.bfloat16, device="cuda")
    bias = torch.zeros(33, dtype=torch.float32, device="cuda")
    with pytest.raises(arl2.Arl2Error) as e:
        big.set_gate_weights(w, w, bias, bias)
    assert e.value.status == arl2.ARL2_ERR_UNSUPPORTED
