"""Token-level access (the ablation the pages contrast with frame-level access) on the GPU
through the C ABI, against the fp64 oracle's token-by-token scan.

The query adds the scan's readout to the intra branch (the query kernel without its readout);
the commit keeps the scan's final state. The scan runs in fp32 on the CUDA cores, eight lanes
per column of S, with the token rows staged in chunks of 32; the shapes cover ragged chunks and
tiles, d in {32, 64, 128} and several frames in a row.
"""
import numpy as np
import pytest
import torch

import oracle
from arl2_cases import O_TOL, S_TOL, Case, dev_bf16, dev_f32, host_f64, o_errors, s_error
from softmax_attention_ar_b200 import arl2, synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the gpu marker deselects these on CPU-only machines
    pytest.skip("needs a CUDA device", allow_module_level=True)


class TokenCase(Case):
    """The GPU layer in token-level mode beside the oracle's token-level functions."""

    def __init__(self, *args, **kw):
        super().__init__(*args, **kw)
        wq, wk, wv = synth.feature_maps(self.seed, self.config, self.H, self.d)
        self.W = tuple(synth.bf16_to_f64(w) for w in (wq, wk, wv))
        self.S = np.zeros((self.B, self.H, self.d, self.d))

    def query(self, frame, pass_):
        q, k, v = self.inputs(frame, pass_)
        a, b = self.gates(frame)
        o = self.gpu.query_token(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_f32(a), dev_f32(b))
        assert self.gpu.status() == arl2.ARL2_OK
        ref = oracle.frame_query_token(*(synth.bf16_to_f64(x) for x in (q, k, v)), a, b, *self.W, self.S)
        return host_f64(o), ref

    def commit(self, frame):
        _, k, v = self.inputs(frame, synth.CLEAN_PASS)
        a, b = self.gates(frame)
        self.gpu.commit_token(dev_bf16(k), dev_bf16(v), dev_f32(a), dev_f32(b))
        assert self.gpu.status() == arl2.ARL2_OK
        self.S = oracle.frame_commit_token(synth.bf16_to_f64(k), synth.bf16_to_f64(v), a, b, self.W[1], self.W[2],
                                           self.S)
        return host_f64(self.gpu.get_state()), self.S


@pytest.mark.parametrize("B,T,H,d", [(1, 1, 2, 32), (1, 64, 2, 32), (2, 300, 4, 64), (1, 129, 3, 128),
                                     (2, 33, 2, 128)])
def test_token_level_matches_the_oracle(B, T, H, d):
    c = TokenCase(B, T, H, d, config=400 + T)
    for f in range(2):
        o_gpu, o_ref = c.query(f, 0)
        g, per = o_errors(o_gpu, o_ref)
        assert g <= O_TOL and per <= O_TOL, f"frame {f}: O error {g:.3e} / {per:.3e}"
        s_gpu, s_ref = c.commit(f)
        assert s_error(s_gpu, s_ref) <= S_TOL, f"frame {f}"


def test_token_level_480p_every_row():
    c = TokenCase(1, 1560, 12, 128, config=401)
    worst_o, worst_s = 0.0, 0.0
    for f in range(2):
        o_gpu, o_ref = c.query(f, 0)
        g, per = o_errors(o_gpu, o_ref)
        assert g <= O_TOL and per <= O_TOL, f"frame {f}: O error {g:.3e} / {per:.3e}"
        s_gpu, s_ref = c.commit(f)
        e = s_error(s_gpu, s_ref)
        assert e <= S_TOL, f"frame {f}: S error {e:.3e}"
        worst_o, worst_s = max(worst_o, per), max(worst_s, e)
    print(f"token-level 480p: worst O error {worst_o:.3e}, worst S error {worst_s:.3e}")


def test_token_query_leaves_the_state_and_is_deterministic():
    c = TokenCase(2, 300, 4, 64, config=402)
    c.commit(0)
    s0 = c.gpu.get_state().clone()
    q, k, v = (dev_bf16(x) for x in c.inputs(1, 0))
    a, b = (dev_f32(x) for x in c.gates(1))
    o1 = c.gpu.query_token(q, k, v, a, b).clone()
    o2 = c.gpu.query_token(q, k, v, a, b).clone()
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert torch.equal(c.gpu.get_state(), s0)
    assert c.gpu.frame_index == 1


def test_token_level_with_no_motion_is_the_frame_level_readout():
    # alpha = 1, beta = 0: the state never moves inside the pass, so every token reads S_{N-1}
    # and the token-level query equals the frame-level one.
    B, T, H, d = 1, 200, 3, 128
    c = Case(B, T, H, d, config=403)
    S = synth.state(0, 403, B, H, d, scale=0.05)
    c.gpu.set_state(dev_f32(S))
    q, k, v = (dev_bf16(x) for x in c.inputs(0, 0))
    ones = torch.ones((B, H, T), dtype=torch.float32, device="cuda")
    zeros = torch.zeros_like(ones)
    o_tok = c.gpu.query_token(q, k, v, ones, zeros)
    o_frame = c.gpu.query(q, k, v)
    torch.cuda.synchronize()
    g, per = o_errors(host_f64(o_tok), host_f64(o_frame))
    assert per <= 1e-2
    c.gpu.commit_token(k, v, ones, zeros)
    torch.cuda.synchronize()
    assert torch.equal(c.gpu.get_state(), dev_f32(S))
