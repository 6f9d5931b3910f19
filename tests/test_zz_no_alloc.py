"""The allocation-free commit (arl2_frame_commit_noalloc) against the context's commit and the oracle.

The entry point is for callers that cannot allocate device memory: a serving engine that
reserved all of it for its own pool, a real-time loop that must not take the allocator's
locks, an embedding that only hands over memory it owns. It keeps its scratch in a fixed
device array inside the library. This test drives it through the C ABI for two frames in
a row: the second call reads the state the first wrote, through the same scratch array.
Its result is compared with the existing context-based commit, to the layer's state
tolerance, and with the fp64 oracle. The file sorts last, so a run that stops at the first
failure has run every other test first.
"""
import numpy as np
import pytest
import torch

import oracle
from arl2_cases import S_TOL, dev_bf16, dev_f32, host_f64, s_error
from softmax_attention_ar_b200 import arl2, synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the gpu marker deselects this on CPU-only machines
    pytest.skip("needs a CUDA device", allow_module_level=True)


def test_noalloc_commit_matches_the_context_commit_on_two_calls_in_a_row():
    B, T, H, d, cfg = 1, 1560, 12, 128, 1
    wq, wk, wv = synth.feature_maps(0, cfg, H, d)
    layer = arl2.ARL2Layer(H, T, d, B)
    layer.set_feature_maps(dev_bf16(wq), dev_bf16(wk), dev_bf16(wv))
    Wk, Wv = dev_bf16(wk), dev_bf16(wv)
    S_a = torch.zeros((B, H, d, d), dtype=torch.float32, device="cuda")
    S_b = torch.empty_like(S_a)
    S_ref = np.zeros((B, H, d, d))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for frame in range(2):
        _, k, v = synth.qkv(0, cfg, frame, synth.CLEAN_PASS, B, T, H, d)
        a, b = synth.gates(0, cfg, frame, B, H, T)
        kd, vd, ad, bd = dev_bf16(k), dev_bf16(v), dev_f32(a), dev_f32(b)
        layer.commit(kd, vd, ad, bd)
        arl2.frame_commit_noalloc(kd, vd, ad, bd, Wk, Wv, S_a, S_b, status=status)
        torch.cuda.synchronize()
        S_ref = oracle.frame_commit(synth.bf16_to_f64(k), synth.bf16_to_f64(v), a, b, synth.bf16_to_f64(wk),
                                    synth.bf16_to_f64(wv), S_ref)
        ctx = host_f64(layer.get_state())
        got = host_f64(S_b)
        assert np.abs(ctx).max() > 0
        assert s_error(got, ctx) <= S_TOL, f"frame {frame}: against the context commit"
        assert s_error(got, S_ref) <= S_TOL, f"frame {frame}: against the oracle"
        assert status.item() == 0
        S_a, S_b = S_b, S_a
    assert layer.status() == arl2.ARL2_OK


def test_noalloc_commit_in_place():
    B, T, H, d, cfg = 2, 300, 3, 64, 7
    _, wk, wv = synth.feature_maps(0, cfg, H, d)
    S0 = synth.state(0, cfg, B, H, d, scale=0.3)
    S = dev_f32(S0)
    S_copy = S.clone()
    out = torch.empty_like(S)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _, k, v = synth.qkv(0, cfg, 0, synth.CLEAN_PASS, B, T, H, d)
    a, b = synth.gates(0, cfg, 0, B, H, T)
    args = (dev_bf16(k), dev_bf16(v), dev_f32(a), dev_f32(b), dev_bf16(wk), dev_bf16(wv))
    arl2.frame_commit_noalloc(*args, S_copy, out, status=status)
    arl2.frame_commit_noalloc(*args, S, S, status=status)          # in place
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(S, out)
    ref = oracle.frame_commit(synth.bf16_to_f64(k), synth.bf16_to_f64(v), a, b, synth.bf16_to_f64(wk),
                              synth.bf16_to_f64(wv), S0.astype(np.float64))
    assert s_error(host_f64(out), ref) <= S_TOL


def test_noalloc_commit_rejects_shapes_beyond_its_scratch():
    B, T, H, d = 64, 4096, 12, 128          # far more than the fixed scratch holds
    lib = arl2.load_library()
    x = torch.zeros(16, dtype=torch.float32, device="cuda")
    p = x.data_ptr()
    st = lib.arl2_frame_commit_noalloc(B, H, T, d, p, p, p, p, p, p, p, p, p,
                                       torch.cuda.current_stream().cuda_stream)
    assert st == arl2.ARL2_ERR_UNSUPPORTED
