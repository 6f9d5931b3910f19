"""Shared helpers for the GPU parity tests: seeded inputs on both sides, error measures,
and a runner that drives the CUDA layer and the fp64 oracle through the same frames.

Tolerances (from the layer's accuracy contract):
  O: max|O_gpu - O_ref| / max|O_ref| <= 2e-2, per (batch, head) and over the whole tensor;
  S: ||S_gpu - S_ref||_F / ||S_ref||_F <= 5e-3 per (batch, head), after every commit.
The GPU computes in bf16 MMAs with fp32 accumulation (and a bf16 copy of S for the MMAs
that read it); the oracle works in fp64 on the same bf16-rounded inputs.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from softmax_attention_ar_b200 import synth
from softmax_attention_ar_b200.arl2 import ARL2Layer

O_TOL = 2e-2
S_TOL = 5e-3


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_f32(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def o_errors(o_gpu: np.ndarray, o_ref: np.ndarray):
    """(global, worst per-(b,h)) max-normalised error of O [B, T, H, d]."""
    glob = np.abs(o_gpu - o_ref).max() / np.abs(o_ref).max()
    per = (np.abs(o_gpu - o_ref).max(axis=(1, 3)) / np.abs(o_ref).max(axis=(1, 3))).max()
    return float(glob), float(per)


def s_error(s_gpu: np.ndarray, s_ref: np.ndarray) -> float:
    """Worst per-(b,h) relative Frobenius error of S [B, H, d, d]."""
    num = np.sqrt(((s_gpu - s_ref) ** 2).sum(axis=(2, 3)))
    den = np.sqrt((s_ref ** 2).sum(axis=(2, 3)))
    return float((num / den).max())


class Case:
    """One layer on both sides, with the same seeded feature maps."""

    def __init__(self, B, T, H, d, config=100, seed=0):
        self.B, self.T, self.H, self.d, self.config, self.seed = B, T, H, d, config, seed
        wq, wk, wv = synth.feature_maps(seed, config, H, d)
        self.gpu = ARL2Layer(H, T, d, B)
        self.gpu.set_feature_maps(dev_bf16(wq), dev_bf16(wk), dev_bf16(wv))
        self.ref = oracle.Layer(synth.bf16_to_f64(wq), synth.bf16_to_f64(wk), synth.bf16_to_f64(wv), B)

    def inputs(self, frame, pass_):
        return synth.qkv(self.seed, self.config, frame, pass_, self.B, self.T, self.H, self.d)

    def gates(self, frame):
        return synth.gates(self.seed, self.config, frame, self.B, self.H, self.T)

    def query(self, frame, pass_, rows=None):
        """Run one query on both sides; return (o_gpu rows, o_ref rows) as fp64."""
        q, k, v = self.inputs(frame, pass_)
        o = self.gpu.query(dev_bf16(q), dev_bf16(k), dev_bf16(v))
        st = self.gpu.status()
        assert st == 0, f"frame {frame} pass {pass_}: device status {st} after the query (a bounded wait ran out)"
        o_gpu = host_f64(o)
        ref = self.ref.query(*(synth.bf16_to_f64(x) for x in (q, k, v)), rows=rows)
        if rows is not None:
            o_gpu = o_gpu[:, rows]
        return o_gpu, ref

    def commit(self, frame):
        """Commit the frame's clean pass on both sides; return (S_gpu, S_ref)."""
        _, k, v = self.inputs(frame, synth.CLEAN_PASS)
        a, b = self.gates(frame)
        self.gpu.commit(dev_bf16(k), dev_bf16(v), dev_f32(a), dev_f32(b))
        st = self.gpu.status()
        assert st == 0, f"frame {frame}: device status {st} after the commit (a bounded wait ran out)"
        s_ref = self.ref.commit(synth.bf16_to_f64(k), synth.bf16_to_f64(v), a, b)
        return host_f64(self.gpu.get_state()), s_ref

    def run(self, frames, queries, rows=None, check_every_query=True, full_rows_at=(), s_errors=None):
        """Drive frames x (queries + commit); assert the tolerances; return the worst errors.

        rows: the query rows compared (None = all); on the frames in full_rows_at the first
        query is compared on every row whatever rows says. s_errors, if a list, receives the
        worst per-(b,h) state error after each commit."""
        worst_o, worst_s = 0.0, 0.0
        for f in range(frames):
            for p in range(queries):
                if check_every_query or p == queries - 1:
                    sel = None if (f in full_rows_at and p == 0) else rows
                    o_gpu, o_ref = self.query(f, p, sel)
                    g, per = o_errors(o_gpu, o_ref)
                    assert g <= O_TOL and per <= O_TOL, f"frame {f} pass {p}: O error {g:.3e} / {per:.3e}"
                    worst_o = max(worst_o, per)
            s_gpu, s_ref = self.commit(f)
            e = s_error(s_gpu, s_ref)
            assert e <= S_TOL, f"frame {f}: S error {e:.3e}"
            worst_s = max(worst_s, e)
            if s_errors is not None:
                s_errors.append(e)
        return worst_o, worst_s


def sample_rows(T: int, n: int = 48, seed: int = 0) -> np.ndarray:
    """Query rows to check at large sizes: the first and last tile edges, the ragged tail, random rows."""
    r = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, T - 1, T - 2, (T // 128) * 128]
    rows = set(x for x in fixed if 0 <= x < T)
    rows.update(r.choice(T, size=min(n, T), replace=False).tolist())
    return np.array(sorted(rows))
