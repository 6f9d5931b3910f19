"""fp64 CPU oracle for the ARL2 hybrid per-frame attention layer.

TEST INFRASTRUCTURE. Only the tests, the package's smoke check and the bench's
CPU-baseline leg may import this module. The CUDA library never calls it, and
it shares no code, table or helper with the CUDA path.

What it restates, from "Attend Locally, Remember Linearly (ARL2)", the
technical summary of arXiv 2605.16579 on gist.science (zh/pt/fr pages):
  * §2.1 hybrid attention decomposition:
      - the intra-frame branch is the original bidirectional softmax
        attention among the tokens of one frame;
      - the inter-frame branch keeps a fixed-size recurrent state S in
        place of the growing KV cache;
      - per-head grouped 1x1 feature maps phi_q, phi_k, phi_v adapt the
        pretrained Q, K, V to that branch;
      - the state update is gated-delta, S_N = a_N S_{N-1} + b_N K'_N (V'_N - K'_N S_{N-1});
      - the readout is O_inter = Q'_N S_{N-1}.
  * §2.2 memory-state management:
      - frame-level access: all tokens of frame N read the same S_{N-1};
      - clean-pass update: denoising passes only read S; S is written
        once per frame, after the clean pass.

Readings of what the pages leave open (plain readings, fixed for this library; the numbers
follow the library's one list of readings, and those missing here fix the schedule, the
input distributions and the tolerances, not this module's arithmetic):
  R1 The update as printed has no transpose and is ill-formed for K' (T x d_k)
     and S (d_k x d_v); it is read as K'^T (V' - K' S).
  R2 alpha and beta are per token; S is per frame. The frame's forget factor is
     the mean of alpha over its T tokens, and token t contributes with rate
     beta_t / T.
  R3 The residual uses the undecayed S_{N-1}, as printed.
  R4 phi maps are linear per head (x' = x W_h), with no bias and no activation.
     Only K' is L2-normalised per token, as k / max(||k||_2, 1e-12).
  R5 The softmax scale is 1/sqrt(d) and no mask is applied inside the frame.
  R6 The two branches are summed: O = O_intra + O_inter.
  R9 Inputs arrive already rounded to bfloat16 and are widened exactly to fp64.
  R13 The per-token gates, where they are produced from the hidden state rather than given,
      are a linear projection of the token's hidden state per head plus a bias, through a
      sigmoid, which keeps both in (0, 1) as a forget gate and a rate must be.
  R15 Token-level access (the ablation of §4 that the pages contrast with frame-level
      access, without giving its form): inside a pass the state advances token by token
      in the frame's token order, with the update rule of §2.1 applied to one token at a
      time (its own alpha_t as the forget gate and beta_t as the rate, the residual against
      the undecayed state as in R3), starting from S_{N-1}. Token t reads the state left by
      tokens 0..t-1, the token-level counterpart of every token reading S_{N-1}. The clean
      pass's final state is S_N.

Array layout: q, k, v are [B, T, H, d] (token-major); feature-map weights are
[H, d_in, d_out]; the state is [B, H, d_k, d_v]; alpha and beta are [B, H, T].
Every function works in float64 with explicit per-(batch, head) loops, so that
each line can be checked against the formulas above by eye.
"""
from __future__ import annotations

import numpy as np

NORM_EPS = 1e-12


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def softmax_rows(scores: np.ndarray) -> np.ndarray:
    """Row-wise softmax of an explicit score matrix (max subtracted for range)."""
    m = scores.max(axis=-1, keepdims=True)
    e = np.exp(scores - m)
    return e / e.sum(axis=-1, keepdims=True)


def attention_matrix(Q: np.ndarray, K: np.ndarray) -> np.ndarray:
    """The explicit T_q x T_k matrix softmax(Q K^T / sqrt(d)) of one head (§2.1, intra branch; R5)."""
    d = Q.shape[-1]
    return softmax_rows((Q @ K.T) / np.sqrt(d))


def intra_attention(q, k, v, rows=None) -> np.ndarray:
    """O_intra = softmax(Q K^T / sqrt(d)) V per (batch, head), unmasked within the frame (§2.1).

    ``rows`` optionally restricts the query rows computed (the keys are always
    the whole frame); the result then has shape [B, len(rows), H, d].
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, H, d = q.shape
    sel = np.arange(T) if rows is None else np.asarray(rows)
    out = np.empty((B, len(sel), H, v.shape[-1]))
    for b in range(B):
        for h in range(H):
            P = attention_matrix(q[b, sel, h, :], k[b, :, h, :])
            out[b, :, h, :] = P @ v[b, :, h, :]
    return out


def feature_map(x, W) -> np.ndarray:
    """phi(x): the per-head grouped 1x1 map, x'[b, t, h, :] = x[b, t, h, :] @ W[h] (§2.1; R4)."""
    x, W = _f64(x), _f64(W)
    B, T, H, _ = x.shape
    out = np.empty((B, T, H, W.shape[2]))
    for h in range(H):
        out[:, :, h, :] = x[:, :, h, :] @ W[h]
    return out


def l2_normalize_rows(x) -> np.ndarray:
    """Each token's vector divided by max(||x||_2, 1e-12) (R4)."""
    x = _f64(x)
    n = np.sqrt((x * x).sum(axis=-1, keepdims=True))
    return x / np.maximum(n, NORM_EPS)


def readout(q, Wq, S, rows=None) -> np.ndarray:
    """O_inter = Q' S_{N-1} with Q' = phi_q(Q) (§2.1 output of the inter-frame branch)."""
    q, S = _f64(q), _f64(S)
    if rows is not None:
        q = q[:, np.asarray(rows)]
    qp = feature_map(q, Wq)
    B, T, H, _ = qp.shape
    out = np.empty((B, T, H, S.shape[-1]))
    for b in range(B):
        for h in range(H):
            out[b, :, h, :] = qp[b, :, h, :] @ S[b, h]
    return out


def frame_query(q, k, v, Wq, S, rows=None):
    """One query pass of the layer: (O, O_intra, O_inter), O = O_intra + O_inter (R6).

    Reads the state of the previous frame and never changes it (§2.2 frame-level access).
    """
    o_intra = intra_attention(q, k, v, rows)
    o_inter = readout(q, Wq, S, rows)
    return o_intra + o_inter, o_intra, o_inter


def frame_commit(k, v, alpha, beta, Wk, Wv, S) -> np.ndarray:
    """The clean-pass state update S_{N-1} -> S_N of one frame (§2.1 update rule, §2.2; R1-R4).

        K' = rownorm(phi_k(K)),  V' = phi_v(V)
        abar = mean_t alpha_t
        S_N = abar * S_{N-1} + K'^T diag(beta / T) (V' - K' S_{N-1})
    """
    kp = l2_normalize_rows(feature_map(k, Wk))
    vp = feature_map(v, Wv)
    alpha, beta, S = _f64(alpha), _f64(beta), _f64(S)
    B, T, H, _ = kp.shape
    S_new = np.empty_like(S)
    for b in range(B):
        for h in range(H):
            Kh, Vh, S0 = kp[b, :, h, :], vp[b, :, h, :], S[b, h]
            abar = alpha[b, h].mean()
            R = (beta[b, h] / T)[:, None] * (Vh - Kh @ S0)
            S_new[b, h] = abar * S0 + Kh.T @ R
    return S_new


class Layer:
    """The layer's per-stream state machine (§2.2): S_0 = 0; queries read S; commits replace it."""

    def __init__(self, Wq, Wk, Wv, B: int):
        self.Wq, self.Wk, self.Wv = _f64(Wq), _f64(Wk), _f64(Wv)
        H, d_k, d_v = self.Wq.shape[0], self.Wk.shape[2], self.Wv.shape[2]
        self.S = np.zeros((B, H, d_k, d_v))
        self.frame = 0

    def reset(self):
        self.S[...] = 0.0
        self.frame = 0

    def query(self, q, k, v, rows=None):
        return frame_query(q, k, v, self.Wq, self.S, rows)[0]

    def commit(self, k, v, alpha, beta):
        self.S = frame_commit(k, v, alpha, beta, self.Wk, self.Wv, self.S)
        self.frame += 1
        return self.S


def gates_from_hidden(x, Wa, ba, Wb, bb):
    """Per-token forget gate and rate from the token's hidden state (§2.1: alpha and beta are
    per-token learned projections; reading R13 fixes their form):

        alpha[b, h, t] = sigmoid(x[b, t, :] . Wa[h, :] + ba[h])
        beta[b, h, t]  = sigmoid(x[b, t, :] . Wb[h, :] + bb[h])

    x is [B, T, D] (D: the layer's model width); Wa, Wb are [H, D]; ba, bb are [H]. Returns
    (alpha, beta), each [B, H, T].
    """
    x, Wa, Wb, ba, bb = _f64(x), _f64(Wa), _f64(Wb), _f64(ba), _f64(bb)
    B, T, _ = x.shape
    H = Wa.shape[0]
    alpha = np.empty((B, H, T))
    beta = np.empty((B, H, T))
    for b in range(B):
        for h in range(H):
            za = x[b] @ Wa[h] + ba[h]
            zb = x[b] @ Wb[h] + bb[h]
            alpha[b, h] = 1.0 / (1.0 + np.exp(-za))
            beta[b, h] = 1.0 / (1.0 + np.exp(-zb))
    return alpha, beta


def frame_commit_gated(x, k, v, Wa, ba, Wb, bb, Wk, Wv, S) -> np.ndarray:
    """The clean-pass commit with its gates produced from the hidden state x (gates_from_hidden)."""
    alpha, beta = gates_from_hidden(x, Wa, ba, Wb, bb)
    return frame_commit(k, v, alpha, beta, Wk, Wv, S)


def token_level_scan(q, k, v, alpha, beta, Wq, Wk, Wv, S):
    """Token-level access (R15): per (batch, head), starting from S_{N-1}, for t = 0..T-1

        o_inter[t] = q'_t S                                    (the state before token t)
        S          = alpha_t S + beta_t k'_t^T (v'_t - k'_t S)   (one token of the §2.1 rule)

    with q' = phi_q(q), k' = rownorm(phi_k(k)), v' = phi_v(v) as in the frame-level layer.
    Returns (O_inter [B, T, H, d_v], the final state [B, H, d_k, d_v]). q may be None (the
    commit needs only the final state)."""
    kp = l2_normalize_rows(feature_map(k, Wk))
    vp = feature_map(v, Wv)
    qp = None if q is None else feature_map(q, Wq)
    alpha, beta, S = _f64(alpha), _f64(beta), _f64(S)
    B, T, H, _ = kp.shape
    o_inter = None if q is None else np.empty((B, T, H, S.shape[-1]))
    S_end = np.empty_like(S)
    for b in range(B):
        for h in range(H):
            St = S[b, h].copy()
            for t in range(T):
                if qp is not None:
                    o_inter[b, t, h] = qp[b, t, h] @ St
                k_t = kp[b, t, h]
                St = alpha[b, h, t] * St + beta[b, h, t] * np.outer(k_t, vp[b, t, h] - k_t @ St)
            S_end[b, h] = St
    return o_inter, S_end


def frame_query_token(q, k, v, alpha, beta, Wq, Wk, Wv, S):
    """One query pass with token-level access (R15): O = O_intra + O_inter, the intra branch as
    in the frame-level layer and the inter branch read token by token. The pass's own k, v and
    gates advance the state inside the pass; the layer's state S_{N-1} is not changed."""
    o_inter, _ = token_level_scan(q, k, v, alpha, beta, Wq, Wk, Wv, S)
    return intra_attention(q, k, v) + o_inter


def frame_commit_token(k, v, alpha, beta, Wk, Wv, S) -> np.ndarray:
    """The clean-pass commit with token-level access (R15): S_N is the state after the clean
    pass's last token."""
    return token_level_scan(None, k, v, alpha, beta, None, Wk, Wv, S)[1]


def kv_cache_attention(q, k_cache, v_cache, length: int, rows=None) -> np.ndarray:
    """The growing-KV-cache baseline the layer replaces (§1 problem statement): the queries of
    the newest frame attend, unmasked, to every cached key of frames 1..N (``length`` tokens)."""
    return intra_attention(q, _f64(k_cache)[:, :length], _f64(v_cache)[:, :length], rows)
