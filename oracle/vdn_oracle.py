"""Plain fp64 CPU oracle of the VideoDeltaNet hybrid attention layer (forward).

TEST INFRASTRUCTURE. Only tests/, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` may import this module. The CUDA
library never calls it and shares no code with it.

What it computes, and where each step comes from:

* Latent frames are grouped into blocks of 5 consecutive frames; each block
  attends exactly with itself and its two neighbouring blocks; the first and
  last frames are boundary anchors visible to every block.
  [VDN-MiniMax-H3 (openi.cn), section "技术原理：局部精确、远程压缩";
  "VDN-MiniMax-H3 - OpenVDN's Open-Source Video Generation Acceleration
  Solution" (nav.superapi.store), Technical Principles, "Local Softmax Branch"]
* Text tokens are visible to every frame in the softmax branch; the linear
  branch writes text into its bidirectional state once, at initialisation.
  [nav.superapi.store page, Technical Principles, "Text Dual-Branch Injection"]
* Video Delta Attention: one joint normal-equation update per frame, replacing
  the token-by-token delta rule; non-expansive.
  [nav.superapi.store page, Technical Principles, "Video Delta Attention";
  openi.cn page, 主要功能 item 3]
* The linear branch sums the context before and after the current window and
  leaves out the window frames and the anchors.
  [openi.cn page, "技术原理：局部精确、远程压缩"]
* Each branch has a content-dependent sigmoid gate; the linear output is
  RMS-normalised before its gate. [openi.cn page, same section, last
  paragraph; nav.superapi.store page, "Gated Fusion Mechanism"]

The pages print no equations. The exact reading used here (the one the CUDA
library implements too):

* softmax scale 1/sqrt(d); video queries only (text tokens are keys/values);
* keys are L2-normalised inside the linear branch (floor 1e-12); lambda = 1;
* S_text = (lam I + Kt^T Kt)^-1 Kt^T Vt;
* frame update S_f = (lam I + K_f^T K_f)^-1 (lam S_prev + K_f^T V_f);
* forward scan over frames 1..F-2 from S_text, backward scan over F-2..1 from
  S_text (anchors excluded from both);
* block b reads R_b = S_fwd[max(w0-1, 0)] + S_bwd[min(w1+1, F-1)] where
  [w0, w1] is b's window of frames and S_fwd[0] = S_bwd[F-1] = S_text;
* o_lin = q^T R_b (q not normalised); RMSNorm over d per head, eps 1e-6,
  weight w[h, :];
* out = sigmoid(g_s) o_soft + sigmoid(g_l) RMSNorm(o_lin);
* with per-branch output projections (w_o = [W_s | W_l], [D, 2 H d]):
  y = W_s (sigmoid(g_s) o_soft) + W_l (sigmoid(g_l) RMSNorm(o_lin)), heads
  flattened as h * d + j.

Parity is pinned by tests/test_oracle_pins.py (dense-mask equivalence,
Sherman-Morrison, ridge closed form, orthonormal-key delta steps, fixed point,
non-expansiveness, pair-set coverage, RMSNorm closed form, readout
orientation, text start of both scans) and tests/test_oracle_proj.py
(projection: identity weights, brute-force loops, gate limits). The comparison of
the pair split with the pages' ~52%/48% and +3.57% figures is reported, not
pinned ("parity unpinned" for those two statistics: no uniform frame layout
reproduces both figures).
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# Frame blocks, windows, anchors (integer structure)
# ---------------------------------------------------------------------------


def num_blocks(F: int, bf: int = 5) -> int:
    """Number of blocks of ``bf`` consecutive latent frames (last may be short)."""
    return -(-F // bf)


def block_of(f: int, bf: int = 5) -> int:
    return f // bf


def window(b: int, F: int, bf: int = 5):
    """First and last frame of block b's softmax window: blocks b-1, b, b+1,
    clipped at the ends of the clip."""
    w0 = bf * max(b - 1, 0)
    w1 = min(bf * (b + 2), F) - 1
    return w0, w1


def softmax_key_frames(b: int, F: int, bf: int = 5):
    """Frames whose tokens are softmax keys for queries of block b: the window
    plus the two boundary anchors (frames 0 and F-1)."""
    w0, w1 = window(b, F, bf)
    return sorted(set(range(w0, w1 + 1)) | {0, F - 1})


def read_indices(b: int, F: int, bf: int = 5):
    """Indices of the forward and backward scan states that block b reads:
    the forward state just before the window and the backward state just
    after it (index 0 / F-1 stand for the text-initialised state)."""
    w0, w1 = window(b, F, bf)
    return max(w0 - 1, 0), min(w1 + 1, F - 1)


def linear_key_frames(b: int, F: int, bf: int = 5):
    """Frames folded into block b's linear read state, derived from the scan
    structure: the forward state at index i covers frames 1..i, the backward
    state at index j covers frames j..F-2."""
    i_f, i_b = read_indices(b, F, bf)
    return sorted(set(range(1, i_f + 1)) | set(range(i_b, F - 1)))


def pair_class_matrix(F: int, bf: int = 5) -> np.ndarray:
    """C[f, g] = 1 if key frame g is in the softmax branch of query frame f,
    2 if it is in the linear branch, 0 if in neither (3 would mean both)."""
    C = np.zeros((F, F), dtype=np.int64)
    for f in range(F):
        b = block_of(f, bf)
        for g in softmax_key_frames(b, F, bf):
            C[f, g] += 1
        for g in linear_key_frames(b, F, bf):
            C[f, g] += 2
    return C


def pair_counts(off, bf: int = 5, T: int = 0):
    """Token-pair counts per (query frame, key frame).

    Returns (soft[F, F+1], lin[F, F]) int64: soft[:, F] counts text pairs.
    """
    off = np.asarray(off, dtype=np.int64)
    F = len(off) - 1
    n = np.diff(off)
    C = pair_class_matrix(F, bf)
    soft = np.zeros((F, F + 1), dtype=np.int64)
    lin = np.zeros((F, F), dtype=np.int64)
    soft[:, :F] = np.where(C == 1, np.outer(n, n), 0)
    soft[:, F] = n * T
    lin[:, :] = np.where(C == 2, np.outer(n, n), 0)
    return soft, lin


# ---------------------------------------------------------------------------
# Softmax branch
# ---------------------------------------------------------------------------


def _softmax_rows(S: np.ndarray) -> np.ndarray:
    m = np.max(S, axis=1, keepdims=True)
    P = np.exp(S - m)
    return P / np.sum(P, axis=1, keepdims=True)


def softmax_branch_head(q, k, v, kt, vt, off, h: int, bf: int = 5,
                        rows=None) -> np.ndarray:
    """o_soft for one head, gathering the allowed keys block by block.

    q, k, v: [N, H, d]; kt, vt: [T, H, d]. If ``rows`` (sorted token indices)
    is given, only those query rows are computed. Returns [len(rows) or N, d]
    float64.
    """
    off = np.asarray(off, dtype=np.int64)
    F = len(off) - 1
    N = int(off[-1])
    d = q.shape[2]
    scale = 1.0 / np.sqrt(d)
    all_rows = np.arange(N) if rows is None else np.asarray(rows)
    frame_of = np.searchsorted(off, all_rows, side="right") - 1
    out = np.zeros((len(all_rows), d), dtype=np.float64)
    ktt = np.asarray(kt[:, h], dtype=np.float64)
    vtt = np.asarray(vt[:, h], dtype=np.float64)
    for b in range(num_blocks(F, bf)):
        sel = np.nonzero(block_of(frame_of, bf) == b)[0]
        if len(sel) == 0:
            continue
        frames = softmax_key_frames(b, F, bf)
        K = np.concatenate([np.asarray(k[off[g]:off[g + 1], h], np.float64)
                            for g in frames] + [ktt])
        V = np.concatenate([np.asarray(v[off[g]:off[g + 1], h], np.float64)
                            for g in frames] + [vtt])
        Q = np.asarray(q[all_rows[sel], h], dtype=np.float64)
        out[sel] = _softmax_rows(Q @ K.T * scale) @ V
    return out


def softmax_branch_dense_mask(q, k, v, kt, vt, off, h: int,
                              bf: int = 5) -> np.ndarray:
    """The same branch written as dense attention over all N+T keys with an
    explicit boolean mask built from per-token frame ids (a second, separate
    formulation used to pin ``softmax_branch_head``)."""
    off = np.asarray(off, dtype=np.int64)
    F = len(off) - 1
    N = int(off[-1])
    d = q.shape[2]
    fid = np.repeat(np.arange(F), np.diff(off))
    bq = fid // bf
    near = np.abs(bq[:, None] - bq[None, :]) <= 1
    anchor = (fid[None, :] == 0) | (fid[None, :] == F - 1)
    mask = np.concatenate([near | anchor, np.ones((N, kt.shape[0]), bool)],
                          axis=1)
    K = np.concatenate([k[:, h], kt[:, h]]).astype(np.float64)
    V = np.concatenate([v[:, h], vt[:, h]]).astype(np.float64)
    S = q[:, h].astype(np.float64) @ K.T / np.sqrt(d)
    S = np.where(mask, S, -np.inf)
    return _softmax_rows(S) @ V


# ---------------------------------------------------------------------------
# Video Delta Attention (linear branch)
# ---------------------------------------------------------------------------


def l2_normalise(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    nrm = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(nrm, 1e-12)


def text_state(Kt_hat, Vt, lam: float) -> np.ndarray:
    """S_text = (lam I + Kt^T Kt)^-1 Kt^T Vt (text written once at init)."""
    Kt_hat = np.asarray(Kt_hat, np.float64)
    Vt = np.asarray(Vt, np.float64)
    d = Kt_hat.shape[1]
    M = lam * np.eye(d) + Kt_hat.T @ Kt_hat
    return np.linalg.solve(M, Kt_hat.T @ Vt)


def frame_update(S_prev, K_hat, V, lam: float) -> np.ndarray:
    """Frame-joint normal-equation update of the d x d state:
    S_f = (lam I + K^T K)^-1 (lam S_prev + K^T V), solved by LU."""
    K_hat = np.asarray(K_hat, np.float64)
    V = np.asarray(V, np.float64)
    d = K_hat.shape[1]
    M = lam * np.eye(d) + K_hat.T @ K_hat
    return np.linalg.solve(M, lam * np.asarray(S_prev, np.float64) + K_hat.T @ V)


def vda_states_head(k, v, kt, vt, off, h: int, lam: float = 1.0,
                    bf: int = 5) -> dict:
    """Text state, per-frame forward/backward states and per-block read
    states for one head.

    Returns dict with S_text [d,d], fwd {i: [d,d]} for i in 0..F-2 (0 is
    S_text), bwd {i: [d,d]} for i in 1..F-1 (F-1 is S_text), R [nb, d, d].
    """
    off = np.asarray(off, dtype=np.int64)
    F = len(off) - 1
    S_text = text_state(l2_normalise(kt[:, h]), vt[:, h], lam)
    fwd = {0: S_text}
    for f in range(1, F - 1):
        fwd[f] = frame_update(fwd[f - 1], l2_normalise(k[off[f]:off[f + 1], h]),
                              v[off[f]:off[f + 1], h], lam)
    bwd = {F - 1: S_text}
    for f in range(F - 2, 0, -1):
        bwd[f] = frame_update(bwd[f + 1], l2_normalise(k[off[f]:off[f + 1], h]),
                              v[off[f]:off[f + 1], h], lam)
    nb = num_blocks(F, bf)
    R = np.zeros((nb,) + S_text.shape)
    for b in range(nb):
        i_f, i_b = read_indices(b, F, bf)
        R[b] = fwd[i_f] + bwd[i_b]
    return dict(S_text=S_text, fwd=fwd, bwd=bwd, R=R)


def rmsnorm(o, w, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: o * w / sqrt(mean(o^2) + eps)."""
    o = np.asarray(o, np.float64)
    return o * np.asarray(w, np.float64) / np.sqrt(np.mean(o * o, axis=-1,
                                                           keepdims=True) + eps)


def sigmoid(x) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-np.asarray(x, np.float64)))


def gate_merge(o_soft, o_lin, g_s, g_l, w, eps: float) -> np.ndarray:
    """out = sigmoid(g_s) o_soft + sigmoid(g_l) RMSNorm(o_lin) (one head)."""
    return (sigmoid(g_s)[:, None] * np.asarray(o_soft, np.float64)
            + sigmoid(g_l)[:, None] * rmsnorm(o_lin, w, eps))


# ---------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------


def layer_head(inp: dict, h: int, rows=None) -> dict:
    """The whole layer for one head (optionally for a subset of query rows).

    ``inp`` holds q, k, v, kt, vt, g_s, g_l, rms_w, off, lam, eps,
    block_frames (as produced by vdn_synth.make_inputs).
    """
    bf = inp["block_frames"]
    off = np.asarray(inp["off"], dtype=np.int64)
    N = int(off[-1])
    all_rows = np.arange(N) if rows is None else np.asarray(rows)
    o_soft = softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"],
                                 inp["vt"], off, h, bf, rows=rows)
    st = vda_states_head(inp["k"], inp["v"], inp["kt"], inp["vt"], off, h,
                         inp["lam"], bf)
    frame_of = np.searchsorted(off, all_rows, side="right") - 1
    blk = block_of(frame_of, bf)
    q = np.asarray(inp["q"][all_rows, h], np.float64)
    o_lin = np.einsum("nd,nde->ne", q, st["R"][blk])
    out = gate_merge(o_soft, o_lin, inp["g_s"][all_rows, h],
                     inp["g_l"][all_rows, h], inp["rms_w"][h], inp["eps"])
    return dict(out=out, o_soft=o_soft, o_lin=o_lin, states=st)


def layer(inp: dict) -> dict:
    """The whole layer, all heads. Returns out, o_soft, o_lin [N, H, d],
    S_text [H, d, d], R [nb, H, d, d]."""
    H = inp["H"]
    res = [layer_head(inp, h) for h in range(H)]
    return dict(
        out=np.stack([r["out"] for r in res], axis=1),
        o_soft=np.stack([r["o_soft"] for r in res], axis=1),
        o_lin=np.stack([r["o_lin"] for r in res], axis=1),
        S_text=np.stack([r["states"]["S_text"] for r in res]),
        R=np.stack([r["states"]["R"] for r in res], axis=1),
        states=[r["states"] for r in res],
    )


# ---------------------------------------------------------------------------
# Per-branch output projections
# ---------------------------------------------------------------------------
#
# Each branch carries its own content-dependent sigmoid gate and its own
# output projection, and the projected branches are merged by a sum
# [nav.superapi.store page, Technical Principles, "Gated Fusion Mechanism";
# openi.cn page, "技术原理：局部精确、远程压缩", last paragraph]. With the gate
# logits given per token and per head, the gate is applied per head before
# the projection:
#   y = W_s (sigmoid(g_s) o_soft) + W_l (sigmoid(g_l) RMSNorm(o_lin))
# where o_soft, o_lin are flattened over heads (index h * d + j). Written as
# one matrix: y = w_o @ [a_s ; a_l], w_o = [W_s | W_l] of shape [D, 2 H d].
# With W_s = W_l = I (D = H d) this is the merged layer output above.


def gated_branches_head(inp: dict, h: int, rows=None) -> dict:
    """The two gated branch outputs of one head, before any projection:
    a_s = sigmoid(g_s) o_soft, a_l = sigmoid(g_l) RMSNorm(o_lin)."""
    res = layer_head(inp, h, rows=rows)
    N = int(np.asarray(inp["off"])[-1])
    all_rows = np.arange(N) if rows is None else np.asarray(rows)
    a_s = sigmoid(inp["g_s"][all_rows, h])[:, None] * res["o_soft"]
    a_l = sigmoid(inp["g_l"][all_rows, h])[:, None] * rmsnorm(res["o_lin"], inp["rms_w"][h],
                                                               inp["eps"])
    return dict(a_s=a_s, a_l=a_l, out=res["out"])


def gated_branches(inp: dict, rows=None) -> np.ndarray:
    """[rows, 2, H, d]: branch 0 = a_s, branch 1 = a_l, every head."""
    H = inp["H"]
    parts = [gated_branches_head(inp, h, rows) for h in range(H)]
    a_s = np.stack([p["a_s"] for p in parts], axis=1)
    a_l = np.stack([p["a_l"] for p in parts], axis=1)
    return np.stack([a_s, a_l], axis=1)


def output_projection(branches, w_o) -> np.ndarray:
    """y = [a_s ; a_l] projected by w_o [D, 2 H d]: branches [rows, 2, H, d]."""
    b = np.asarray(branches, np.float64)
    return b.reshape(b.shape[0], -1) @ np.asarray(w_o, np.float64).T


def layer_proj(inp: dict, w_o, rows=None) -> np.ndarray:
    """The layer with per-branch output projections: [rows, D]."""
    return output_projection(gated_branches(inp, rows), w_o)
