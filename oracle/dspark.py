"""fp64 CPU oracle of the DSpark draft round -- TEST INFRASTRUCTURE, not product code.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. It shares no code with the CUDA library:
it reads the same seeded inputs (``synthetic``) and nothing else.

Every function restates one step of the round as the pages define it, in
float64, from the exact input bits (bf16 and fp32 inputs upcast exactly).
Source page: "@mlx-bun/inference 0.0.0-stage -> 1.0.0",
``package/src/models/speculative/deepspec.ts`` (class ``DeepspecDrafter``),
plus "mlx-bun 0.2.0 -> 0.4.0" page 75 for ``plainDeepspecContext`` and
``projectContextKV``. Method names below are the page's.

Readings where the page leaves a step open:
  * RoPE pairs lane i with lane i + hd/2 (rotate-half, the HF
    ``apply_rotary_pos_emb`` convention the page says it was checked against);
    angle = position / wavelength, wavelength = theta^(2k/hd) for
    k < floor(hd * partial)/2 and +inf (identity) beyond.
  * RMSNorm multiplies by the stored gain (not 1 + gain); eps sits inside the root.
  * argmax ties go to the lowest index.
  * the Markov sum U + bias is taken in fp64 (the page rounds it to bf16 only
    to mimic torch's near-tie order).
  * quantized weights are dequantized exactly (scale * code + bias in fp64).
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

__all__ = [
    "OracleWeights", "dequantize_affine4", "rope_wavelengths", "rms_norm", "apply_rope",
    "gelu_tanh", "store_rounded", "project_context", "project_context_kv", "attention_weights", "attend_concat", "attend_split",
    "embed_block", "decoder_layer", "backbone", "compute_logits", "markov_bias", "markov_walk", "teacher_forced_walk",
    "confidence", "prefix_length", "prune_lengths", "draft_rows", "block_ids",
]


def _f64(t) -> np.ndarray:
    """Exact upcast of a torch tensor (bf16 / fp32 / int) or array to float64 NumPy."""
    if isinstance(t, np.ndarray):
        return t.astype(np.float64, copy=False)
    import torch  # local: the oracle itself is NumPy; torch only carries the input bits
    return t.detach().to("cpu").to(torch.float64).numpy()


# ---------------------------------------------------------------------------
# Weights: dense or 4-bit affine (deepspec.ts, ``MatW`` / ``TableW``,
# ``matmulW`` = x @ W^T, ``gatherW`` = row gather then dequantize).
# ---------------------------------------------------------------------------

def dequantize_affine4(words, scales, biases, group: int) -> np.ndarray:
    """Affine 4-bit dequantization (MLX QuantizedLinear / QuantizedEmbedding semantics).

    ``words`` [out, in/8] 32-bit: code j of a word sits in bits 4j..4j+3 and
    is input column 8*word + j. ``scales``/``biases`` [out, in/group].
    Weight = scale * code + bias, in fp64.
    """
    w = np.asarray(words if isinstance(words, np.ndarray) else words.numpy()).astype(np.int64) & 0xFFFFFFFF
    out_f, nw = w.shape
    shifts = np.arange(8, dtype=np.int64) * 4
    codes = (w[:, :, None] >> shifts[None, None, :]) & 0xF          # [out, in/8, 8]
    codes = codes.reshape(out_f, nw * 8).astype(np.float64)
    s = np.repeat(_f64(scales), group, axis=1)
    b = np.repeat(_f64(biases), group, axis=1)
    return s * codes + b


class OracleWeights:
    """Read access to the drafter's weights in fp64 (upcast on demand, never cached whole)."""

    def __init__(self, tensors: Dict[str, object], model):
        self.t = tensors
        self.m = model

    def is_quantized(self, name: str) -> bool:
        return (name + ".q") in self.t

    def rows(self, name: str, lo: int, hi: int) -> np.ndarray:
        if self.is_quantized(name):
            return dequantize_affine4(self.t[name + ".q"][lo:hi], self.t[name + ".scales"][lo:hi],
                                      self.t[name + ".biases"][lo:hi], self.m.quant_group_size)
        return _f64(self.t[name][lo:hi])

    def n_rows(self, name: str) -> int:
        return int(self.t[name + ".q"].shape[0] if self.is_quantized(name) else self.t[name].shape[0])

    def matrix(self, name: str) -> np.ndarray:
        return self.rows(name, 0, self.n_rows(name))

    def vector(self, name: str) -> np.ndarray:
        return _f64(self.t[name]).reshape(-1)

    def linear(self, x: np.ndarray, name: str, chunk: int = 32768) -> np.ndarray:
        """``matmulW``: x @ W^T with W stored [out, in], streamed in row chunks."""
        n = self.n_rows(name)
        out = np.empty(x.shape[:-1] + (n,), dtype=np.float64)
        for lo in range(0, n, chunk):
            hi = min(n, lo + chunk)
            out[..., lo:hi] = x @ self.rows(name, lo, hi).T
        return out

    def gather(self, name: str, ids: np.ndarray) -> np.ndarray:
        """``gatherW``: table rows for ``ids`` (dequantize-on-gather for a quantized table)."""
        ids = np.asarray(ids, dtype=np.int64)
        flat = ids.reshape(-1)
        rows = np.stack([self.rows(name, int(i), int(i) + 1)[0] for i in flat]) if flat.size else \
            np.zeros((0, 0))
        return rows.reshape(ids.shape + (rows.shape[-1],))


# ---------------------------------------------------------------------------
# Elementwise / row primitives.
# ---------------------------------------------------------------------------

def rope_wavelengths(head_dim: int, theta: float, partial: float) -> np.ndarray:
    """Proportional-RoPE wavelengths (``DeepspecDrafter`` constructor, ``ropeFreqs``).

    rotated = floor(head_dim * partial); entry k is theta^(2k/head_dim) for
    k < rotated/2 (exponent over the FULL head_dim) and +inf otherwise, which
    makes the angle 0 and the rotation the identity on those lanes.
    """
    rotated = math.floor(head_dim * partial)
    n = head_dim // 2
    out = np.full(n, np.inf, dtype=np.float64)
    k = 0
    while k < rotated / 2 and k < n:
        out[k] = float(theta) ** (2.0 * k / head_dim)
        k += 1
    return out


def rms_norm(x: np.ndarray, weight: Optional[np.ndarray], eps: float) -> np.ndarray:
    """Gemma4RMSNorm (``#rms``): x / sqrt(mean(x^2) + eps), times the gain when given.

    ``weight=None`` is the scale-less ``v_norm``. Normalises the last axis.
    """
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + eps)
    return y if weight is None else y * weight


def apply_rope(x: np.ndarray, positions: np.ndarray, wavelengths: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE at absolute ``positions``.

    ``x`` [..., T, hd] (any leading axes), ``positions`` broadcastable to
    [..., T]. For i < hd/2 with angle a = p / wavelength[i]:
    x'[i] = x[i] cos a - x[i+hd/2] sin a;  x'[i+hd/2] = x[i+hd/2] cos a + x[i] sin a.
    """
    hd = x.shape[-1]
    half = hd // 2
    p = np.asarray(positions, dtype=np.float64)[..., None]          # [..., T, 1]
    ang = p / wavelengths                                            # inf wavelength -> 0
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """gelu_pytorch_tanh: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def _sigmoid(z: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-z))


# ---------------------------------------------------------------------------
# Stage 1: context K/V (``#projectContextKVRows``).
# ---------------------------------------------------------------------------

def store_rounded(x: np.ndarray, store_dtype: Optional[str]) -> np.ndarray:
    """Round to the cache's storage type (round to nearest even): cached K/V rows
    hold values of that type, which every later round reads. The drafter keeps
    ContextKV rows in the model dtype (``#rms`` casts back to it): "bf16" for its
    bf16 models; "fp16" is the two-byte type with an 11-bit significand.
    None / "fp32" / "fp64" keep the fp64 values."""
    if store_dtype == "fp16":
        return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)
    if store_dtype != "bf16":
        return x
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to(torch.float64).numpy()


def project_context(fc, hidden_norm, target_hiddens, eps: float) -> np.ndarray:
    """``#projectContext``: the context hidden the K/V projection reads, from the
    target model's tap hiddens (``extract_context_feature`` concatenates them over
    the taps, in ``target_layer_ids`` order, then ``hidden_norm(fc(.))``).

    ``target_hiddens`` [..., taps * H]; ``fc`` [H, taps * H] stored [out, in]
    (``matmulW``: x @ fc^T); ``hidden_norm`` [H], the gain of a Gemma4RMSNorm
    over the last axis with the config's eps. Returns [..., H] in fp64.
    """
    x = _f64(target_hiddens)
    proj = x @ _f64(fc).T
    return rms_norm(proj, _f64(hidden_norm).reshape(-1), eps)


def project_context_kv(W: OracleWeights, hidden, pos0: Sequence[int], lengths: Optional[Sequence[int]] = None,
                       chunk: int = 8192, store_dtype: Optional[str] = None) -> List[List[tuple]]:
    """Per-layer context K/V of every row, ready to cache across rounds.

    For each layer: k_raw = hidden @ Wk^T viewed [L, nKv, hd];
    v = rms(k_raw, none) (attention_k_eq_v: v is k before the norms diverge,
    and gets no rope); k = rope(rms(k_raw, k_norm), pos0 + t).
    ``store_dtype="bf16"`` returns the values the cache holds for a bf16
    model (fp64 values rounded to bf16); the default keeps fp64.
    Returns ``out[b][layer] = (k [L_b, nKv, hd], v [L_b, nKv, hd])``.
    """
    m = W.m
    nKv, hd = m.num_global_key_value_heads, m.global_head_dim
    wl = rope_wavelengths(hd, m.rope_theta, m.partial_rotary_factor)
    B = len(pos0)
    out = []
    for b in range(B):
        L = int(lengths[b]) if lengths is not None else int(hidden.shape[1])
        per_layer = []
        for li in range(m.num_hidden_layers):
            kn = W.vector(f"layers.{li}.k_norm")
            ks, vs = [], []
            for lo in range(0, L, chunk):
                hi = min(L, lo + chunk)
                x = _f64(hidden[b, lo:hi])
                k_raw = W.linear(x, f"layers.{li}.k_proj").reshape(hi - lo, nKv, hd)
                v = rms_norm(k_raw, None, m.rms_norm_eps)
                k = rms_norm(k_raw, kn, m.rms_norm_eps)
                pos = int(pos0[b]) + np.arange(lo, hi)
                k = apply_rope(k.transpose(1, 0, 2), pos[None, :], wl).transpose(1, 0, 2)
                ks.append(store_rounded(k, store_dtype))
                vs.append(store_rounded(v, store_dtype))
            per_layer.append((np.concatenate(ks, 0) if ks else np.zeros((0, nKv, hd)),
                              np.concatenate(vs, 0) if vs else np.zeros((0, nKv, hd))))
        out.append(per_layer)
    return out


# ---------------------------------------------------------------------------
# Stage 2: KV-injection attention (``DeepspecContextAttention.attend`` and
# its reference form ``plainDeepspecContext``: concat along the sequence,
# then non-causal SDPA at scale 1.0).
# ---------------------------------------------------------------------------

def _gqa_keys(k: np.ndarray, n_heads: int) -> np.ndarray:
    """[T, nKv, hd] -> [nH, T, hd]: query head h reads kv head h // (nH / nKv)."""
    grp = n_heads // k.shape[1]
    return np.repeat(k.transpose(1, 0, 2), grp, axis=0)


def attention_weights(q: np.ndarray, k_ctx, k_blk) -> np.ndarray:
    """Softmax weights [nH, G, Lctx + G] of one row (scale 1.0, no mask)."""
    nH = q.shape[1]
    K = _gqa_keys(np.concatenate([k_ctx, k_blk], axis=0), nH)        # [nH, T, hd]
    s = np.einsum("gnd,ntd->ngt", q, K)                              # [nH, G, T]
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=-1, keepdims=True)


def attend_concat(q: np.ndarray, k_ctx, v_ctx, k_blk, v_blk) -> np.ndarray:
    """``plainDeepspecContext.attend`` for one row.

    q [G, nH, hd] (block queries), k_ctx/v_ctx [Lctx, nKv, hd], k_blk/v_blk
    [G, nKv, hd]. Keys and values are the context rows followed by the block
    rows; every query sees every key. Returns [G, nH, hd].
    """
    nH = q.shape[1]
    P = attention_weights(q, k_ctx, k_blk)
    V = _gqa_keys(np.concatenate([v_ctx, v_blk], axis=0), nH)        # [nH, T, hd]
    return np.einsum("ngt,ntd->gnd", P, V)


def attend_split(q: np.ndarray, k_ctx, v_ctx, k_blk, v_blk, n_splits: int = 3) -> np.ndarray:
    """The storage-side form of ``attend``: context keys in ``n_splits`` chunks plus
    the block keys as one more part, each reduced to (max, sum, weighted values)
    and merged by the online-softmax rule. Equal to ``attend_concat`` in exact
    arithmetic; kept as a self-check of the merge the CUDA path uses."""
    nH = q.shape[1]
    L = k_ctx.shape[0]
    bounds = np.linspace(0, L, n_splits + 1).astype(int) if L > 0 else np.array([0, 0])
    parts = [(k_ctx[a:b], v_ctx[a:b]) for a, b in zip(bounds[:-1], bounds[1:]) if b > a]
    parts.append((k_blk, v_blk))
    m_all, l_all, o_all = [], [], []
    for kk, vv in parts:
        K = _gqa_keys(kk, nH)
        V = _gqa_keys(vv, nH)
        s = np.einsum("gnd,ntd->ngt", q, K)
        mx = s.max(axis=-1)
        p = np.exp(s - mx[..., None])
        m_all.append(mx)
        l_all.append(p.sum(axis=-1))
        o_all.append(np.einsum("ngt,ntd->ngd", p, V))
    M = np.max(np.stack(m_all), axis=0)
    num = sum(np.exp(mi - M)[..., None] * oi for mi, oi in zip(m_all, o_all))
    den = sum(np.exp(mi - M) * li for mi, li in zip(m_all, l_all))
    return (num / den[..., None]).transpose(1, 0, 2)


# ---------------------------------------------------------------------------
# Backbone (``#forwardBackbone``), logits (``#computeLogits``).
# ---------------------------------------------------------------------------

def block_ids(anchors: Sequence[int], gamma: int, mask_token_id: int) -> np.ndarray:
    """[A, gamma] = [anchor, MASK x (gamma - 1)] per row (``draftRows``)."""
    a = np.asarray(anchors, dtype=np.int64)
    ids = np.full((a.shape[0], gamma), mask_token_id, dtype=np.int64)
    ids[:, 0] = a
    return ids


def embed_block(W: OracleWeights, anchors: Sequence[int]) -> np.ndarray:
    """Block embedding [A, G, H]: embed([anchor, MASK x (G-1)]) * sqrt(hidden)
    (Gemma4TextScaledWordEmbedding; dequantize-on-gather for a quantized table)."""
    m = W.m
    ids = block_ids(anchors, m.block_size, m.mask_token_id)
    return W.gather("embed_tokens", ids) * math.sqrt(m.hidden_size)


def decoder_layer(W: OracleWeights, li: int, h: np.ndarray, ctx_kv_layer: List[tuple],
                  block_pos: Sequence[int]):
    """One DSpark decoder layer over the noise blocks of A rows (``#forwardBackbone`` loop body).

    h [A, G, H]; ``ctx_kv_layer[b] = (k, v)`` are row b's cached context rows of
    this layer. x = rms(h, input_layernorm); q = rope(rms(x Wq^T, q_norm));
    k_raw = x Wk^T; v_blk = rms(k_raw); k_blk = rope(rms(k_raw, k_norm)); the
    block positions are block_pos + t. Attention over context ++ block; o_proj;
    post-attention norm; residual add; pre-ff norm; gelu-tanh MLP; post-ff norm;
    residual add; the sum times layer_scalar. Returns (h_out, attention output
    [A, G, nH, hd]).
    """
    m = W.m
    A, G, _ = h.shape
    nH, nKv, hd = m.num_attention_heads, m.num_global_key_value_heads, m.global_head_dim
    eps = m.rms_norm_eps
    wl = rope_wavelengths(hd, m.rope_theta, m.partial_rotary_factor)
    pos = np.asarray(block_pos, dtype=np.float64)[:, None] + np.arange(G)[None, :]   # [A, G]
    p = f"layers.{li}."
    residual = h
    x = rms_norm(h, W.vector(p + "input_layernorm"), eps)
    q = W.linear(x, p + "q_proj").reshape(A, G, nH, hd)
    q = rms_norm(q, W.vector(p + "q_norm"), eps)
    q = apply_rope(q.transpose(0, 2, 1, 3), pos[:, None, :], wl).transpose(0, 2, 1, 3)
    k_raw = W.linear(x, p + "k_proj").reshape(A, G, nKv, hd)
    v_blk = rms_norm(k_raw, None, eps)
    k_blk = rms_norm(k_raw, W.vector(p + "k_norm"), eps)
    k_blk = apply_rope(k_blk.transpose(0, 2, 1, 3), pos[:, None, :], wl).transpose(0, 2, 1, 3)
    o = np.stack([attend_concat(q[b], ctx_kv_layer[b][0], ctx_kv_layer[b][1], k_blk[b], v_blk[b])
                  for b in range(A)])                                  # [A, G, nH, hd]
    a = W.linear(o.reshape(A, G, nH * hd), p + "o_proj")
    a = rms_norm(a, W.vector(p + "post_attention_layernorm"), eps)
    h = residual + a
    f = rms_norm(h, W.vector(p + "pre_feedforward_layernorm"), eps)
    mlp = W.linear(gelu_tanh(W.linear(f, p + "gate_proj")) * W.linear(f, p + "up_proj"), p + "down_proj")
    mlp = rms_norm(mlp, W.vector(p + "post_feedforward_layernorm"), eps)
    h = (h + mlp) * W.vector(p + "layer_scalar")[0]
    return h, o


def backbone(W: OracleWeights, ctx_kv: List[List[tuple]], anchors: Sequence[int], block_pos: Sequence[int],
             attn_out: Optional[list] = None) -> np.ndarray:
    """One backbone pass over the noise blocks of A rows -> final-normed hidden [A, G, H].

    ``ctx_kv[b][layer] = (k, v)``. ``attn_out`` (if a list) receives each
    layer's attention output [A, G, nH, hd].
    """
    m = W.m
    h = embed_block(W, anchors)
    for li in range(m.num_hidden_layers):
        h, o = decoder_layer(W, li, h, [ctx_kv[b][li] for b in range(len(anchors))], block_pos)
        if attn_out is not None:
            attn_out.append(o)
    return rms_norm(h, W.vector("norm"), m.rms_norm_eps)


def compute_logits(W: OracleWeights, h_final: np.ndarray) -> np.ndarray:
    """lm_head(h), then cap * tanh(logits / cap) when final_logit_softcapping is set."""
    logits = W.linear(h_final, "lm_head")
    cap = W.m.final_logit_softcapping
    if cap:
        logits = cap * np.tanh(logits / cap)
    return logits


# ---------------------------------------------------------------------------
# Stage 3: the Markov walk (``#markovStepBias`` / ``#selectStep``), the
# confidence head (``#confidence``) and truncation (``_confident_prefix_length``).
# ---------------------------------------------------------------------------

def markov_bias(W: OracleWeights, prev: Sequence[int]) -> np.ndarray:
    """VanillaMarkov step bias [A, V] = markov_w2(markov_w1[prev]) = w1[prev] @ W2^T."""
    e = W.gather("markov_w1", np.asarray(prev, dtype=np.int64))       # [A, r]
    return W.linear(e, "markov_w2")


def _top2(row: np.ndarray):
    i = int(np.argmax(row))                                          # first maximum
    best = row[i]
    rest = np.delete(row, i)
    return i, float(best - rest.max()) if rest.size else math.inf


def markov_walk(W: OracleWeights, U: np.ndarray, anchors: Sequence[int]) -> np.ndarray:
    """Temperature-0 sequential walk: prev = anchor; tok_k = argmax(U[:, k] + bias(prev)).

    With markov_rank == 0 the bias is absent and each step is a plain argmax.
    Returns tokens [A, G] int64.
    """
    tokens, _ = teacher_forced_walk(W, U, anchors, None)
    return tokens


def teacher_forced_walk(W: OracleWeights, U: np.ndarray, anchors: Sequence[int],
                        forced: Optional[np.ndarray]):
    """The walk, optionally feeding ``forced[:, k-1]`` (e.g. another implementation's
    tokens) as the previous token of step k instead of the walk's own choice.

    Returns (tokens [A, G], margins [A, G]) where margins are top-1 minus
    top-2 of the step's corrected logits.
    """
    A, G, _ = U.shape
    prev = np.asarray(anchors, dtype=np.int64).copy()
    toks = np.zeros((A, G), dtype=np.int64)
    margins = np.zeros((A, G), dtype=np.float64)
    for k in range(G):
        step = U[:, k, :]
        if W.m.markov_rank > 0:
            step = step + markov_bias(W, prev)
        for b in range(A):
            toks[b, k], margins[b, k] = _top2(step[b])
        prev = toks[:, k].copy() if forced is None else np.asarray(forced[:, k], dtype=np.int64).copy()
    return toks, margins


def confidence(W: OracleWeights, h_final: np.ndarray, anchors: Sequence[int], tokens: np.ndarray) -> np.ndarray:
    """c[b, k] = sigmoid(proj([h_final[b, k] ; markov_w1[prev_k]]) + bias), prev_0 = anchor,
    prev_k = tokens[b, k-1]; without ``confidence_head_with_markov`` the feature is h alone."""
    A, G, H = h_final.shape
    prev = np.concatenate([np.asarray(anchors, dtype=np.int64)[:, None], tokens[:, :-1]], axis=1)
    feat = h_final
    if W.m.confidence_head_with_markov:
        feat = np.concatenate([h_final, W.gather("markov_w1", prev)], axis=-1)
    z = W.linear(feat, "confidence_proj")[..., 0] + W.vector("confidence_bias")[0]
    return _sigmoid(z)


def prefix_length(conf_row: Sequence[float], threshold: float, gamma: int) -> int:
    """_confident_prefix_length: gamma if threshold <= 0; else the first index whose
    confidence is below the threshold (0 is an empty proposal), or gamma if none."""
    if threshold <= 0:
        return gamma
    for k, c in enumerate(conf_row):
        if c < threshold:
            return k
    return gamma


def prune_lengths(conf: np.ndarray, thresholds: Sequence[float]) -> np.ndarray:
    """Confidence-scheduled draft-length pruning (Alg 1, the DFlash generator's
    ``forwardInfer``, "@mlx-bun/inference 0.0.0-stage -> 1.0.0"): row b keeps
    positions [0, k) where k is the first position >= 1 whose confidence is
    below that position's threshold, else the whole block; position 0 always
    survives. ``conf`` [A, gamma]; ``thresholds`` [gamma] (entry 0 unused).
    A NaN confidence is not below any threshold.
    """
    conf = np.asarray(conf, dtype=np.float64)
    A, gamma = conf.shape
    out = np.full(A, gamma, dtype=np.int64)
    for b in range(A):
        for k in range(1, gamma):
            if conf[b, k] < float(thresholds[k]):
                out[b] = k
                break
    return out


def draft_rows(W: OracleWeights, ctx_kv: List[List[tuple]], anchors: Sequence[int], block_pos: Sequence[int],
               keep_attention: bool = False) -> Dict[str, np.ndarray]:
    """One whole round (``draftRows``): backbone, logits, walk, confidence, lengths."""
    m = W.m
    attn = [] if keep_attention else None
    h = backbone(W, ctx_kv, anchors, block_pos, attn_out=attn)
    U = compute_logits(W, h)
    toks, margins = teacher_forced_walk(W, U, anchors, None)
    out = {"hidden": h, "base_logits": U, "tokens": toks, "margins": margins}
    if m.enable_confidence_head:
        conf = confidence(W, h, anchors, toks)
        out["conf"] = conf
        out["lengths"] = np.array([prefix_length(conf[b], m.confidence_threshold, m.block_size)
                                   for b in range(len(anchors))], dtype=np.int64)
    else:
        out["lengths"] = np.full(len(anchors), m.block_size, dtype=np.int64)
    if attn is not None:
        out["attention"] = attn
    return out
