"""Seeded synthetic workloads for the DSpark draft round.

This module is the one place both sides of every parity check get their
inputs from: the fp64 oracle (``oracle/``) and the CUDA library
(``block_draft_model_dspark_b200``). It holds model shapes, seeded random
draws and the storage formats the pages name (bf16 tensors, and 4-bit affine
packing for the quantized workload). It holds none of the round's arithmetic.

Shapes follow the five workloads of the DSpark draft round (deepspec.ts,
``DeepspecConfig`` field names, kept verbatim). Every tensor is drawn on the
CPU with its own ``torch.Generator`` seeded from (workload seed, tensor index),
in fp32, then rounded to nearest-even bf16 for the bf16 workloads, so the
bits do not depend on the device that later holds them.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import torch

__all__ = [
    "ModelShape", "Workload", "WORKLOADS", "workload", "make_weights",
    "make_round_inputs", "round_meta", "make_append_schedule", "quantize_affine4", "weight_names",
    "QUANTIZED_MATRICES", "make_context_projection", "make_target_hiddens",
]


@dataclasses.dataclass(frozen=True)
class ModelShape:
    """The drafter's config.json keys (deepspec.ts, ``DeepspecConfig``)."""
    hidden_size: int
    num_hidden_layers: int
    num_attention_heads: int
    global_head_dim: int
    num_global_key_value_heads: int
    intermediate_size: int
    vocab_size: int
    block_size: int
    mask_token_id: int
    markov_rank: int
    rope_theta: float = 1e6            # readConfig default
    partial_rotary_factor: float = 1.0  # readConfig default
    rms_norm_eps: float = 1e-6          # readConfig default
    final_logit_softcapping: Optional[float] = None
    enable_confidence_head: bool = True
    confidence_head_with_markov: bool = True
    confidence_threshold: float = 0.0
    attention_k_eq_v: bool = True
    markov_head_type: str = "vanilla"
    hidden_activation: str = "gelu_pytorch_tanh"
    dtype: str = "bf16"                 # storage/activation dtype: "fp32" or "bf16"
    quant_bits: int = 0                 # 0 = dense weights, 4 = affine 4-bit
    quant_group_size: int = 64

    def replace(self, **kw) -> "ModelShape":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    model: ModelShape
    rows: int                 # A (request rows in one round)
    ctx_len: int              # fixed context length (or the upper end when ragged)
    seed: int
    ragged_min: int = 0       # >0: per-row context length ~ U[ragged_min, ctx_len]
    start_max: int = 0        # >0: per-row start position ~ U[0, start_max)
    append_rounds: int = 0    # >0: rounds of append(n ~ U[1, append_max]) + draft
    append_max: int = 0

    @property
    def capacity(self) -> int:
        return self.ctx_len + self.append_rounds * self.append_max


_GEMMA_LIKE = dict(
    hidden_size=3840, num_hidden_layers=4, num_attention_heads=16, global_head_dim=256,
    num_global_key_value_heads=2, intermediate_size=15360, vocab_size=262144,
    markov_rank=64, mask_token_id=262143, final_logit_softcapping=30.0,
)

WORKLOADS: Dict[str, Workload] = {
    # 1 layer, hidden 256, 4x64 heads, 1 kv head, vocab 1024, rank 8, gamma 4, fp32.
    "tiny_fp32": Workload(
        "tiny_fp32",
        ModelShape(hidden_size=256, num_hidden_layers=1, num_attention_heads=4, global_head_dim=64,
                   num_global_key_value_heads=1, intermediate_size=512, vocab_size=1024,
                   block_size=4, mask_token_id=1023, markov_rank=8, rope_theta=10000.0,
                   partial_rotary_factor=0.25, rms_norm_eps=1e-6, final_logit_softcapping=None,
                   dtype="fp32"),
        rows=1, ctx_len=32, seed=0),
    # Single request: 4 layers, hidden 3840, 16x256 heads, 2 kv heads, vocab 262144, gamma 16.
    "single_bf16": Workload("single_bf16", ModelShape(block_size=16, **_GEMMA_LIKE),
                            rows=1, ctx_len=4096, seed=1),
    # 32 rows, per-row context in [512, 4096], per-row start position in [0, 8192).
    "ragged_bf16": Workload("ragged_bf16", ModelShape(block_size=16, **_GEMMA_LIKE),
                            rows=32, ctx_len=4096, seed=2, ragged_min=512, start_max=8192),
    # 4 rows x 32768 context, then 8 rounds of append(U[1,16]) + draft.
    "long_incremental_bf16": Workload("long_incremental_bf16", ModelShape(block_size=16, **_GEMMA_LIKE),
                                      rows=4, ctx_len=32768, seed=3, append_rounds=8, append_max=16),
    # Every matmul weight and the embedding / lm-head tables as 4-bit affine, g=64.
    "quant4_bf16": Workload("quant4_bf16", ModelShape(block_size=8, quant_bits=4, quant_group_size=64,
                                                      **_GEMMA_LIKE),
                            rows=64, ctx_len=8192, seed=4),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


# Matrices stored as 4-bit affine in the quantized workload: every 2-D matmul
# weight plus the embedding table (markov_w1 stays dense).
QUANTIZED_MATRICES = ("q_proj", "k_proj", "o_proj", "gate_proj", "up_proj", "down_proj",
                      "lm_head", "embed_tokens", "markov_w2", "confidence_proj")


def _matrix_kind(name: str) -> str:
    return name.split(".")[-1]


def weight_names(m: ModelShape) -> List[tuple]:
    """(name, shape, kind) in draw order; kind is 'mat', 'gain' or 'scalar'.

    Order follows the drafter's constructor: embedding, final norm, lm-head,
    per-layer attention / norms / MLP / layer scalar, Markov head, confidence head.
    """
    H, V, r = m.hidden_size, m.vocab_size, m.markov_rank
    nH, nKv, hd, I = m.num_attention_heads, m.num_global_key_value_heads, m.global_head_dim, m.intermediate_size
    out = [("embed_tokens", (V, H), "mat"), ("norm", (H,), "gain"), ("lm_head", (V, H), "mat")]
    for i in range(m.num_hidden_layers):
        p = f"layers.{i}."
        out += [
            (p + "q_proj", (nH * hd, H), "mat"), (p + "k_proj", (nKv * hd, H), "mat"),
            (p + "o_proj", (H, nH * hd), "mat"),
            (p + "q_norm", (hd,), "gain"), (p + "k_norm", (hd,), "gain"),
            (p + "input_layernorm", (H,), "gain"), (p + "post_attention_layernorm", (H,), "gain"),
            (p + "pre_feedforward_layernorm", (H,), "gain"), (p + "post_feedforward_layernorm", (H,), "gain"),
            (p + "gate_proj", (I, H), "mat"), (p + "up_proj", (I, H), "mat"), (p + "down_proj", (H, I), "mat"),
            (p + "layer_scalar", (1,), "scalar"),
        ]
    if r > 0:
        out += [("markov_w1", (V, r), "mat"), ("markov_w2", (V, r), "mat")]
    if m.enable_confidence_head:
        conf_in = H + (r if m.confidence_head_with_markov else 0)
        out += [("confidence_proj", (1, conf_in), "mat"), ("confidence_bias", (1,), "bias")]
    return out


def _draw(seed: int, index: int, shape, std: float = 1.0, mean: float = 0.0) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed((seed + 1) * 1_000_003 + index * 7919)
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t


def _store(t: torch.Tensor, dtype: str) -> torch.Tensor:
    return t.to(torch.bfloat16) if dtype == "bf16" else t.contiguous()


def quantize_affine4(w: torch.Tensor, group: int = 64):
    """Pack an fp32 [out, in] matrix as 4-bit affine codes (a fixture, not the method).

    Storage format (MLX QuantizedLinear affine layout): eight 4-bit codes per
    32-bit word along the input dimension, code j of a word in bits 4j..4j+3,
    plus bf16 ``scales`` and ``biases`` of shape [out, in/group]; a weight
    reads back as ``scale * code + bias``. Scales and biases are rounded to
    bf16 first and the codes are chosen against the rounded values.
    Returns (packed int32 [out, in/8], scales bf16, biases bf16).
    """
    out_f, in_f = w.shape
    assert in_f % group == 0 and group % 8 == 0
    g = w.reshape(out_f, in_f // group, group).to(torch.float32)
    lo = g.amin(dim=-1)
    hi = g.amax(dim=-1)
    scale = ((hi - lo) / 15.0).clamp_min(1e-8).to(torch.bfloat16)
    bias = lo.to(torch.bfloat16)
    codes = torch.round((g - bias.float().unsqueeze(-1)) / scale.float().unsqueeze(-1)).clamp_(0, 15)
    codes = codes.to(torch.int64).reshape(out_f, in_f // 8, 8)
    shifts = torch.arange(8, dtype=torch.int64) * 4
    words = (codes << shifts).sum(dim=-1)                     # < 2**32
    words = torch.where(words >= 2 ** 31, words - 2 ** 32, words).to(torch.int32)
    return words.contiguous(), scale.contiguous(), bias.contiguous()


def make_weights(m: ModelShape, seed: int, literal: bool = False, unit_attention_logits: bool = True,
                 markov_scale: float = 1.0) -> Dict[str, torch.Tensor]:
    """Seeded synthetic drafter weights on the CPU.

    Matmul, embedding, Markov and confidence weights are N(0, 0.02); RMSNorm
    gains are 1 + N(0, 0.02) and layer_scalar is 1.0. The q_norm and k_norm
    gains are further scaled by head_dim^(-1/4) (``unit_attention_logits``):
    attention runs at scale 1.0 on QK-normed vectors, so gains of 1 give
    logits of standard deviation sqrt(head_dim) and a near one-hot softmax
    whose output, from the second layer on, hinges on the last bits of the
    stored keys; the scaled gains give unit-variance logits, the temperature a
    trained model has. ``literal=True`` instead draws every gain and the
    layer scalar as N(0, 0.02). ``markov_scale`` multiplies both Markov
    tables (a test knob that makes the transition bias matter). For
    ``quant_bits == 4`` each quantized matrix ``X`` is stored as ``X.q``
    (int32 words), ``X.scales``, ``X.biases`` instead of ``X``.
    """
    out: Dict[str, torch.Tensor] = {}
    qk_scale = m.global_head_dim ** -0.25 if unit_attention_logits else 1.0
    for idx, (name, shape, kind) in enumerate(weight_names(m)):
        if kind == "mat":
            t = _draw(seed, idx, shape, std=0.02)
            if name.startswith("markov_w") and markov_scale != 1.0:
                t.mul_(markov_scale)
        elif kind == "gain":
            t = _draw(seed, idx, shape, std=0.02) if literal else _draw(seed, idx, shape, std=0.02, mean=1.0)
            if not literal and name.endswith(("q_norm", "k_norm")):
                t.mul_(qk_scale)
        elif kind == "scalar":
            t = _draw(seed, idx, shape, std=0.02) if literal else torch.ones(shape)
        else:  # bias
            t = _draw(seed, idx, shape, std=0.02)
        if m.quant_bits == 4 and _matrix_kind(name) in QUANTIZED_MATRICES:
            q, s, b = quantize_affine4(t, m.quant_group_size)
            out[name + ".q"], out[name + ".scales"], out[name + ".biases"] = q, s, b
        else:
            out[name] = _store(t, m.dtype)
    return out


def round_meta(w: Workload):
    """Per-row context lengths, start positions and anchors of a round
    (int64 CPU tensors [A]); the first draws of make_round_inputs."""
    m = w.model
    A = w.rows
    g = torch.Generator(device="cpu")
    g.manual_seed((w.seed + 1) * 104_729 + 17)
    if w.ragged_min > 0:
        lens = torch.randint(w.ragged_min, w.ctx_len + 1, (A,), generator=g, dtype=torch.int64)
    else:
        lens = torch.full((A,), w.ctx_len, dtype=torch.int64)
    if w.start_max > 0:
        pos0 = torch.randint(0, w.start_max, (A,), generator=g, dtype=torch.int64)
    else:
        pos0 = torch.zeros(A, dtype=torch.int64)
    anchors = torch.randint(0, m.vocab_size - 1, (A,), generator=g, dtype=torch.int64)
    return lens, pos0, anchors


def make_round_inputs(w: Workload, rows: Optional[List[int]] = None) -> Dict[str, torch.Tensor]:
    """Context hiddens, positions, lengths and anchors of one draft round.

    Returns CPU tensors: ``hidden`` [A, Lmax, H] (rows past a row's length are
    padding drawn like the rest), ``ctx_len`` [A] int32, ``pos0`` [A] int32
    (absolute position of context row 0), ``block_pos`` [A] int32 (= pos0 +
    ctx_len: the block follows the context), ``anchors`` [A] int32 uniform in
    [0, V-1). ``rows`` selects a subset of the A rows (same values as in the
    full draw), for checking sampled rows of a large workload.
    """
    m = w.model
    A = w.rows
    lens, pos0, anchors = round_meta(w)
    sel = list(range(A)) if rows is None else list(rows)
    Lmax = int(lens[sel].max()) if w.ragged_min > 0 else w.ctx_len
    hid = []
    for b in sel:
        hid.append(_store(_draw(w.seed, 100_000 + b, (Lmax, m.hidden_size)), m.dtype))
    hidden = torch.stack(hid, dim=0).contiguous()
    lens_s, pos0_s, anc_s = lens[sel], pos0[sel], anchors[sel]
    return {
        "hidden": hidden,
        "ctx_len": lens_s.to(torch.int32),
        "pos0": pos0_s.to(torch.int32),
        "block_pos": (pos0_s + lens_s).to(torch.int32),
        "anchors": anc_s.to(torch.int32),
    }


def make_append_schedule(w: Workload, rows: Optional[List[int]] = None) -> List[Dict[str, torch.Tensor]]:
    """Per-round appends of the incremental workload.

    Each round r: ``n_new`` [A] int32 ~ U[1, append_max] drawn per row,
    ``hidden`` [A, append_max, H] fresh N(0,1) rows (entries past n_new are
    padding), and ``anchors`` [A] int32 for the draft that follows.
    """
    m = w.model
    A = w.rows
    sel = list(range(A)) if rows is None else list(rows)
    out = []
    for r in range(w.append_rounds):
        g = torch.Generator(device="cpu")
        g.manual_seed((w.seed + 1) * 15_485_863 + r * 31)
        n_new = torch.randint(1, w.append_max + 1, (A,), generator=g, dtype=torch.int64)
        anchors = torch.randint(0, m.vocab_size - 1, (A,), generator=g, dtype=torch.int64)
        hid = [_store(_draw(w.seed, 200_000 + r * 4096 + b, (w.append_max, m.hidden_size)), m.dtype)
               for b in sel]
        out.append({"n_new": n_new[sel].to(torch.int32), "anchors": anchors[sel].to(torch.int32),
                    "hidden": torch.stack(hid).contiguous()})
    return out


def scaled_down(w: Workload, **model_kw) -> Workload:
    """A copy of a workload with a smaller model (test sizes); shape keys as in ModelShape."""
    return dataclasses.replace(w, model=w.model.replace(**model_kw))


def small_model(dtype: str = "bf16", quant_bits: int = 0, **kw) -> ModelShape:
    """A small Gemma-like drafter used by the fast parity tests (several tiles, ragged tails)."""
    base = dict(hidden_size=512, num_hidden_layers=2, num_attention_heads=8, global_head_dim=128,
                num_global_key_value_heads=2, intermediate_size=1024, vocab_size=4096 + 64,
                block_size=8, mask_token_id=4096 + 63, markov_rank=64 if quant_bits else 16, rope_theta=1e6,
                partial_rotary_factor=0.5, final_logit_softcapping=30.0, dtype=dtype,
                quant_bits=quant_bits)
    base.update(kw)
    return ModelShape(**base)


def make_context_projection(m: ModelShape, taps: int, seed: int) -> Dict[str, torch.Tensor]:
    """Seeded weights of the context feature projection (deepspec.ts ``#projectContext``):
    ``fc`` [hidden, taps * hidden] N(0, 0.02) and ``hidden_norm`` [hidden] 1 + N(0, 0.02), in the
    model's dtype (dense: the projection's GEMM reads them as stored)."""
    H = m.hidden_size
    fc = _draw(seed, 10_001, (H, taps * H), std=0.02)
    g = _draw(seed, 10_002, (H,), std=0.02, mean=1.0)
    return {"fc": _store(fc, m.dtype), "hidden_norm": _store(g, m.dtype)}


def make_target_hiddens(m: ModelShape, taps: int, B: int, L: int, seed: int) -> torch.Tensor:
    """The target model's tap hiddens for B rows of L context positions, concatenated over the
    taps: [B, L, taps * hidden], N(0, 1) in the model's dtype."""
    return _store(_draw(seed, 10_003, (B, L, taps * m.hidden_size)), m.dtype)
