"""The round at unit q_norm / k_norm gains (the literal 1 + N(0, 0.02) gains, without the
head_dim^-1/4 scaling the other workloads' synthetic weights use).

Attention runs at scale 1.0 on QK-normed vectors, so unit gains give attention logits of
standard deviation sqrt(head_dim) (16 at head_dim 256) and a near one-hot softmax; from the
second layer on, the output depends on the last bits of the stored keys, and no finite-precision
implementation holds the logits to a fixed tolerance against the fp64 oracle. What such a model
still pins: the K/V cache rows element by element (no attention involved); the first layer's
attention output (its inputs are exact embeddings through one GEMM) with at least 99% of its
elements within the bf16 bar and none far outside (q enters the tensor cores in fp16, and the
near one-hot softmax turns its ~5e-3 logit error into occasional ~0.02 output errors); and the
tokens wherever the oracle's top-1 / top-2 margin is larger than the logit error this
conditioning allows."""
import numpy as np
import pytest
import torch

from oracle import dspark as O
from synthetic import WORKLOADS, make_round_inputs, small_model
from parity_util import as_stored, assert_close, build, check_tokens, ensure_built

pytestmark = pytest.mark.gpu

# Token margin at unit gains: the largest logit error a bf16 K/V cache allows at this
# conditioning (a CPU emulation of bf16 storage against the fp64 oracle finds ~0.1 at the
# single-request size) with a 2.5x allowance.
UNSCALED_MARGIN = 0.25


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    ensure_built()


def _round(model, W, m, hid, lens, pos0, anchors):
    import block_draft_model_dspark_b200 as dsp
    A = len(lens)
    cache = dsp.KvCache(model, A, int(hid.shape[1]))
    cache.set_lengths([0] * A)
    model.dspark_append_context_kv(cache, hid.cuda(), [int(x) for x in lens],
                                   torch.tensor(pos0, dtype=torch.int32, device="cuda"))
    block_pos = [p + L for p, L in zip(pos0, lens)]
    dump = torch.empty((m.num_hidden_layers, A, m.block_size, m.num_attention_heads, m.global_head_dim),
                       dtype=torch.float32, device="cuda")
    model.dspark_debug_attention_dump(dump)
    try:
        out = model.draft(cache, torch.tensor(anchors, dtype=torch.int32, device="cuda"),
                          torch.tensor(block_pos, dtype=torch.int32, device="cuda"), max(lens))
        torch.cuda.synchronize()
    finally:
        model.dspark_debug_attention_dump(None)
    assert model.dspark_read_device_status() == 0
    return cache, out, dump, block_pos


def _check(name, m, W, cache, kv, out, dump, anchors, block_pos, lens, rows_to_check=None):
    k = cache.k.float().cpu().numpy()
    v = cache.v.float().cpu().numpy()
    for b, L in enumerate(lens):
        idx = np.arange(L) if rows_to_check is None else rows_to_check
        for l in range(m.num_hidden_layers):
            assert_close(k[l, b, idx], kv[b][l][0][idx], "bf16", f"{name}: K layer {l} row {b}")
            assert_close(v[l, b, idx], kv[b][l][1][idx], "bf16", f"{name}: V layer {l} row {b}")
    ref = O.draft_rows(W, as_stored(kv, "bf16"), anchors, block_pos, keep_attention=True)
    a0 = dump[0].cpu().numpy()
    w0 = ref["attention"][0]
    aerr = np.abs(a0 - w0)
    outside = aerr > 1e-2 + 2e-2 * np.abs(w0)
    print(f"{name}: layer-0 attention max error {aerr.max():.4f}, {outside.mean():.2e} of elements outside the bf16 bar")
    assert outside.mean() <= 1e-2 and aerr.max() < 0.1, f"{name}: layer-0 attention"
    err = np.abs(out["base_logits"].cpu().numpy() - ref["base_logits"])
    tol = 1e-2 + 2e-2 * np.abs(ref["base_logits"])
    print(f"{name}: logits max error {err.max():.4f}, {(err > tol).mean():.2e} of them outside the bf16 tolerance")
    assert err.max() < UNSCALED_MARGIN / 2.5 * 1.5, f"{name}: logit error {err.max():.3f} above the conditioning's range"
    gtok = out["tokens"].cpu().numpy().astype(np.int64)
    toks, margins = O.teacher_forced_walk(W, ref["base_logits"], anchors, gtok)
    decisive = margins > UNSCALED_MARGIN
    assert (toks[decisive] == gtok[decisive]).all(), f"{name}: token differs at a margin above {UNSCALED_MARGIN}"
    assert decisive.sum() >= 1, f"{name}: no position with a margin above {UNSCALED_MARGIN}"


def test_unit_gains_small_model():
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 91, unit_attention_logits=False)
    lens, pos0 = [64, 300, 1], [0, 40, 9]
    hid = torch.randn(3, 300, m.hidden_size, generator=torch.Generator().manual_seed(12)).to(torch.bfloat16)
    anchors = [17, 4000, 3]
    cache, out, dump, block_pos = _round(model, W, m, hid, lens, pos0, anchors)
    kv = O.project_context_kv(W, hid, pos0, lengths=lens)
    _check("small, unit gains", m, W, cache, kv, out, dump, anchors, block_pos, lens)


@pytest.mark.slow
def test_unit_gains_single_request():
    wl = WORKLOADS["single_bf16"]
    m = wl.model
    cpu, W, model = build(m, wl.seed, unit_attention_logits=False)
    inp = make_round_inputs(wl)
    lens, pos0, anchors = inp["ctx_len"].tolist(), inp["pos0"].tolist(), inp["anchors"].tolist()
    cache, out, dump, block_pos = _round(model, W, m, inp["hidden"], lens, pos0, anchors)
    kv = O.project_context_kv(W, inp["hidden"], pos0, lengths=lens)
    _check("single request, unit gains", m, W, cache, kv, out, dump, anchors, block_pos, lens,
           rows_to_check=np.r_[0:64, 2000:2064, 4032:4096])
