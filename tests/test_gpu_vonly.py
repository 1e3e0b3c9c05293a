"""The V-only context cache (dspark_kv_cache.k = NULL) against the fp64 oracle.

With attention_k_eq_v the keys and values come from one k_proj row and one
normalisation, so k = rope(v * k_norm, position) ("@mlx-bun/inference 0.0.0-stage
-> 1.0.0", deepspec.ts #projectContextKVRows). A V-only cache stores v alone and
the attention rebuilds k from it; the round must then match the oracle's round on
the full K/V exactly as the K+V cache does. Rotary widths: partial 1.0 (every
pair, the workloads' setting), 0.5, and 0.2 (13 of 64 pairs; the rest at
frequency 0, where the rebuild reduces to k = v * k_norm).
"""
import numpy as np
import pytest
import torch

from oracle import dspark as O
from synthetic import small_model
from parity_util import CONF_TOL, as_stored, assert_close, build, check_tokens, ensure_built

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    ensure_built()


def _cache(model, hid, lens, pos0, v_only, capacity=None):
    import block_draft_model_dspark_b200 as dsp
    B, L = hid.shape[0], hid.shape[1]
    pos = torch.tensor(pos0, dtype=torch.int32, device="cuda")
    cache = dsp.KvCache(model, B, capacity or L, v_only=v_only, pos0=pos if v_only else None)
    cache.set_lengths([0] * B)
    model.dspark_append_context_kv(cache, hid.cuda(), [int(x) for x in lens], pos)
    return cache


def _round_with_dump(model, m, cache, anchors, block_pos, max_len):
    A = len(anchors)
    dump = torch.full((m.num_hidden_layers, A, m.block_size, m.num_attention_heads, m.global_head_dim),
                      float("nan"), dtype=torch.float32, device="cuda")
    model.dspark_debug_attention_dump(dump)
    try:
        out = model.draft(cache, torch.tensor(anchors, dtype=torch.int32, device="cuda"),
                          torch.tensor(block_pos, dtype=torch.int32, device="cuda"), max_len)
        torch.cuda.synchronize()
    finally:
        model.dspark_debug_attention_dump(None)
    assert model.dspark_read_device_status() == 0
    return out, dump


@pytest.mark.parametrize("partial", [1.0, 0.5, 0.2])
@pytest.mark.parametrize("lens,pos0", [([37, 0, 200], [0, 50, 4000]), ([1500, 3, 777], [0, 9, 123456])],
                         ids=["short", "split"])
def test_vonly_round_matches_oracle(partial, lens, pos0):
    """Every layer's attention, the logits, tokens and confidences of a round on a V-only
    cache against the oracle; "split" spreads each row over several CTAs (merge kernel)."""
    m = small_model(dtype="bf16", partial_rotary_factor=partial)
    cpu, W, model = build(m, 71)
    A, Lmax = len(lens), max(lens)
    hid = torch.randn(A, Lmax, m.hidden_size, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    cache = _cache(model, hid, lens, pos0, v_only=True)
    assert cache.k is None
    kv = O.project_context_kv(W, hid, pos0, lengths=lens)
    v = cache.v.float().cpu().numpy()
    for b, L in enumerate(lens):
        for l in range(m.num_hidden_layers):
            assert_close(v[l, b, :L], kv[b][l][1], "bf16", f"V layer {l} row {b}")
    anchors = [5, m.vocab_size - 2, 1234][:A]
    block_pos = [p + L for p, L in zip(pos0, lens)]
    out, dump = _round_with_dump(model, m, cache, anchors, block_pos, Lmax)
    ref = O.draft_rows(W, as_stored(kv, "bf16"), anchors, block_pos, keep_attention=True)
    for l in range(m.num_hidden_layers):
        assert_close(dump[l].cpu().numpy(), ref["attention"][l], "bf16", f"V-only attention layer {l}")
    assert_close(out["base_logits"].cpu().numpy(), ref["base_logits"], "bf16", "V-only base logits")
    gtok = out["tokens"].cpu().numpy().astype(np.int64)
    checked, total = check_tokens(W, ref["base_logits"], anchors, gtok, "V-only tokens")
    assert checked >= total // 2
    if m.enable_confidence_head:
        conf_ref = O.confidence(W, ref["hidden"], anchors, gtok)
        assert np.max(np.abs(out["conf"].cpu().numpy() - conf_ref)) <= CONF_TOL


def test_vonly_matches_full_cache():
    """The same rows through a K+V cache and a V-only cache: identical v rows (bit for bit),
    attention outputs within the bf16 bar of each other, the same decisive tokens."""
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 72)
    lens, pos0 = [1500, 3, 777, 64], [0, 10, 123, 5000]
    A, Lmax = len(lens), max(lens)
    hid = torch.randn(A, Lmax, m.hidden_size, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    full = _cache(model, hid, lens, pos0, v_only=False)
    vc = _cache(model, hid, lens, pos0, v_only=True)
    torch.cuda.synchronize()
    for b, L in enumerate(lens):
        assert torch.equal(full.v[:, b, :L].view(torch.int16), vc.v[:, b, :L].view(torch.int16)), f"v rows of row {b}"
    anchors = [1, 2, 3, m.vocab_size - 1]
    block_pos = [p + L for p, L in zip(pos0, lens)]
    out_f, dump_f = _round_with_dump(model, m, full, anchors, block_pos, Lmax)
    out_v, dump_v = _round_with_dump(model, m, vc, anchors, block_pos, Lmax)
    assert_close(dump_v.cpu().numpy(), dump_f.cpu().numpy(), "bf16", "V-only vs K+V attention")
    U = out_f["base_logits"].cpu().numpy()
    assert_close(out_v["base_logits"].cpu().numpy(), U, "bf16", "V-only vs K+V logits")
    srt = np.sort(U, -1)
    decisive = (srt[..., -1] - srt[..., -2]) > 5e-2
    tf, tv = out_f["tokens"].cpu().numpy(), out_v["tokens"].cpu().numpy()
    # the walk adds the Markov bias of the previous token: compare the first step, where both
    # walks start from the same anchor, at every decisive position
    assert (tf[:, 0][decisive[:, 0]] == tv[:, 0][decisive[:, 0]]).all()


def test_vonly_refusals():
    import block_draft_model_dspark_b200 as dsp
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 73)
    A, G, nH, nKv, hd = 2, m.block_size, m.num_attention_heads, m.num_global_key_value_heads, m.global_head_dim
    pos = torch.zeros(A, dtype=torch.int32, device="cuda")
    vc = dsp.KvCache(model, A, 64, v_only=True, pos0=pos)
    vc.set_lengths([10, 20])
    t = model.kv_torch_dtype
    q = torch.zeros(A, G, nH, hd, dtype=t, device="cuda")
    kb = torch.zeros(A, G, nKv, hd, dtype=t, device="cuda")
    out = torch.empty_like(q)
    # the attend seam takes explicit keys: a V-only cache is refused
    with pytest.raises(dsp.DsparkError) as e:
        model.dspark_attend(0, vc, q, kb, kb, out, 20)
    assert e.value.code == dsp.DSPARK_ERR_INVALID_ARGUMENT
    # a V-only cache without pos0
    nopos = dsp.KvCache(model, A, 64, v_only=True, pos0=None)
    nopos.set_lengths([10, 20])
    anchors = torch.zeros(A, dtype=torch.int32, device="cuda")
    with pytest.raises(dsp.DsparkError) as e:
        model.draft(nopos, anchors, pos, 20)
    assert e.value.code == dsp.DSPARK_ERR_INVALID_ARGUMENT
    # an fp32 model runs the CUDA-core attention: V-only is unsupported there
    m32 = small_model(dtype="fp32")
    _, _, model32 = build(m32, 74)
    vc32 = dsp.KvCache(model32, A, 64, v_only=True, pos0=pos)
    vc32.set_lengths([0, 0])
    with pytest.raises(dsp.DsparkError) as e:
        model32.draft(vc32, anchors, pos, 0)
    assert e.value.code == dsp.DSPARK_ERR_UNSUPPORTED
    hid = torch.zeros(A, 4, m32.hidden_size, dtype=torch.float32, device="cuda")
    with pytest.raises(dsp.DsparkError) as e:
        model32.dspark_append_context_kv(vc32, hid, [1, 1], pos)
    assert e.value.code == dsp.DSPARK_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert model.dspark_read_device_status() == 0


def test_project_without_k_writes_v_alone():
    """dspark_project_context_kv with k_out = NULL writes the same v rows as with k_out, and a
    round on the resulting V-only cache equals the round on the appended one."""
    import block_draft_model_dspark_b200 as dsp
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 75)
    B, L = 2, 300
    pos0 = torch.tensor([0, 777], dtype=torch.int32, device="cuda")
    hid = torch.randn(B, L, m.hidden_size, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16).cuda()
    full = dsp.KvCache(model, B, L)
    model.dspark_project_context_kv(hid, full.k, full.v, pos0=pos0)
    vc = dsp.KvCache(model, B, L, v_only=True, pos0=pos0)
    vc.v.fill_(float("nan"))
    model.dspark_project_context_kv(hid, None, vc.v, pos0=pos0)
    torch.cuda.synchronize()
    assert torch.equal(full.v.view(torch.int16), vc.v.view(torch.int16))
    appended = _cache(model, hid.cpu(), [L, L], pos0.tolist(), v_only=True)
    vc.set_lengths([L, L])
    anchors, block_pos = [3, 4], [L, 777 + L]
    a = model.draft(vc, torch.tensor(anchors, dtype=torch.int32, device="cuda"),
                    torch.tensor(block_pos, dtype=torch.int32, device="cuda"), L)
    b = model.draft(appended, torch.tensor(anchors, dtype=torch.int32, device="cuda"),
                    torch.tensor(block_pos, dtype=torch.int32, device="cuda"), L)
    torch.cuda.synchronize()
    assert torch.equal(a["tokens"], b["tokens"])
    assert torch.equal(a["base_logits"], b["base_logits"])
