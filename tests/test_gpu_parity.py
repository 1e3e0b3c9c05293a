"""GPU parity: libdspark's kernels (through the C ABI) against the fp64 oracle.

Small models here span several tiles and ragged tails in every dimension;
the full-size workloads are in test_gpu_full_size.py.
"""
import math

import numpy as np
import pytest
import torch

from oracle import dspark as O
from synthetic import WORKLOADS, make_round_inputs, make_weights, small_model
from parity_util import as_stored, assert_close, build, check_tokens, CONF_TOL, ensure_built

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    ensure_built()


def _project_into_cache(model, hidden_cpu, lens, pos0, capacity=None):
    """Cache of `capacity` rows per batch row with rows [0, lens[b]) appended at pos0[b]."""
    import block_draft_model_dspark_b200 as dsp
    B, L = hidden_cpu.shape[0], hidden_cpu.shape[1]
    cache = dsp.KvCache(model, B, capacity or L)
    cache.set_lengths([0] * B)
    model.dspark_append_context_kv(cache, hidden_cpu.cuda(), [int(x) for x in lens],
                                   torch.tensor(pos0, dtype=torch.int32, device="cuda"))
    return cache


def _check_cache_rows(cache, kv_oracle, lens, dtype):
    k = cache.k.float().cpu().numpy()
    v = cache.v.float().cpu().numpy()
    for b, L in enumerate(lens):
        for l in range(k.shape[0]):
            assert_close(k[l, b, :L], kv_oracle[b][l][0], dtype, f"K layer {l} row {b}")
            assert_close(v[l, b, :L], kv_oracle[b][l][1], dtype, f"V layer {l} row {b}")


def _round_and_compare(shape, W, model, cache, kv_oracle, anchors, block_pos, lens, what):
    A = len(anchors)
    dev_anchors = torch.tensor(anchors, dtype=torch.int32, device="cuda")
    dev_bpos = torch.tensor(block_pos, dtype=torch.int32, device="cuda")
    out = model.draft(cache, dev_anchors, dev_bpos, max(lens) if len(lens) else 0)
    torch.cuda.synchronize()
    assert model.dspark_read_device_status() == 0
    ref = O.draft_rows(W, as_stored(kv_oracle, shape.dtype), anchors, block_pos)
    assert_close(out["base_logits"].cpu().numpy(), ref["base_logits"], shape.dtype, f"{what}: base logits")
    gtok = out["tokens"].cpu().numpy().astype(np.int64)
    checked, total = check_tokens(W, ref["base_logits"], anchors, gtok, f"{what}: tokens")
    assert checked >= total // 2, f"{what}: too few decisive steps ({checked}/{total})"
    if shape.enable_confidence_head:
        conf_ref = O.confidence(W, ref["hidden"], anchors, gtok)
        gconf = out["conf"].cpu().numpy()
        assert np.max(np.abs(gconf - conf_ref)) <= CONF_TOL, f"{what}: confidence"
        lens_gpu = out["lengths"].cpu().numpy()
        for b in range(A):
            assert lens_gpu[b] == O.prefix_length(gconf[b], shape.confidence_threshold, shape.block_size)
    else:
        assert (out["lengths"].cpu().numpy() == shape.block_size).all()
    return out, ref


# ----------------------------------------------------------------------------- the tiny fp32 workload

def test_tiny_fp32_workload_round():
    wl = WORKLOADS["tiny_fp32"]
    m = wl.model
    cpu, W, model = build(m, wl.seed)
    inp = make_round_inputs(wl)
    lens = inp["ctx_len"].tolist()
    cache = _project_into_cache(model, inp["hidden"], lens, inp["pos0"].tolist())
    kv = O.project_context_kv(W, inp["hidden"], inp["pos0"].tolist(), lengths=lens)
    _check_cache_rows(cache, kv, lens, "fp32")
    _round_and_compare(m, W, model, cache, kv, inp["anchors"].tolist(), inp["block_pos"].tolist(), lens, "tiny_fp32")


def test_project_context_kv_static_and_dynamic_positions():
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 3)
    import block_draft_model_dspark_b200 as dsp
    hid = torch.randn(3, 70, m.hidden_size, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    for pos0 in (None, [5, 0, 9000]):
        cache = dsp.KvCache(model, 3, 70)
        model.dspark_project_context_kv(hid.cuda(), cache.k, cache.v,
                                        pos0=None if pos0 is None else torch.tensor(pos0, dtype=torch.int32, device="cuda"),
                                        static_pos=17)
        torch.cuda.synchronize()
        kv = O.project_context_kv(W, hid, pos0 if pos0 is not None else [17, 17, 17])
        _check_cache_rows(cache, kv, [70, 70, 70], "bf16")


# ----------------------------------------------------------------------------- attention seam

@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_attend_matches_concat_sdpa(dtype):
    m = small_model(dtype=dtype, block_size=8)
    cpu, W, model = build(m, 5)
    import block_draft_model_dspark_b200 as dsp
    tdt = model.kv_torch_dtype              # the seam's tensors are in the KV dtype (fp16 for a bf16 model)
    A, G, nH, nKv, hd = 4, m.block_size, m.num_attention_heads, m.num_global_key_value_heads, m.global_head_dim
    lens = [0, 1, 333, 1000]
    cap = 1003
    g = torch.Generator().manual_seed(7)
    cache = dsp.KvCache(model, A, cap)
    cache.k.copy_((torch.randn(cache.k.shape, generator=g) * 0.6).to(tdt))
    cache.v.copy_(torch.randn(cache.v.shape, generator=g).to(tdt))
    cache.set_lengths(lens)
    q = (torch.randn(A, G, nH, hd, generator=g) * 0.6).to(tdt)
    kb = (torch.randn(A, G, nKv, hd, generator=g) * 0.6).to(tdt)
    vb = torch.randn(A, G, nKv, hd, generator=g).to(tdt)
    out = torch.empty(A, G, nH, hd, dtype=tdt, device="cuda")
    for layer in range(m.num_hidden_layers):
        model.dspark_attend(layer, cache, q.cuda(), kb.cuda(), vb.cuda(), out, max(lens))
        torch.cuda.synchronize()
        kc, vc = cache.k[layer].float().cpu().numpy(), cache.v[layer].float().cpu().numpy()
        for b in range(A):
            ref = O.attend_concat(q[b].double().numpy(), kc[b, :lens[b]], vc[b, :lens[b]], kb[b].double().numpy(),
                                  vb[b].double().numpy())
            assert_close(out[b].float().cpu().numpy(), ref, dtype, f"attend layer {layer} row {b}")


@pytest.mark.parametrize("slope", [0.25, -0.25])
def test_attend_rising_and_falling_logits(slope):
    """Logits that rise along the keys by 16 per 64-key tile (every tile raises the
    running maximum past the kernel's rescale headroom, so the output state is
    rescaled at every tile, and the block's keys rise further), and the mirror case
    (the first tile holds the maximum: never rescaled). q . k_j = slope * j exactly
    in fp16 (k_j = j / 16 in head dimension 0, q = 4 slope there)."""
    import block_draft_model_dspark_b200 as dsp
    m = small_model(dtype="bf16", block_size=8)
    cpu, W, model = build(m, 5)
    tdt = model.kv_torch_dtype
    A, G, nH, nKv, hd = 3, m.block_size, m.num_attention_heads, m.num_global_key_value_heads, m.global_head_dim
    lens = [1000, 64, 7]
    cap = 1000
    g = torch.Generator().manual_seed(17)
    cache = dsp.KvCache(model, A, cap)
    k = torch.zeros(cache.k.shape)
    v = torch.randn(cache.v.shape, generator=g)
    for b in range(A):
        k[:, b, :, :, 0] = (torch.arange(cap, dtype=torch.float32) / 16.0)[None, :, None]
    cache.k.copy_(k.to(tdt))
    cache.v.copy_(v.to(tdt))
    cache.set_lengths(lens)
    q = torch.zeros(A, G, nH, hd)
    q[..., 0] = 4.0 * slope
    kb = torch.zeros(A, G, nKv, hd)
    for b in range(A):
        kb[b, :, :, 0] = ((lens[b] + torch.arange(G, dtype=torch.float32)) / 16.0)[:, None]
    vb = torch.randn(A, G, nKv, hd, generator=g)
    q, kb, vb = q.to(tdt), kb.to(tdt), vb.to(tdt)
    out = torch.empty(A, G, nH, hd, dtype=tdt, device="cuda")
    model.dspark_attend(0, cache, q.cuda(), kb.cuda(), vb.cuda(), out, max(lens))
    torch.cuda.synchronize()
    assert model.dspark_read_device_status() == 0
    kc, vc = cache.k[0].float().cpu().numpy(), cache.v[0].float().cpu().numpy()
    for b in range(A):
        ref = O.attend_concat(q[b].double().numpy(), kc[b, :lens[b]], vc[b, :lens[b]], kb[b].double().numpy(),
                              vb[b].double().numpy())
        assert_close(out[b].float().cpu().numpy(), ref, "bf16", f"attend slope {slope} row {b}")


def test_attend_refuses_misaligned_buffers():
    """The seam's vector loads and stores need 16-byte aligned q, k_blk, v_blk and
    out: both entry points refuse a misaligned one before any launch."""
    import block_draft_model_dspark_b200 as dsp
    m = small_model(dtype="bf16", block_size=8)
    cpu, W, model = build(m, 5)
    tdt = model.kv_torch_dtype
    A, G, nH, nKv, hd = 2, m.block_size, m.num_attention_heads, m.num_global_key_value_heads, m.global_head_dim
    cache = dsp.KvCache(model, A, 64)
    cache.k.zero_(); cache.v.zero_()
    cache.set_lengths([10, 64])
    q = torch.zeros(A, G, nH, hd, dtype=tdt, device="cuda")
    kb = torch.zeros(A, G, nKv, hd, dtype=tdt, device="cuda")
    vb = torch.zeros_like(kb)
    n = A * G * nH * hd
    flat = torch.zeros(n + 8, dtype=tdt, device="cuda")
    bad = flat[1:1 + n].view(A, G, nH, hd)                 # 2 bytes past a 256-byte boundary
    for call in (model.dspark_attend, model.dspark_attend_no_alloc):
        for args in ((bad, kb, vb, q.clone()), (q, kb, vb, bad)):
            with pytest.raises(dsp.DsparkError) as ei:
                call(0, cache, *args, 64)
            assert ei.value.code == dsp.DSPARK_ERR_INVALID_ARGUMENT
    torch.cuda.synchronize()
    assert model.dspark_read_device_status() == 0


# ----------------------------------------------------------------------------- whole rounds, small models

@pytest.mark.parametrize("quant", [0, 4])
def test_small_bf16_ragged_round(quant):
    m = small_model(dtype="bf16", quant_bits=quant)
    cpu, W, model = build(m, 11 + quant)
    A = 3
    lens = [37, 0, 200]
    pos0 = [0, 50, 4000]
    hid = torch.randn(A, 200, m.hidden_size, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    cache = _project_into_cache(model, hid, lens, pos0)
    kv = O.project_context_kv(W, hid, pos0, lengths=lens)
    _check_cache_rows(cache, kv, lens, "bf16")
    anchors = [5, m.vocab_size - 2, 1234]
    block_pos = [p + L for p, L in zip(pos0, lens)]
    _round_and_compare(m, W, model, cache, kv, anchors, block_pos, lens, f"small bf16 q{quant}")


def test_strong_markov_walk_and_threshold():
    """Markov tables scaled so the transition bias reorders tokens; threshold 0.5 truncates."""
    m = small_model(dtype="bf16", confidence_threshold=0.5)
    cpu, W, model = build(m, 21, markov_scale=60.0)
    A, lens, pos0 = 2, [64, 129], [0, 7]
    hid = torch.randn(A, 129, m.hidden_size, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    cache = _project_into_cache(model, hid, lens, pos0)
    kv = O.project_context_kv(W, hid, pos0, lengths=lens)
    out, ref = _round_and_compare(m, W, model, cache, kv, [3, 4], [64, 136], lens, "strong markov")
    # the bias matters: the walk differs from per-step argmax of U somewhere
    assert (ref["tokens"] != np.argmax(ref["base_logits"], -1)).any()


@pytest.mark.parametrize("A", [1, 8, 9])
def test_rank64_markov_walk(A):
    """markov_rank 64 with a strong bias: the tensor-core walk (A <= 8) and the
    CUDA-core persistent walk (A = 9) against the oracle's teacher-forced walk."""
    m = small_model(dtype="bf16", markov_rank=64)
    cpu, W, model = build(m, 41, markov_scale=30.0)
    g = torch.Generator().manual_seed(40 + A)
    lens = [int(x) for x in torch.randint(1, 97, (A,), generator=g)]
    pos0 = [int(x) for x in torch.randint(0, 500, (A,), generator=g)]
    hid = torch.randn(A, max(lens), m.hidden_size, generator=g).to(torch.bfloat16)
    cache = _project_into_cache(model, hid, lens, pos0)
    kv = O.project_context_kv(W, hid, pos0, lengths=lens)
    anchors = [int(x) for x in torch.randint(0, m.vocab_size - 1, (A,), generator=g)]
    block_pos = [p + L for p, L in zip(pos0, lens)]
    out, ref = _round_and_compare(m, W, model, cache, kv, anchors, block_pos, lens, f"rank 64, A={A}")
    assert (ref["tokens"] != np.argmax(ref["base_logits"], -1)).any()


def test_pruned_markov_walk():
    """markov_rank 64 with a moderate bias (markov_scale 3): every position keeps
    16-192 candidates under the norm bound, so the pruned walk decides the tokens
    (the strong-bias case above overflows the lists and exercises the fallback to
    the full walk); the bias changes the argmax at some positions."""
    m = small_model(dtype="bf16", markov_rank=64)
    cpu, W, model = build(m, 43, markov_scale=3.0)
    A = 4
    g = torch.Generator().manual_seed(70 + A)
    lens = [int(x) for x in torch.randint(1, 97, (A,), generator=g)]
    pos0 = [int(x) for x in torch.randint(0, 500, (A,), generator=g)]
    hid = torch.randn(A, max(lens), m.hidden_size, generator=g).to(torch.bfloat16)
    cache = _project_into_cache(model, hid, lens, pos0)
    kv = O.project_context_kv(W, hid, pos0, lengths=lens)
    anchors = [int(x) for x in torch.randint(0, m.vocab_size - 1, (A,), generator=g)]
    block_pos = [p + L for p, L in zip(pos0, lens)]
    out, ref = _round_and_compare(m, W, model, cache, kv, anchors, block_pos, lens, "pruned walk, A=4")
    assert (ref["tokens"] != np.argmax(ref["base_logits"], -1)).any()


def test_rank0_no_confidence_head():
    m = small_model(dtype="bf16", markov_rank=0, enable_confidence_head=False, confidence_head_with_markov=False)
    cpu, W, model = build(m, 31)
    lens, pos0 = [90], [3]
    hid = torch.randn(1, 90, m.hidden_size, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    cache = _project_into_cache(model, hid, lens, pos0)
    kv = O.project_context_kv(W, hid, pos0, lengths=lens)
    _round_and_compare(m, W, model, cache, kv, [9], [93], lens, "rank 0")


# ----------------------------------------------------------------------------- the incremental cache

def test_append_equals_recompute_with_sentinels():
    import block_draft_model_dspark_b200 as dsp
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 41)
    B, cap = 3, 96
    pos0 = torch.tensor([0, 100, 7], dtype=torch.int32, device="cuda")
    cache = dsp.KvCache(model, B, cap)
    sentinel = torch.tensor(-12345.0, dtype=cache.k.dtype)
    cache.k.fill_(sentinel)
    cache.v.fill_(sentinel)
    cache.set_lengths([0, 0, 0])
    g = torch.Generator().manual_seed(9)
    rows = [[] for _ in range(B)]
    sched = [[5, 1, 16], [16, 0, 3], [1, 16, 16], [7, 9, 0]]
    for n_new in sched:
        hid = torch.randn(B, 16, m.hidden_size, generator=g).to(torch.bfloat16)
        model.dspark_append_context_kv(cache, hid.cuda(), n_new, pos0)
        for b in range(B):
            rows[b].append(hid[b, :n_new[b]])
    torch.cuda.synchronize()
    lens = [sum(s[b] for s in sched) for b in range(B)]
    assert cache.len.cpu().tolist() == lens
    full = [torch.cat(r) for r in rows]
    Lmax = max(lens)
    hid_full = torch.zeros(B, Lmax, m.hidden_size, dtype=torch.bfloat16)
    for b in range(B):
        hid_full[b, :lens[b]] = full[b]
    # recompute all rows at once on the GPU
    ref = dsp.KvCache(model, B, Lmax)
    model.dspark_project_context_kv(hid_full.cuda(), ref.k, ref.v, pos0=pos0)
    torch.cuda.synchronize()
    kv = O.project_context_kv(W, hid_full, pos0.cpu().tolist(), lengths=lens)
    _check_cache_rows(cache, kv, lens, "bf16")
    same = total = 0
    for b in range(B):
        a = cache.k[:, b, :lens[b]]
        r = ref.k[:, b, :lens[b]]
        same += int((a.view(torch.int16) == r.view(torch.int16)).sum())
        total += a.numel()
        # rows past len were never written
        assert (cache.k[:, b, lens[b]:].view(torch.int16) == sentinel.view(torch.int16).item()).all()
        assert (cache.v[:, b, lens[b]:].view(torch.int16) == sentinel.view(torch.int16).item()).all()
    assert same / total > 0.99, f"append vs recompute: only {same}/{total} bf16 values bit-identical"


def test_refused_append_leaves_cache_untouched():
    """The accepted-row counts live on the device, so the append validates them there: a count
    past the capacity (or outside [0, Lnew_max]) refuses the whole append, writes no cache row,
    leaves len unchanged and sets DSPARK_DEV_CAPACITY; the next valid append goes through."""
    import block_draft_model_dspark_b200 as dsp
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 43)
    cache = dsp.KvCache(model, 2, 20)
    cache.k.zero_(); cache.v.zero_()
    cache.set_lengths([10, 18])
    k0, v0 = cache.k.clone(), cache.v.clone()
    hid = torch.randn(2, 4, m.hidden_size).to(torch.bfloat16).cuda()
    pos0 = torch.zeros(2, dtype=torch.int32, device="cuda")
    for bad in ([4, 3], [1, -1], [5, 0]):          # past capacity; a negative count; above Lnew_max = 4
        model.dspark_append_context_kv(cache, hid, torch.tensor(bad, dtype=torch.int32, device="cuda"), pos0)
        assert model.dspark_read_device_status() == dsp.DSPARK_DEV_CAPACITY, bad
        assert torch.equal(cache.k, k0) and torch.equal(cache.v, v0) and cache.len.cpu().tolist() == [10, 18], bad
    model.dspark_append_context_kv(cache, hid, torch.tensor([4, 2], dtype=torch.int32, device="cuda"), pos0)
    assert model.dspark_read_device_status() == 0
    assert cache.len.cpu().tolist() == [14, 20]
    assert not torch.equal(cache.k, k0)
    with pytest.raises(dsp.DsparkError) as ei:      # host-side argument check: Lnew_max above the capacity
        model.dspark_append_context_kv(cache, torch.zeros(2, 21, m.hidden_size, dtype=torch.bfloat16, device="cuda"),
                                       torch.zeros(2, dtype=torch.int32, device="cuda"), pos0)
    assert ei.value.code == dsp.DSPARK_ERR_INVALID_ARGUMENT


def test_workspace_too_small_and_bad_anchor_status():
    import block_draft_model_dspark_b200 as dsp
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 47)
    cache = dsp.KvCache(model, 1, 8)
    cache.k.zero_(); cache.v.zero_()
    cache.set_lengths([8])
    anchors = torch.tensor([m.vocab_size + 5], dtype=torch.int32, device="cuda")
    bpos = torch.tensor([8], dtype=torch.int32, device="cuda")
    tok = torch.empty(1, m.block_size, dtype=torch.int32, device="cuda")
    lens = torch.empty(1, dtype=torch.int32, device="cuda")
    small = model.workspace(1024)
    with pytest.raises(dsp.DsparkError) as ei:
        model.dspark_draft_rows(cache, anchors, bpos, 8, tok, lens, ws=small)
    assert ei.value.code == dsp.DSPARK_ERR_WORKSPACE
    model.dspark_draft_rows(cache, anchors, bpos, 8, tok, lens)
    assert model.dspark_read_device_status() & dsp.DSPARK_DEV_BAD_TOKEN
    assert model.dspark_read_device_status() == 0     # read clears it
    t = tok.cpu()
    assert ((t >= 0) & (t < m.vocab_size)).all()


# ----------------------------------------------------------------------------- in-round dumps

def test_attention_dump_every_layer_and_logit_stats():
    """Each layer's attention output inside a round (the attend seam on the round's own
    activations) and the per-position logit statistics of the lm-head epilogue, against the
    oracle's round."""
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 61)
    A, lens, pos0 = 3, [40, 0, 150], [0, 9, 300]
    hid = torch.randn(A, 150, m.hidden_size, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    cache = _project_into_cache(model, hid, lens, pos0)
    kv = O.project_context_kv(W, hid, pos0, lengths=lens)
    anchors, block_pos = [7, 11, m.vocab_size - 2], [p + L for p, L in zip(pos0, lens)]
    G, nH, hd, L = m.block_size, m.num_attention_heads, m.global_head_dim, m.num_hidden_layers
    dump = torch.full((L, A, G, nH, hd), float("nan"), dtype=torch.float32, device="cuda")
    stats = torch.zeros(A * G * 4, dtype=torch.int32, device="cuda")
    model.dspark_debug_attention_dump(dump)
    model.dspark_debug_logit_stats(stats)
    try:
        out = model.draft(cache, torch.tensor(anchors, dtype=torch.int32, device="cuda"),
                          torch.tensor(block_pos, dtype=torch.int32, device="cuda"), max(lens))
        torch.cuda.synchronize()
    finally:
        model.dspark_debug_attention_dump(None)
        model.dspark_debug_logit_stats(None)
    ref = O.draft_rows(W, as_stored(kv, "bf16"), anchors, block_pos, keep_attention=True)
    for l in range(L):
        assert_close(dump[l].cpu().numpy(), ref["attention"][l], "bf16", f"attention dump layer {l}")
    st = stats.view(A * G, 4).cpu()
    fmax = st[:, 0].view(torch.float32).numpy().reshape(A, G)
    flse = st[:, 1].view(torch.float32).numpy().reshape(A, G)
    farg = st[:, 2].numpy().reshape(A, G)
    ncand = st[:, 3].numpy().reshape(A, G)
    U = ref["base_logits"]
    umax = U.max(-1)
    lse = umax + np.log(np.exp(U - umax[..., None]).sum(-1))
    assert_close(fmax, umax, "bf16", "row max")
    assert_close(flse, lse, "bf16", "row logsumexp")
    srt = np.sort(U, -1)
    decisive = (srt[..., -1] - srt[..., -2]) > 1e-2
    assert (farg[decisive] == U.argmax(-1)[decisive]).all(), "row argmax"
    assert (ncand >= 1).all() and (ncand <= 1024).all(), ncand
    # the dumps stay off once cleared: a round with them off does not touch the buffers
    dump.fill_(0.0)
    model.draft(cache, torch.tensor(anchors, dtype=torch.int32, device="cuda"),
                torch.tensor(block_pos, dtype=torch.int32, device="cuda"), max(lens))
    torch.cuda.synchronize()
    assert float(dump.abs().max()) == 0.0


@pytest.mark.parametrize("scale", [3.0, 30.0])
def test_walk_above_64_rows(scale):
    """A = 65 request rows: with a moderate bias the pruned walk decides every position; with a
    strong one the candidate lists overflow and the per-step full walk (the A > 64 path) runs."""
    m = small_model(dtype="bf16", markov_rank=64, num_hidden_layers=1)
    cpu, W, model = build(m, 71, markov_scale=scale)
    A = 65
    g = torch.Generator().manual_seed(72)
    lens = [int(x) for x in torch.randint(1, 33, (A,), generator=g)]
    pos0 = [int(x) for x in torch.randint(0, 500, (A,), generator=g)]
    hid = torch.randn(A, max(lens), m.hidden_size, generator=g).to(torch.bfloat16)
    cache = _project_into_cache(model, hid, lens, pos0)
    kv = O.project_context_kv(W, hid, pos0, lengths=lens)
    anchors = [int(x) for x in torch.randint(0, m.vocab_size - 1, (A,), generator=g)]
    block_pos = [p + L for p, L in zip(pos0, lens)]
    stats = torch.zeros(A * m.block_size * 4, dtype=torch.int32, device="cuda")
    model.dspark_debug_logit_stats(stats)
    try:
        out, ref = _round_and_compare(m, W, model, cache, kv, anchors, block_pos, lens, f"A=65, markov scale {scale}")
    finally:
        model.dspark_debug_logit_stats(None)
    ncand = stats.view(-1, 4)[:, 3].cpu().numpy()
    if scale == 3.0:
        assert (ncand <= 1024).all(), "the pruned walk should decide every position"
    else:
        assert (ncand > 1024).any(), "the strong bias should overflow a list and run the full walk"
    assert (ref["tokens"] != np.argmax(ref["base_logits"], -1)).any()


# ----------------------------------------------------------------------------- failure detection

def test_bounded_wait_times_out_and_context_stays_usable():
    """A device wait that nothing satisfies gives up after its limit, records
    DSPARK_DEV_WAIT_TIMEOUT, and the next round on the same context is correct."""
    import block_draft_model_dspark_b200 as dsp
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 81)
    model.dspark_debug_wait_probe(50_000)                   # 50 ms
    torch.cuda.synchronize()
    assert model.dspark_read_device_status() == dsp.DSPARK_DEV_WAIT_TIMEOUT
    assert model.dspark_read_device_status() == 0
    lens, pos0 = [33, 70], [0, 5]
    hid = torch.randn(2, 70, m.hidden_size, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16)
    cache = _project_into_cache(model, hid, lens, pos0)
    kv = O.project_context_kv(W, hid, pos0, lengths=lens)
    _round_and_compare(m, W, model, cache, kv, [1, 2], [33, 75], lens, "round after a wait timeout")
