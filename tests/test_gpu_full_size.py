"""GPU parity at the five workloads' full sizes, in the launch configuration the
benchmark uses (the K+V context cache; single_bf16, quant4_bf16 and the
incremental rounds also on the V-only cache). The GPU runs every row; the oracle
recomputes sampled rows (rows are independent in every step of the round), so
it finishes in minutes on the host cores."""
import numpy as np
import pytest
import torch

from oracle import dspark as O
from synthetic import WORKLOADS, make_append_schedule, make_round_inputs
from parity_util import as_stored, assert_close, build, check_tokens, CONF_TOL, ensure_built

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    ensure_built()


def _compare_rows(wl, W, out, kv_rows, sample, anchors, block_pos):
    m = wl.model
    ref = O.draft_rows(W, as_stored(kv_rows, m.dtype), [anchors[b] for b in sample], [block_pos[b] for b in sample])
    U = out["base_logits"][sample].cpu().numpy()
    assert_close(U, ref["base_logits"], m.dtype, f"{wl.name}: base logits rows {sample}")
    gtok = out["tokens"][sample].cpu().numpy().astype(np.int64)
    checked, total = check_tokens(W, ref["base_logits"], [anchors[b] for b in sample], gtok, f"{wl.name}: tokens")
    assert checked >= total // 2
    conf_ref = O.confidence(W, ref["hidden"], [anchors[b] for b in sample], gtok)
    assert np.max(np.abs(out["conf"][sample].cpu().numpy() - conf_ref)) <= CONF_TOL
    assert (out["lengths"].cpu().numpy() == m.block_size).all()


def _check_kv(cache, kv_rows, sample, lens, dtype, name, rows_to_check=None):
    for i, b in enumerate(sample):
        L = lens[i]
        idx = np.arange(L) if rows_to_check is None else rows_to_check
        v = cache.v[:, b, idx].float().cpu().numpy()
        for l in range(v.shape[0]):
            if cache.k is not None:                       # a V-only cache holds v alone
                k = cache.k[l, b, idx].float().cpu().numpy()
                assert_close(k, kv_rows[i][l][0][idx], dtype, f"{name}: K layer {l} row {b}")
            assert_close(v[l], kv_rows[i][l][1][idx], dtype, f"{name}: V layer {l} row {b}")


def _ragged_extremes():
    """Row 0 plus the rows with the shortest and the longest context of the ragged workload."""
    from synthetic import round_meta
    lens = round_meta(WORKLOADS["ragged_bf16"])[0]
    return sorted({0, int(lens.argmin()), int(lens.argmax())})


@pytest.mark.parametrize("name,sample,v_only", [("single_bf16", [0], False), ("single_bf16", [0], True),
                                                ("ragged_bf16", _ragged_extremes(), False),
                                                ("quant4_bf16", [0, 63], False), ("quant4_bf16", [0, 63], True)])
def test_full_size_round(name, sample, v_only):
    import block_draft_model_dspark_b200 as dsp
    wl = WORKLOADS[name]
    m = wl.model
    cpu, W, model = build(m, wl.seed)
    inp = make_round_inputs(wl)
    lens = inp["ctx_len"].tolist()
    cache = dsp.KvCache(model, wl.rows, int(inp["hidden"].shape[1]), v_only=v_only,
                        pos0=inp["pos0"].cuda() if v_only else None)
    cache.set_lengths([0] * wl.rows)
    model.dspark_append_context_kv(cache, inp["hidden"].cuda(), lens, inp["pos0"].cuda())
    anchors, block_pos = inp["anchors"].tolist(), inp["block_pos"].tolist()
    out = model.draft(cache, inp["anchors"].cuda(), inp["block_pos"].cuda(), max(lens))
    torch.cuda.synchronize()
    assert model.dspark_read_device_status() == 0
    del inp
    sub = make_round_inputs(wl, rows=sample)
    kv_rows = O.project_context_kv(W, sub["hidden"], sub["pos0"].tolist(), lengths=sub["ctx_len"].tolist())
    _check_kv(cache, kv_rows, sample, sub["ctx_len"].tolist(), m.dtype, name,
              rows_to_check=None if max(lens) <= 4096 else np.r_[0:64, 4000:4100, -64:0])
    _compare_rows(wl, W, out, kv_rows, sample, anchors, block_pos)


@pytest.mark.parametrize("v_only", [False, True])
def test_long_incremental_rounds(v_only):
    import block_draft_model_dspark_b200 as dsp
    wl = WORKLOADS["long_incremental_bf16"]
    m = wl.model
    cpu, W, model = build(m, wl.seed)
    inp = make_round_inputs(wl)
    A = wl.rows
    pos0 = inp["pos0"].cuda()
    cache = dsp.KvCache(model, A, wl.capacity, v_only=v_only, pos0=pos0 if v_only else None)
    cache.set_lengths([0] * A)
    model.dspark_append_context_kv(cache, inp["hidden"].cuda(), inp["ctx_len"].tolist(), pos0)
    sample = [1]
    sub = make_round_inputs(wl, rows=sample)
    kv_rows = O.project_context_kv(W, sub["hidden"], sub["pos0"].tolist(), lengths=sub["ctx_len"].tolist())
    del inp
    lens = [wl.ctx_len] * A
    for r, step in enumerate(make_append_schedule(wl)):
        model.dspark_append_context_kv(cache, step["hidden"].cuda(), step["n_new"].tolist(), pos0)
        n_new = step["n_new"].tolist()
        for i, b in enumerate(sample):
            new = O.project_context_kv(W, step["hidden"][b:b + 1], [lens[b]], lengths=[n_new[b]])
            kv_rows[i] = [(np.concatenate([kv_rows[i][l][0], new[0][l][0]]),
                           np.concatenate([kv_rows[i][l][1], new[0][l][1]])) for l in range(m.num_hidden_layers)]
        lens = [lens[b] + n_new[b] for b in range(A)]
        block_pos = lens[:]                     # positions start at 0: the block follows the context
        bp = torch.tensor(block_pos, dtype=torch.int32, device="cuda")
        out = model.draft(cache, step["anchors"].cuda(), bp, max(lens))
        torch.cuda.synchronize()
        assert cache.len.cpu().tolist() == lens
        if r in (0, wl.append_rounds - 1):
            new_rows = np.arange(lens[sample[0]] - 40, lens[sample[0]])
            _check_kv(cache, kv_rows, sample, [lens[b] for b in sample], m.dtype, f"round {r}", rows_to_check=new_rows)
            _compare_rows(wl, W, out, kv_rows, sample, step["anchors"].tolist(), block_pos)
    assert model.dspark_read_device_status() == 0
