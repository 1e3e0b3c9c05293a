"""The context feature projection (deepspec.ts #projectContext) against the fp64 oracle:
out = rms(target_hiddens @ fc^T, hidden_norm) from the target's tap hiddens."""
import numpy as np
import pytest
import torch

from oracle import dspark as O
from synthetic import make_context_projection, make_target_hiddens, quantize_affine4, small_model
from parity_util import as_stored, assert_close, build, ensure_built

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    ensure_built()


@pytest.mark.parametrize("dtype,taps", [("bf16", 3), ("bf16", 1), ("fp32", 2)])
def test_context_features_match_oracle(dtype, taps):
    m = small_model(dtype=dtype)
    cpu, W, model = build(m, 81)
    proj = make_context_projection(m, taps, 5)
    x = make_target_hiddens(m, taps, 2, 77, 6)
    out = model.dspark_project_context_features(x.cuda(), proj["fc"].cuda(), proj["hidden_norm"].cuda())
    torch.cuda.synchronize()
    assert model.dspark_read_device_status() == 0
    ref = O.project_context(proj["fc"], proj["hidden_norm"], x, m.rms_norm_eps)
    assert out.dtype == model.torch_dtype
    assert_close(out.float().cpu().numpy(), ref, dtype, f"context features ({dtype}, {taps} taps)")


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_context_features_with_a_4bit_fc(dtype):
    """A 4-bit affine fc (group 64), dequantized on load, against the oracle on the exact
    dequantized matrix."""
    m = small_model(dtype=dtype)
    cpu, W, model = build(m, 85)
    taps = 2
    proj = make_context_projection(m, taps, 13)
    q, sc, bi = quantize_affine4(proj["fc"].float(), 64)
    x = make_target_hiddens(m, taps, 2, 33, 14)
    out = model.dspark_project_context_features(x.cuda(), (q.cuda(), sc.cuda(), bi.cuda()),
                                                proj["hidden_norm"].cuda())
    torch.cuda.synchronize()
    fc = O.dequantize_affine4(q, sc, bi, 64)
    ref = O.project_context(fc, proj["hidden_norm"], x, m.rms_norm_eps)
    assert_close(out.float().cpu().numpy(), ref, dtype, f"context features, 4-bit fc ({dtype})")


def test_context_features_over_two_chunks():
    """More rows than one chunk of the projection's GEMM (16384): the rows on both sides of the
    seam and the last row."""
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 82)
    taps, L = 2, 16500
    proj = make_context_projection(m, taps, 7)
    x = make_target_hiddens(m, taps, 1, L, 8)
    out = model.dspark_project_context_features(x.cuda(), proj["fc"].cuda(), proj["hidden_norm"].cuda())
    torch.cuda.synchronize()
    rows = [0, 1, 16383, 16384, 16385, L - 1]
    ref = O.project_context(proj["fc"], proj["hidden_norm"], x[0, rows], m.rms_norm_eps)
    assert_close(out[0, rows].float().cpu().numpy(), ref, "bf16", "context features across the chunk seam")


def test_context_features_feed_the_kv_projection():
    """Features -> dspark_project_context_kv on the GPU against the oracle's chain (its features
    rounded to the model dtype, as the GPU stores them)."""
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 83)
    taps, B, L = 3, 2, 50
    proj = make_context_projection(m, taps, 9)
    x = make_target_hiddens(m, taps, B, L, 10)
    feats = model.dspark_project_context_features(x.cuda(), proj["fc"].cuda(), proj["hidden_norm"].cuda())
    import block_draft_model_dspark_b200 as dsp
    cache = dsp.KvCache(model, B, L)
    pos0 = torch.tensor([0, 300], dtype=torch.int32, device="cuda")
    model.dspark_project_context_kv(feats, cache.k, cache.v, pos0=pos0)
    torch.cuda.synchronize()
    ref_feats = O.store_rounded(O.project_context(proj["fc"], proj["hidden_norm"], x, m.rms_norm_eps), "bf16")
    kv = O.project_context_kv(W, ref_feats, [0, 300])
    k, v = cache.k.float().cpu().numpy(), cache.v.float().cpu().numpy()
    for b in range(B):
        for l in range(m.num_hidden_layers):
            assert_close(k[l, b], kv[b][l][0], "bf16", f"K layer {l} row {b}")
            assert_close(v[l, b], kv[b][l][1], "bf16", f"V layer {l} row {b}")


def test_context_features_refusals():
    import ctypes
    import block_draft_model_dspark_b200 as dsp
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 84)
    proj = make_context_projection(m, 2, 11)
    x = make_target_hiddens(m, 2, 1, 8, 12).cuda()
    fc, g = proj["fc"].cuda(), proj["hidden_norm"].cuda()
    lib = dsp.get_lib()
    out = torch.empty(1, 8, m.hidden_size, dtype=model.torch_dtype, device="cuda")
    ws = model.workspace(lib.dspark_context_features_workspace_bytes(model.handle, 2, 8))
    mat = dsp.dspark_matrix()
    mat.w = fc.data_ptr()
    mat.scales = fc.data_ptr()                        # a 4-bit fc needs scales and biases
    rc = lib.dspark_project_context_features(model.handle, ctypes.byref(mat), g.data_ptr(), 2, x.data_ptr(), 1, 8,
                                             out.data_ptr(), ws.data_ptr(), ws.numel(), None)
    assert rc == dsp.DSPARK_ERR_INVALID_ARGUMENT
    mat.scales = None
    rc = lib.dspark_project_context_features(model.handle, ctypes.byref(mat), g.data_ptr(), 0, x.data_ptr(), 1, 8,
                                             out.data_ptr(), ws.data_ptr(), ws.numel(), None)
    assert rc == dsp.DSPARK_ERR_INVALID_ARGUMENT       # taps < 1
    rc = lib.dspark_project_context_features(model.handle, ctypes.byref(mat), g.data_ptr(), 2, x.data_ptr(), 1, 8,
                                             out.data_ptr() + 2, ws.data_ptr(), ws.numel(), None)
    assert rc == dsp.DSPARK_ERR_INVALID_ARGUMENT       # misaligned out
    rc = lib.dspark_project_context_features(model.handle, ctypes.byref(mat), g.data_ptr(), 2, x.data_ptr(), 1, 8,
                                             out.data_ptr(), ws.data_ptr(), 16, None)
    assert rc == dsp.DSPARK_ERR_WORKSPACE
    with pytest.raises(dsp.DsparkError):
        model.dspark_project_context_features(x[..., :-1], fc, g)   # last axis not taps * hidden
    torch.cuda.synchronize()
    assert model.dspark_read_device_status() == 0
