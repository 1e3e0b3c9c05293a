"""The C ABI without a GPU: the library loads, exports every symbol that
include/dspark.h declares, sizes its workspaces, and refuses the configs the
drafter page refuses (readConfig's guards) before touching any device memory."""
import ctypes
import re
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def dsp():
    from block_draft_model_dspark_b200 import build
    build.build()
    import block_draft_model_dspark_b200 as d
    d.get_lib()
    return d


def declared_functions():
    src = open(os.path.join(ROOT, "include", "dspark.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dspark_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol(dsp):
    names = declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(dsp.get_lib(), n), n
    assert set(names) == set(dsp._PROTOTYPES), "binding prototypes must match the header"


def _cfg(dsp, **kw):
    from synthetic import WORKLOADS
    c = dsp.make_config(WORKLOADS["single_bf16"].model)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_workspace_bytes_and_refusals(dsp):
    lib = dsp.get_lib()
    good = _cfg(dsp)
    n = lib.dspark_model_workspace_bytes(ctypes.byref(good))
    # fp16 copies of every round GEMM's weights ([Wq;Wk], [Wg;Wu], o_proj and down_proj per layer,
    # the lm-head), the all-layer k_proj in bf16; the pruned walk's |markov_w2| bounds (fp32 per
    # vocabulary entry); RoPE table, status and padding under 64 KB
    stacks = 2 * 3840 * (4 * (4608 + 30720 + 4096 + 15360) + 262144 + 4 * 512)
    norms = 4 * 262144
    assert stacks + norms <= n <= stacks + norms + (64 << 10)
    for bad in (dict(attention_k_eq_v=0), dict(markov_head_vanilla=0), dict(hidden_activation_gelu_tanh=0),
                dict(global_head_dim=100), dict(num_global_key_value_heads=3), dict(quant_bits=8),
                dict(mask_token_id=262144), dict(block_size=0)):
        c = _cfg(dsp, **bad)
        assert lib.dspark_model_workspace_bytes(ctypes.byref(c)) == 0, bad
        out = ctypes.c_void_p()
        w = dsp.dspark_weights()
        rc = lib.dspark_model_create(ctypes.byref(c), ctypes.byref(w), 256, 1 << 40, None, ctypes.byref(out))
        assert rc in (dsp.DSPARK_ERR_UNSUPPORTED, dsp.DSPARK_ERR_INVALID_ARGUMENT), bad
        assert lib.dspark_last_error().decode()
    c = _cfg(dsp, attention_k_eq_v=0)
    out = ctypes.c_void_p()
    rc = lib.dspark_model_create(ctypes.byref(c), ctypes.byref(dsp.dspark_weights()), 256, 1 << 40, None,
                                 ctypes.byref(out))
    assert rc == dsp.DSPARK_ERR_UNSUPPORTED and "v_proj" in lib.dspark_last_error().decode()


def test_null_arguments_are_rejected(dsp):
    lib = dsp.get_lib()
    assert lib.dspark_model_destroy(None) == dsp.DSPARK_ERR_INVALID_ARGUMENT
    assert lib.dspark_project_workspace_bytes(None, 10) == 0
    assert lib.dspark_draft_workspace_bytes(None, 1, 10) == 0
    st = ctypes.c_int32()
    assert lib.dspark_read_device_status(None, None, ctypes.byref(st)) == dsp.DSPARK_ERR_INVALID_ARGUMENT
    good = _cfg(dsp)
    out = ctypes.c_void_p()
    rc = lib.dspark_model_create(ctypes.byref(good), None, 256, 1 << 40, None, ctypes.byref(out))
    assert rc == dsp.DSPARK_ERR_INVALID_ARGUMENT


def test_binding_structs_match_the_header(dsp, tmp_path):
    """Every struct the binding passes by pointer has the header's size and field offsets
    (compiled with the host C compiler against include/dspark.h)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    structs = {"dspark_kv_cache": dsp.dspark_kv_cache, "dspark_config": dsp.dspark_config,
               "dspark_matrix": dsp.dspark_matrix, "dspark_layer_weights": dsp.dspark_layer_weights,
               "dspark_weights": dsp.dspark_weights}
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "dspark.h"', "int main(void) {"]
    for name, cls in structs.items():
        lines.append(f'  printf("{name} size %zu\\n", sizeof({name}));')
        for f, _ in cls._fields_:
            lines.append(f'  printf("{name} {f} %zu\\n", offsetof({name}, {f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {(p[0], p[1]): int(p[2]) for p in (l.split() for l in out) if len(p) == 3}
    for name, cls in structs.items():
        assert got[(name, "size")] == ctypes.sizeof(cls), name
        for f, _ in cls._fields_:
            assert got[(name, f)] == getattr(cls, f).offset, (name, f)
