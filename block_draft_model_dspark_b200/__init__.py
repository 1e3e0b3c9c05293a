"""Python binding of libdspark: the DSpark draft round on one B200.

Argument marshalling only. Every step of the round runs in libdspark.so's
CUDA kernels (see ``include/dspark.h``); PyTorch supplies device memory and
streams. There is no fallback path: the first call that needs the library
raises ImportError if libdspark.so is not built, and every call raises
``DsparkError`` on a non-zero status.

The ctypes functions carry the C names (``dspark_model_create``,
``dspark_project_context_kv``, ``dspark_append_context_kv``,
``dspark_draft_rows``, ``dspark_attend``, ...). ``DsparkModel`` and
``KvCache`` wrap them for torch tensors.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdspark.so")

DSPARK_OK = 0
DSPARK_ERR_INVALID_ARGUMENT = -1
DSPARK_ERR_UNSUPPORTED = -2
DSPARK_ERR_CAPACITY = -3
DSPARK_ERR_WORKSPACE = -4
DSPARK_ERR_CUDA = -5
DSPARK_ERR_DEVICE = -6
DSPARK_DEV_BAD_TOKEN = 1
DSPARK_DEV_BAD_LENGTH = 2
DSPARK_DEV_WAIT_TIMEOUT = 4
DSPARK_DEV_CAPACITY = 8
DSPARK_DEV_RANGE = 16
DSPARK_DTYPE_F32 = 0
DSPARK_DTYPE_BF16 = 1
DSPARK_DTYPE_F16 = 2

c_i32, c_f32, c_vp, c_size = ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
c_i32p = ctypes.POINTER(ctypes.c_int32)


class dspark_config(ctypes.Structure):
    _fields_ = [(n, c_i32) for n in (
        "hidden_size", "num_hidden_layers", "num_attention_heads", "global_head_dim",
        "num_global_key_value_heads", "intermediate_size", "vocab_size", "block_size", "mask_token_id",
        "markov_rank", "attention_k_eq_v", "markov_head_vanilla", "hidden_activation_gelu_tanh",
        "enable_confidence_head", "confidence_head_with_markov", "dtype", "quant_bits", "quant_group_size")] + \
        [(n, c_f32) for n in ("rope_theta", "partial_rotary_factor", "rms_norm_eps",
                              "final_logit_softcapping", "confidence_threshold")]


class dspark_matrix(ctypes.Structure):
    _fields_ = [("w", c_vp), ("scales", c_vp), ("biases", c_vp)]


class dspark_layer_weights(ctypes.Structure):
    _fields_ = [(n, dspark_matrix) for n in ("q_proj", "k_proj", "o_proj", "gate_proj", "up_proj", "down_proj")] + \
        [(n, c_vp) for n in ("q_norm", "k_norm", "input_layernorm", "post_attention_layernorm",
                             "pre_feedforward_layernorm", "post_feedforward_layernorm", "layer_scalar")]


class dspark_weights(ctypes.Structure):
    _fields_ = [("embed_tokens", dspark_matrix), ("lm_head", dspark_matrix), ("markov_w2", dspark_matrix),
                ("confidence_proj", dspark_matrix), ("markov_w1", c_vp), ("norm", c_vp),
                ("confidence_bias", c_vp), ("layers", ctypes.POINTER(dspark_layer_weights))]


class dspark_kv_cache(ctypes.Structure):
    _fields_ = [("k", c_vp), ("v", c_vp), ("len", c_i32p), ("len_host", c_i32p), ("batch", c_i32),
                ("capacity", c_i32), ("pos0", c_i32p)]


_PROTOTYPES = {
    "dspark_kv_dtype": (c_i32, [ctypes.POINTER(dspark_config)]),
    "dspark_model_workspace_bytes": (c_size, [ctypes.POINTER(dspark_config)]),
    "dspark_model_create": (c_i32, [ctypes.POINTER(dspark_config), ctypes.POINTER(dspark_weights), c_vp, c_size, c_vp,
                                    ctypes.POINTER(c_vp)]),
    "dspark_model_destroy": (c_i32, [c_vp]),
    "dspark_prune_lengths": (c_i32, [c_vp, c_i32, c_i32, c_vp, c_vp, c_vp]),
    "dspark_context_features_workspace_bytes": (c_size, [c_vp, c_i32, ctypes.c_int64]),
    "dspark_project_context_features": (c_i32, [c_vp, ctypes.POINTER(dspark_matrix), c_vp, c_i32, c_vp, c_i32, c_i32,
                                                c_vp, c_vp, c_size, c_vp]),
    "dspark_project_workspace_bytes": (c_size, [c_vp, ctypes.c_int64]),
    "dspark_project_context_kv": (c_i32, [c_vp, c_vp, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_size, c_vp]),
    "dspark_append_context_kv": (c_i32, [c_vp, c_vp, c_i32, c_vp, c_vp, ctypes.POINTER(dspark_kv_cache), c_vp,
                                         c_size, c_vp]),
    "dspark_draft_workspace_bytes": (c_size, [c_vp, c_i32, c_i32]),
    "dspark_draft_rows": (c_i32, [c_vp, ctypes.POINTER(dspark_kv_cache), c_vp, c_vp, c_i32, c_i32, c_vp, c_vp, c_vp,
                                  c_vp, c_vp, c_size, c_vp]),
    "dspark_attend": (c_i32, [c_vp, c_i32, ctypes.POINTER(dspark_kv_cache), c_vp, c_vp, c_vp, c_vp, c_i32, c_i32, c_vp,
                              c_size, c_vp]),
    "dspark_attend_no_alloc": (c_i32, [c_vp, c_i32, ctypes.POINTER(dspark_kv_cache), c_vp, c_vp, c_vp, c_vp, c_i32,
                                       c_i32, c_vp]),
    "dspark_debug_attention_dump": (c_i32, [c_vp, c_vp, c_size]),
    "dspark_debug_logit_stats": (c_i32, [c_vp, c_vp, c_size]),
    "dspark_debug_wait_probe": (c_i32, [c_vp, c_i32, c_vp]),
    "dspark_read_device_status": (c_i32, [c_vp, c_vp, c_i32p]),
    "dspark_last_error": (ctypes.c_char_p, []),
    "dspark_kernel_launches": (ctypes.c_uint64, []),
    "dspark_timer_enable": (c_i32, [c_i32]),
    "dspark_timer_read": (c_i32, [c_i32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64),
                                  ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]),
}

DSPARK_TIMER_KINDS = {"gemm_qk": 0, "lm_head": 1, "attention": 2, "walk": 3, "kv_project": 4, "rows": 5,
                      "gemm_o": 6, "gemm_gu": 7, "gemm_down": 8}


def dspark_kernel_launches() -> int:
    """Kernels libdspark has launched in this process."""
    return int(get_lib().dspark_kernel_launches())


def dspark_timer_enable(enable: bool) -> None:
    _check(get_lib().dspark_timer_enable(1 if enable else 0))


def dspark_timer_read(kind: str):
    """(device ms, launches, algorithmic bytes, flops) summed over the timed launches of a kernel class."""
    ms, n, by, fl = ctypes.c_double(), ctypes.c_int64(), ctypes.c_double(), ctypes.c_double()
    _check(get_lib().dspark_timer_read(DSPARK_TIMER_KINDS[kind], ctypes.byref(ms), ctypes.byref(n),
                                       ctypes.byref(by), ctypes.byref(fl)))
    return ms.value, n.value, by.value, fl.value


class DsparkError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libdspark error {code}: {msg}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m block_draft_model_dspark_b200.build` "
                          "(there is no non-CUDA path)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_LIB: Optional[ctypes.CDLL] = None


def get_lib() -> ctypes.CDLL:
    """The loaded libdspark.so (loads it on first use; raises if it is not built)."""
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):   # ``block_draft_model_dspark_b200.lib``
    if name == "lib":
        return get_lib()
    raise AttributeError(name)


def _check(rc: int) -> None:
    if rc != DSPARK_OK:
        raise DsparkError(rc, get_lib().dspark_last_error().decode())


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_ptr(stream) -> Optional[int]:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def make_config(shape) -> dspark_config:
    """A ``dspark_config`` from an object with the drafter's config.json attribute names."""
    c = dspark_config()
    for n in ("hidden_size", "num_hidden_layers", "num_attention_heads", "global_head_dim",
              "num_global_key_value_heads", "intermediate_size", "vocab_size", "block_size", "mask_token_id",
              "markov_rank"):
        setattr(c, n, int(getattr(shape, n)))
    c.attention_k_eq_v = 1 if getattr(shape, "attention_k_eq_v", True) else 0
    c.markov_head_vanilla = 1 if getattr(shape, "markov_head_type", "vanilla") == "vanilla" else 0
    c.hidden_activation_gelu_tanh = 1 if getattr(shape, "hidden_activation", "gelu_pytorch_tanh") == "gelu_pytorch_tanh" else 0
    c.enable_confidence_head = 1 if shape.enable_confidence_head else 0
    c.confidence_head_with_markov = 1 if shape.confidence_head_with_markov else 0
    c.dtype = DSPARK_DTYPE_F32 if shape.dtype == "fp32" else DSPARK_DTYPE_BF16
    c.quant_bits = int(getattr(shape, "quant_bits", 0))
    c.quant_group_size = int(getattr(shape, "quant_group_size", 64))
    c.rope_theta = float(shape.rope_theta)
    c.partial_rotary_factor = float(shape.partial_rotary_factor)
    c.rms_norm_eps = float(shape.rms_norm_eps)
    c.final_logit_softcapping = float(shape.final_logit_softcapping or 0.0)
    c.confidence_threshold = float(shape.confidence_threshold)
    return c


_MATS = ("q_proj", "k_proj", "o_proj", "gate_proj", "up_proj", "down_proj")
_GAINS = ("q_norm", "k_norm", "input_layernorm", "post_attention_layernorm", "pre_feedforward_layernorm",
          "post_feedforward_layernorm", "layer_scalar")


def _matrix(tensors: Dict, name: str) -> dspark_matrix:
    m = dspark_matrix()
    if name + ".q" in tensors:
        m.w, m.scales, m.biases = (tensors[name + ".q"].data_ptr(), tensors[name + ".scales"].data_ptr(),
                                   tensors[name + ".biases"].data_ptr())
    elif name in tensors:
        m.w = tensors[name].data_ptr()
    return m


def prune_lengths(conf, thresholds, lengths=None, stream=None):
    """Alg 1 draft-length pruning on the device (``dspark_prune_lengths``): the first position
    k >= 1 of each row with conf[b, k] < thresholds[k], else gamma. ``conf`` float32 [A, gamma],
    ``thresholds`` float32 [gamma], both CUDA tensors; returns int32 lengths [A]."""
    import torch
    A, gamma = int(conf.shape[0]), int(conf.shape[1])
    if lengths is None:
        lengths = torch.empty(A, dtype=torch.int32, device=conf.device)
    _check(get_lib().dspark_prune_lengths(conf.data_ptr(), A, gamma, thresholds.data_ptr(), lengths.data_ptr(),
                                          _stream_ptr(stream)))
    return lengths


class KvCache:
    """Caller-owned context K/V (``dspark_kv_cache``): k, v [Lyr, batch, capacity, nKv, hd] in the
    model's KV dtype (``dspark_kv_dtype``: fp16 for a bf16 model), len [batch].

    ``v_only=True`` keeps v alone (k is None; the attention rebuilds k = rope(v * k_norm) at the
    positions ``pos0[b] + t``): ``pos0`` is then the int32 device tensor [batch] of the absolute
    position of each batch row's cache row 0."""

    def __init__(self, model: "DsparkModel", batch: int, capacity: int, k=None, v=None, v_only: bool = False,
                 pos0=None):
        import torch
        s = model.shape
        shp = (s.num_hidden_layers, batch, capacity, s.num_global_key_value_heads, s.global_head_dim)
        self.v_only = bool(v_only)
        if self.v_only:
            self.k = None
        else:
            self.k = k if k is not None else torch.empty(shp, dtype=model.kv_torch_dtype, device=model.device)
        self.v = v if v is not None else torch.empty(shp, dtype=model.kv_torch_dtype, device=model.device)
        self.pos0 = pos0
        self.len = torch.zeros(batch, dtype=torch.int32, device=model.device)
        self.len_host = (ctypes.c_int32 * batch)()
        self.batch, self.capacity = batch, capacity

    def set_lengths(self, lengths: Sequence[int]) -> None:
        import torch
        for b, n in enumerate(lengths):
            self.len_host[b] = int(n)
        self.len.copy_(torch.tensor(list(lengths), dtype=torch.int32))

    def struct(self) -> dspark_kv_cache:
        c = dspark_kv_cache()
        c.k = self.k.data_ptr() if self.k is not None else None
        c.v = self.v.data_ptr()
        if self.pos0 is not None:
            c.pos0 = ctypes.cast(ctypes.c_void_p(self.pos0.data_ptr()), c_i32p)
        c.len = ctypes.cast(ctypes.c_void_p(self.len.data_ptr()), c_i32p)
        c.len_host = ctypes.cast(self.len_host, c_i32p)
        c.batch, c.capacity = self.batch, self.capacity
        return c


class DsparkModel:
    """A libdspark model over CUDA tensors named as the drafter checkpoint's modules.

    ``tensors`` maps ``embed_tokens``, ``lm_head``, ``norm``, ``markov_w1``,
    ``markov_w2``, ``confidence_proj``, ``confidence_bias`` and
    ``layers.{i}.{q_proj,k_proj,o_proj,gate_proj,up_proj,down_proj,q_norm,k_norm,
    input_layernorm,post_attention_layernorm,pre_feedforward_layernorm,
    post_feedforward_layernorm,layer_scalar}`` to CUDA tensors; a 4-bit
    matrix ``X`` is given as ``X.q`` / ``X.scales`` / ``X.biases``.
    """

    def __init__(self, shape, tensors: Dict, stream=None):
        import torch
        self.shape = shape
        self.tensors = tensors
        self.device = next(iter(tensors.values())).device
        self.torch_dtype = torch.float32 if shape.dtype == "fp32" else torch.bfloat16
        self.cfg = make_config(shape)
        kvd = get_lib().dspark_kv_dtype(ctypes.byref(self.cfg))
        if kvd < 0:
            raise DsparkError(DSPARK_ERR_UNSUPPORTED, "invalid config")
        # element type of caches, projected K/V and the attention seam's tensors
        self.kv_torch_dtype = {DSPARK_DTYPE_F32: torch.float32, DSPARK_DTYPE_F16: torch.float16}[kvd]
        L = shape.num_hidden_layers
        self._layers = (dspark_layer_weights * L)()
        for i in range(L):
            lw = self._layers[i]
            for n in _MATS:
                setattr(lw, n, _matrix(tensors, f"layers.{i}.{n}"))
            for n in _GAINS:
                setattr(lw, n, tensors[f"layers.{i}.{n}"].data_ptr())
        w = dspark_weights()
        w.embed_tokens = _matrix(tensors, "embed_tokens")
        w.lm_head = _matrix(tensors, "lm_head")
        w.markov_w2 = _matrix(tensors, "markov_w2")
        w.confidence_proj = _matrix(tensors, "confidence_proj")
        w.markov_w1 = _ptr(tensors.get("markov_w1"))
        w.norm = tensors["norm"].data_ptr()
        w.confidence_bias = _ptr(tensors.get("confidence_bias"))
        w.layers = self._layers
        self._weights = w
        lib = get_lib()
        nbytes = lib.dspark_model_workspace_bytes(ctypes.byref(self.cfg))
        if nbytes == 0:
            raise DsparkError(DSPARK_ERR_UNSUPPORTED, "invalid config")
        self.model_ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        h = c_vp()
        _check(lib.dspark_model_create(ctypes.byref(self.cfg), ctypes.byref(w), self.model_ws.data_ptr(), nbytes,
                                       _stream_ptr(stream), ctypes.byref(h)))
        self.handle = h

    def close(self) -> None:
        if getattr(self, "handle", None):
            get_lib().dspark_model_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- workspaces
    def workspace(self, nbytes: int):
        import torch
        return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=self.device)

    def project_workspace_bytes(self, rows: int) -> int:
        return get_lib().dspark_project_workspace_bytes(self.handle, rows)

    def draft_workspace_bytes(self, A: int, max_ctx_len: int) -> int:
        return get_lib().dspark_draft_workspace_bytes(self.handle, A, max_ctx_len)

    # -- the calls
    def dspark_project_context_features(self, target_hiddens, fc, hidden_norm, out=None, ws=None, stream=None):
        """The context hidden [B, L, H] from the target's tap hiddens [B, L, taps * H]
        (deepspec.ts #projectContext): rms(target_hiddens @ fc^T, hidden_norm). ``fc`` is a dense
        tensor [H, taps * H] in the model dtype, or a 4-bit affine triple (words, scales, biases)."""
        import torch
        B, L, KT = (int(x) for x in target_hiddens.shape)
        H = self.shape.hidden_size
        if KT % H:
            raise DsparkError(DSPARK_ERR_INVALID_ARGUMENT, "target_hiddens' last axis must be taps * hidden")
        taps = KT // H
        if out is None:
            out = torch.empty(B, L, H, dtype=self.torch_dtype, device=self.device)
        lib = get_lib()
        ws = ws if ws is not None else self.workspace(lib.dspark_context_features_workspace_bytes(self.handle, taps,
                                                                                              B * L))
        m = dspark_matrix()
        if isinstance(fc, (tuple, list)):
            m.w, m.scales, m.biases = (t.data_ptr() for t in fc)
        else:
            m.w = fc.data_ptr()
        _check(lib.dspark_project_context_features(self.handle, ctypes.byref(m), hidden_norm.data_ptr(), taps,
                                                   target_hiddens.data_ptr(), B, L, out.data_ptr(), ws.data_ptr(),
                                                   ws.numel(), _stream_ptr(stream)))
        return out

    def dspark_project_context_kv(self, hidden, k_out, v_out, pos0=None, static_pos: int = 0, ws=None, stream=None):
        B, L = int(hidden.shape[0]), int(hidden.shape[1])
        ws = ws if ws is not None else self.workspace(self.project_workspace_bytes(B * L))
        _check(get_lib().dspark_project_context_kv(self.handle, hidden.data_ptr(), B, L, static_pos, _ptr(pos0),
                                             _ptr(k_out), v_out.data_ptr(), ws.data_ptr(), ws.numel(),
                                             _stream_ptr(stream)))

    def dspark_append_context_kv(self, cache: KvCache, hidden, n_new, pos0, ws=None, stream=None):
        """Appends hidden[b, :n_new[b]] to row b of `cache`. ``n_new`` is an int32 tensor on the
        model's device (a sequence of ints is copied there first); the counts are validated on
        the device (a refused append sets DSPARK_DEV_CAPACITY in the device status)."""
        import torch
        B, Lnew = cache.batch, int(hidden.shape[1])
        if not torch.is_tensor(n_new):
            n_new = torch.tensor([int(x) for x in n_new], dtype=torch.int32).to(self.device, non_blocking=False)
        ws = ws if ws is not None else self.workspace(self.project_workspace_bytes(B * Lnew))
        st = cache.struct()
        _check(get_lib().dspark_append_context_kv(self.handle, hidden.data_ptr(), Lnew, n_new.data_ptr(), pos0.data_ptr(),
                                                  ctypes.byref(st), ws.data_ptr(), ws.numel(), _stream_ptr(stream)))

    def dspark_draft_rows(self, cache: KvCache, anchors, block_pos, max_ctx_len: int, tokens, lengths, conf=None,
                          base_logits=None, ws=None, stream=None):
        A = int(anchors.shape[0])
        ws = ws if ws is not None else self.workspace(self.draft_workspace_bytes(A, max_ctx_len))
        st = cache.struct()
        _check(get_lib().dspark_draft_rows(self.handle, ctypes.byref(st), anchors.data_ptr(), block_pos.data_ptr(), A,
                                     max_ctx_len, tokens.data_ptr(), _ptr(conf), lengths.data_ptr(), _ptr(base_logits),
                                     ws.data_ptr(), ws.numel(), _stream_ptr(stream)))

    def dspark_attend(self, layer: int, cache: KvCache, q, k_blk, v_blk, out, max_ctx_len: int, ws=None, stream=None):
        A = int(q.shape[0])
        ws = ws if ws is not None else self.workspace(self.draft_workspace_bytes(A, max_ctx_len))
        st = cache.struct()
        _check(get_lib().dspark_attend(self.handle, layer, ctypes.byref(st), q.data_ptr(), k_blk.data_ptr(),
                                 v_blk.data_ptr(), out.data_ptr(), A, max_ctx_len, ws.data_ptr(), ws.numel(),
                                 _stream_ptr(stream)))

    def dspark_attend_no_alloc(self, layer: int, cache: KvCache, q, k_blk, v_blk, out, max_ctx_len: int,
                               stream=None):
        """The attention seam with the library's static scratch: no workspace tensor is passed."""
        A = int(q.shape[0])
        st = cache.struct()
        _check(get_lib().dspark_attend_no_alloc(self.handle, layer, ctypes.byref(st), q.data_ptr(), k_blk.data_ptr(),
                                                v_blk.data_ptr(), out.data_ptr(), A, max_ctx_len, _stream_ptr(stream)))

    def dspark_debug_attention_dump(self, dst) -> None:
        """Per-layer attention outputs of later rounds into `dst` (fp32 CUDA tensor
        [layers, A, gamma, nH, hd]); None turns the dump off."""
        _check(get_lib().dspark_debug_attention_dump(self.handle, _ptr(dst),
                                                     0 if dst is None else dst.numel() * dst.element_size()))

    def dspark_debug_logit_stats(self, dst) -> None:
        """Per-position logit statistics of later rounds into `dst` (a CUDA tensor of
        A * gamma * 16 bytes: float max, float logsumexp, int32 argmax, int32 candidates);
        None turns the dump off."""
        _check(get_lib().dspark_debug_logit_stats(self.handle, _ptr(dst),
                                                  0 if dst is None else dst.numel() * dst.element_size()))

    def dspark_debug_wait_probe(self, limit_us: int, stream=None) -> None:
        """Enqueues a bounded device wait that nothing satisfies (it gives up after limit_us)."""
        _check(get_lib().dspark_debug_wait_probe(self.handle, int(limit_us), _stream_ptr(stream)))

    def dspark_read_device_status(self, stream=None) -> int:
        v = ctypes.c_int32(0)
        _check(get_lib().dspark_read_device_status(self.handle, _stream_ptr(stream), ctypes.byref(v)))
        return int(v.value)

    # -- convenience: one round with fresh output tensors
    def draft(self, cache: KvCache, anchors, block_pos, max_ctx_len: int, collect_logits: bool = True, stream=None):
        import torch
        A, G, V = int(anchors.shape[0]), self.shape.block_size, self.shape.vocab_size
        dev = self.device
        out = {"tokens": torch.empty(A, G, dtype=torch.int32, device=dev),
               "lengths": torch.empty(A, dtype=torch.int32, device=dev),
               "conf": torch.empty(A, G, dtype=torch.float32, device=dev) if self.shape.enable_confidence_head else None,
               "base_logits": torch.empty(A, G, V, dtype=torch.float32, device=dev) if collect_logits else None}
        self.dspark_draft_rows(cache, anchors, block_pos, max_ctx_len, out["tokens"], out["lengths"], out["conf"],
                               out["base_logits"], stream=stream)
        return out
