"""Python binding of libdg.so, the C ABI declared in include/dg.h.

Argument marshalling only: every step of the denoising path runs in the CUDA
kernels of the library.  Importing works without a GPU (the tests check the
exported symbols on CPU); creating a context needs the built library and a
CUDA device and fails loudly otherwise — there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("DG_LIBRARY", os.path.join(HERE, "libdg.so"))
# the same library with per-CTA timeline records (select it with DG_LIBRARY)
TIMELINE_LIB_PATH = os.path.join(HERE, "libdg_timeline.so")

DG_OK = 0
STATUS = {0: "DG_OK", 1: "DG_ERR_INVALID_ARG", 2: "DG_ERR_OOM", 3: "DG_ERR_CAPACITY", 4: "DG_ERR_CUDA",
          5: "DG_ERR_DEVICE_TIMEOUT", 6: "DG_ERR_STATE", 7: "DG_ERR_UNSUPPORTED"}

# every function declared in include/dg.h
EXPORTS = ["dg_create", "dg_destroy", "dg_prefill", "dg_denoise_step", "dg_denoise_step_entropy",
           "dg_set_self_conditioning", "dg_debug_self_cond",
           "dg_denoise_step_host",
           "dg_commit_block", "dg_sync", "dg_cached_len", "dg_last_error", "dg_debug_capture",
           "dg_debug_hidden", "dg_debug_experts", "dg_debug_norm_rows", "dg_debug_lmhead", "dg_debug_router",
           "dg_debug_sample", "dg_debug_entropy_sample", "dg_debug_entropy", "dg_debug_wait_timeout",
           "dg_debug_gemm", "dg_debug_profile",
           "dg_debug_profile_read", "dg_debug_launch_count", "dg_debug_timeline_reset", "dg_debug_timeline",
           "dg_lmhead_argmax_static"]

# kernel ids of the timeline records (DG_K_* in dg.h)
TIMELINE_KERNELS = {10: "gemm_dense", 11: "gemm_moe", 13: "gemm_lmhead", 20: "attention", 21: "attn_merge", 30: "route_dispatch",
                    31: "combine_norm", 32: "embed_norm", 33: "residual_norm", 34: "reduce_splits",
                    35: "swiglu_splits", 36: "rope_qkv", 37: "lmhead_merge_sample", 38: "entropy_sample",
                    39: "router_topk", 40: "sample_only", 50: "other"}

# kernel classes of dg_debug_profile (DG_PROF_* in dg.h)
PROF_CLASSES = ["experts", "routing", "lm_head", "attention", "dense_proj", "other"]


class dg_config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("expert_hidden", ctypes.c_int32),
                ("shared_hidden", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("rope_base", ctypes.c_float), ("rms_eps", ctypes.c_float),
                ("temperature", ctypes.c_float), ("canvas", ctypes.c_int32),
                ("max_batch", ctypes.c_int32), ("max_seq", ctypes.c_int32),
                ("prefill_rows", ctypes.c_int32)]


LAYER_FIELDS = ["attn_norm", "wqkv", "wo", "ffn_norm", "w_router", "w_gate", "w_up", "w_down",
                "ws_gate", "ws_up", "ws_down"]


class dg_layer_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in LAYER_FIELDS]


class dg_weights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("final_norm", ctypes.c_void_p),
                ("router_bias", ctypes.c_void_p), ("layers", ctypes.POINTER(dg_layer_weights)),
                ("sc_gate", ctypes.c_void_p), ("sc_up", ctypes.c_void_p), ("sc_down", ctypes.c_void_p)]


class dg_timeline_record(ctypes.Structure):
    _fields_ = [("t0_ns", ctypes.c_uint64), ("t1_ns", ctypes.c_uint64), ("kernel", ctypes.c_int32),
                ("cta", ctypes.c_int32)]


class dg_entropy_args(ctypes.Structure):
    _fields_ = [("temperature", ctypes.c_float), ("gamma", ctypes.c_float), ("stop_entropy", ctypes.c_float)]


class DGError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libdg.so and declare its signatures (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run python -m block_discrete_diffusion_denoise_b200.build")
    lib = ctypes.CDLL(path)
    P, I32, I64, U64, F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float
    sig = {
        "dg_create": ([ctypes.POINTER(dg_config), ctypes.POINTER(dg_weights), P, ctypes.POINTER(P)], I32),
        "dg_destroy": ([P], I32),
        "dg_prefill": ([P, P, I32, I32], I32),
        "dg_denoise_step": ([P, P, I32, U64, F32, P, P, P], I32),
        "dg_denoise_step_host": ([P, P, I32, U64, F32, P, P, P], I32),
        "dg_denoise_step_entropy": ([P, P, I32, U64, ctypes.POINTER(dg_entropy_args), P, P, P, P, P], I32),
        "dg_debug_entropy_sample": ([P, P, P, P, I32, I32, U64, F32, F32, P, P], I32),
        "dg_debug_entropy": ([P, P], I32),
        "dg_set_self_conditioning": ([P, I32], I32),
        "dg_debug_self_cond": ([P, P], I32),
        "dg_commit_block": ([P, P], I32),
        "dg_sync": ([P], I32),
        "dg_cached_len": ([P], I32),
        "dg_last_error": ([P], ctypes.c_char_p),
        "dg_debug_capture": ([P, I32], I32),
        "dg_debug_hidden": ([P, I32, P], I32),
        "dg_debug_experts": ([P, I32, P], I32),
        "dg_debug_norm_rows": ([P, I32, P], I32),
        "dg_debug_lmhead": ([P, P, P, P, P], I32),
        "dg_debug_router": ([P, P, I32, P, P], I32),
        "dg_debug_sample": ([P, P, P, I32, I32, U64, F32, P], I32),
        "dg_debug_wait_timeout": ([P, U64], I32),
        "dg_debug_gemm": ([P, P, I32, I32, P, I32, I32, P], I32),
        "dg_debug_profile": ([P, I32], I32),
        "dg_debug_profile_read": ([P, I32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(I64)], I32),
        "dg_debug_launch_count": ([P], I64),
        "dg_debug_timeline_reset": ([P], I32),
        "dg_debug_timeline": ([P, P, I32, ctypes.POINTER(I64)], I32),
        "dg_lmhead_argmax_static": ([P, I32, I32, P, I32, F32, P, P, P, P], I32),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


DG_ERR_INVALID_ARG = 1


def _invalid(msg: str):
    raise DGError(DG_ERR_INVALID_ARG, msg)


def _check_tensor(t, dtype, n: int, what: str, device_type: str = "cuda", exact: bool = False,
                  optional: bool = False):
    """The checks a bare pointer cannot carry through the C ABI: t is a
    contiguous torch tensor of `dtype` on `device_type` holding at least (with
    exact, exactly) n elements.  The library reads or writes n elements at the
    address; a smaller, strided, misplaced or wrongly typed buffer would be
    read or written out of bounds or misread, so it is refused here
    (DG_ERR_INVALID_ARG) with nothing launched."""
    import torch
    if t is None:
        if optional:
            return
        _invalid(f"{what}: required")
    if not isinstance(t, torch.Tensor) or t.device.type != device_type or t.dtype != dtype \
            or not t.is_contiguous():
        _invalid(f"{what}: expected a contiguous {device_type} tensor of {dtype}, got "
                 f"{getattr(t, 'dtype', type(t).__name__)} on {getattr(t, 'device', '?')}"
                 f"{'' if getattr(t, 'is_contiguous', lambda: True)() else ' (strided)'}")
    if (t.numel() != n) if exact else (t.numel() < n):
        _invalid(f"{what}: {t.numel()} elements, {'expected' if exact else 'the call needs'} {n}")


def _check_host(a, dtype, n: int, what: str, optional: bool = False):
    """Host buffers of dg_denoise_step_host: a C-contiguous numpy array or a
    contiguous CPU tensor of `dtype` with at least n elements."""
    import numpy as np
    import torch
    if a is None:
        if optional:
            return
        _invalid(f"{what}: required")
    if isinstance(a, np.ndarray):
        if a.dtype != np.dtype(dtype) or not a.flags["C_CONTIGUOUS"] or a.size < n:
            _invalid(f"{what}: expected a C-contiguous {np.dtype(dtype)} array of at least {n} elements")
        return
    tdt = {np.int32: torch.int32, np.float32: torch.float32}[dtype]
    _check_tensor(a, tdt, n, what, device_type="cpu")


def weight_numels(cfg: dict) -> dict:
    """Element count of every weight tensor the C ABI reads for a dg_config
    (dg_weights / dg_layer_weights layouts of include/dg.h)."""
    d, E, F, Fs = cfg["d_model"], cfg["n_experts"], cfg["expert_hidden"], cfg["shared_hidden"]
    Hq, Hkv, D = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    return {
        "embed": cfg["vocab"] * d, "final_norm": d, "router_bias": E,
        "sc_gate": F * d, "sc_up": F * d, "sc_down": d * F,
        "layer": {"attn_norm": d, "wqkv": (Hq + 2 * Hkv) * D * d, "wo": d * Hq * D, "ffn_norm": d,
                  "w_router": E * d, "w_gate": E * F * d, "w_up": E * F * d, "w_down": E * d * F,
                  "ws_gate": Fs * d, "ws_up": Fs * d, "ws_down": d * Fs},
    }


def check_weights(cfg: dict, weights: dict, device_type: str = "cuda"):
    """Refuse (DG_ERR_INVALID_ARG) weights the library would read out of
    bounds or misread: every tensor contiguous on the device, bf16 (the router
    bias fp32), with the element count the configuration implies, one layer
    dict per layer; the self-conditioning weights all three or none."""
    import torch
    n = weight_numels(cfg)
    bf16 = torch.bfloat16
    _check_tensor(weights.get("embed"), bf16, n["embed"], "embed", device_type, exact=True)
    _check_tensor(weights.get("final_norm"), bf16, n["final_norm"], "final_norm", device_type, exact=True)
    _check_tensor(weights.get("router_bias"), torch.float32, n["router_bias"], "router_bias", device_type,
                  exact=True, optional=True)
    layers = weights.get("layers")
    if layers is None or len(layers) != cfg["n_layers"]:
        _invalid(f"layers: expected {cfg['n_layers']} layer dicts, got {None if layers is None else len(layers)}")
    for i, lw in enumerate(layers):
        for f in LAYER_FIELDS:
            _check_tensor(lw.get(f), bf16, n["layer"][f], f"layers[{i}].{f}", device_type, exact=True)
    sc = [weights.get(k) is not None for k in ("sc_gate", "sc_up", "sc_down")]
    if any(sc) and not all(sc):
        _invalid("self-conditioning weights: give sc_gate, sc_up and sc_down, or none")
    for k in ("sc_gate", "sc_up", "sc_down"):
        _check_tensor(weights.get(k), bf16, n[k], k, device_type, exact=True, optional=True)


class Context:
    """One dg_ctx.  `weights` holds torch CUDA tensors (bf16) named as in
    dg.h: embed, final_norm, router_bias (fp32 or None) and layers (list of
    dicts with the LAYER_FIELDS keys).  The tensors are referenced for the
    lifetime of the context.  Every call runs on `stream` (a cudaStream_t
    handle, e.g. torch.cuda.Stream().cuda_stream; None is the legacy default
    stream, on which steps are not captured into a graph): make inputs on it
    (torch.cuda.stream(...)) or make it wait for the stream that did."""

    # where the context's buffers must live (the tests of the argument checks
    # set "cpu" on an instance that never reaches the library)
    _device_type = "cuda"

    def __init__(self, cfg: dict, weights: dict, stream=None):
        self.lib = load_library()
        self._batch = None            # batch of the last successful prefill
        check_weights(cfg, weights, self._device_type)
        self._weights = weights
        c = dg_config()
        for name, _ in dg_config._fields_:
            setattr(c, name, cfg[name])
        self.cfg = dict(cfg)
        layers = (dg_layer_weights * cfg["n_layers"])()
        for i, lw in enumerate(weights["layers"]):
            for f in LAYER_FIELDS:
                setattr(layers[i], f, _ptr(lw[f]))
        w = dg_weights(embed=_ptr(weights["embed"]), final_norm=_ptr(weights["final_norm"]),
                       router_bias=_ptr(weights.get("router_bias")),
                       layers=ctypes.cast(layers, ctypes.POINTER(dg_layer_weights)),
                       sc_gate=_ptr(weights.get("sc_gate")), sc_up=_ptr(weights.get("sc_up")),
                       sc_down=_ptr(weights.get("sc_down")))
        self._layers_c = layers
        handle = ctypes.c_void_p()
        st = self.lib.dg_create(ctypes.byref(c), ctypes.byref(w), stream, ctypes.byref(handle))
        if st != DG_OK:
            raise DGError(st, "dg_create failed (check shape and weight alignment)")
        self.ctx = handle

    def _check(self, st):
        if st != DG_OK:
            raise DGError(st, self.lib.dg_last_error(self.ctx).decode())

    def close(self):
        if getattr(self, "ctx", None):
            self.lib.dg_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # --- the path ---
    # The library sees bare pointers; the buffers are checked here against the
    # sizes the call reads and writes (the batch of the last prefill times the
    # canvas), and a bad one raises DGError(DG_ERR_INVALID_ARG) with nothing
    # launched.  Before the first prefill the library itself refuses the call.
    def _n(self) -> int:
        return 0 if self._batch is None else self._batch * int(self.cfg["canvas"])

    def _dev(self, t, dtype, n, what, optional=False):
        _check_tensor(t, dtype, n, what, self._device_type, optional=optional)
        return _ptr(t)

    def prefill(self, tokens):
        import torch
        if getattr(tokens, "dim", lambda: 0)() != 2:
            _invalid("prefill: tokens must be a [batch, prefix_len] tensor")
        B, P = tokens.shape
        self._check(self.lib.dg_prefill(self.ctx, self._dev(tokens, torch.int32, B * P, "tokens"), B, P))
        self._batch = int(B)

    def denoise_step(self, canvas_in, step, seed, tau, canvas_out, conf, settled=None):
        import torch
        n, B = self._n(), self._batch or 0
        self._check(self.lib.dg_denoise_step(
            self.ctx, self._dev(canvas_in, torch.int32, n, "canvas_in"), int(step), int(seed), float(tau),
            self._dev(canvas_out, torch.int32, n, "canvas_out"), self._dev(conf, torch.float32, n, "conf"),
            self._dev(settled, torch.int32, B, "settled", optional=True)))

    def denoise_step_entropy(self, canvas_in, step, seed, temperature, gamma, stop_entropy, canvas_out,
                             prev_argmax=None, argmax_out=None, entropy=None, stopped=None):
        import torch
        n, B = self._n(), self._batch or 0
        a = dg_entropy_args(float(temperature), float(gamma), float(stop_entropy))
        self._check(self.lib.dg_denoise_step_entropy(
            self.ctx, self._dev(canvas_in, torch.int32, n, "canvas_in"), int(step), int(seed), ctypes.byref(a),
            self._dev(prev_argmax, torch.int32, n, "prev_argmax", optional=True),
            self._dev(argmax_out, torch.int32, n, "argmax_out", optional=True),
            self._dev(canvas_out, torch.int32, n, "canvas_out"),
            self._dev(entropy, torch.float32, n, "entropy", optional=True),
            self._dev(stopped, torch.int32, B, "stopped", optional=True)))

    def denoise_step_host(self, canvas_in, step, seed, tau, canvas_out, conf=None, settled=None):
        """Host-buffer variant: numpy int32/float32 arrays (or pinned CPU tensors)."""
        import numpy as np
        n, B = self._n(), self._batch or 0
        _check_host(canvas_in, np.int32, n, "canvas_in")
        _check_host(canvas_out, np.int32, n, "canvas_out")
        _check_host(conf, np.float32, n, "conf", optional=True)
        _check_host(settled, np.int32, B, "settled", optional=True)

        def hp(a):
            if a is None:
                return None
            return a.ctypes.data if hasattr(a, "ctypes") else a.data_ptr()
        self._check(self.lib.dg_denoise_step_host(self.ctx, hp(canvas_in), int(step), int(seed), float(tau),
                                                  hp(canvas_out), hp(conf), hp(settled)))

    def commit_block(self, block):
        import torch
        self._check(self.lib.dg_commit_block(self.ctx, self._dev(block, torch.int32, self._n(), "block")))

    def sync(self):
        self._check(self.lib.dg_sync(self.ctx))

    @property
    def cached_len(self) -> int:
        return self.lib.dg_cached_len(self.ctx)

    # --- test hooks ---
    def debug_capture(self, enable: bool):
        self._check(self.lib.dg_debug_capture(self.ctx, 1 if enable else 0))

    def debug_hidden(self, layer, out):
        self._check(self.lib.dg_debug_hidden(self.ctx, layer, _ptr(out)))

    def debug_experts(self, layer, out):
        self._check(self.lib.dg_debug_experts(self.ctx, layer, _ptr(out)))

    def debug_norm_rows(self, layer, out):
        self._check(self.lib.dg_debug_norm_rows(self.ctx, layer, _ptr(out)))

    def debug_lmhead(self, argmax=None, lse=None, conf=None, margin=None):
        self._check(self.lib.dg_debug_lmhead(self.ctx, _ptr(argmax), _ptr(lse), _ptr(conf), _ptr(margin)))

    def debug_router(self, logits, idx, gates):
        self._check(self.lib.dg_debug_router(self.ctx, _ptr(logits), logits.shape[0], _ptr(idx), _ptr(gates)))

    def debug_sample(self, argmax, conf, batch, step, seed, tau, out):
        self._check(self.lib.dg_debug_sample(self.ctx, _ptr(argmax), _ptr(conf), batch, int(step), int(seed),
                                             float(tau), _ptr(out)))

    def debug_entropy_sample(self, argmax, entropy, prev_argmax, batch, step, seed, gamma, stop_entropy, out,
                             stopped=None):
        self._check(self.lib.dg_debug_entropy_sample(self.ctx, _ptr(argmax), _ptr(entropy), _ptr(prev_argmax), batch,
                                                     int(step), int(seed), float(gamma), float(stop_entropy),
                                                     _ptr(out), _ptr(stopped)))

    def set_self_conditioning(self, enable: bool):
        self._check(self.lib.dg_set_self_conditioning(self.ctx, 1 if enable else 0))

    def debug_self_cond(self, out):
        self._check(self.lib.dg_debug_self_cond(self.ctx, _ptr(out)))

    def debug_entropy(self, out):
        self._check(self.lib.dg_debug_entropy(self.ctx, _ptr(out)))

    def debug_wait_timeout(self, limit_ns: int):
        self._check(self.lib.dg_debug_wait_timeout(self.ctx, int(limit_ns)))

    def debug_gemm(self, w, x, splits, out):
        M, K = w.shape
        self._check(self.lib.dg_debug_gemm(self.ctx, _ptr(w), M, K, _ptr(x), x.shape[0], int(splits), _ptr(out)))

    def debug_profile(self, classes=()):
        mask = 0
        for c in classes:
            mask |= 1 << (PROF_CLASSES.index(c) if isinstance(c, str) else int(c))
        self._check(self.lib.dg_debug_profile(self.ctx, mask))

    def debug_profile_read(self) -> dict:
        out = {}
        for i, name in enumerate(PROF_CLASSES):
            ms, n = ctypes.c_double(), ctypes.c_int64()
            self._check(self.lib.dg_debug_profile_read(self.ctx, i, ctypes.byref(ms), ctypes.byref(n)))
            out[name] = (ms.value, n.value)
        return out

    @property
    def launch_count(self) -> int:
        return self.lib.dg_debug_launch_count(self.ctx)

    def debug_timeline_reset(self):
        """Empty the timeline buffer (libdg_timeline.so only)."""
        self._check(self.lib.dg_debug_timeline_reset(self.ctx))

    def debug_timeline(self, capacity: int = 1 << 18):
        """Records appended since the last reset as a numpy structured array
        (t0_ns, t1_ns, kernel, cta), and how many were appended in all."""
        import numpy as np
        buf = (dg_timeline_record * capacity)()
        n = ctypes.c_int64()
        self._check(self.lib.dg_debug_timeline(self.ctx, buf, capacity, ctypes.byref(n)))
        dt = np.dtype([("t0_ns", "<u8"), ("t1_ns", "<u8"), ("kernel", "<i4"), ("cta", "<i4")])
        arr = np.frombuffer(buf, dtype=dt, count=min(n.value, capacity)).copy()
        return arr, n.value


def config_from_shape(shape, max_batch=1, max_seq=4096, canvas=256, temperature=1.0, prefill_rows=0) -> dict:
    """dg_config fields for a model shape (anything with the dg_config names)."""
    return dict(n_layers=shape.n_layers, d_model=shape.d_model, n_q_heads=shape.n_q_heads,
                n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim, n_experts=shape.n_experts,
                top_k=shape.top_k, expert_hidden=shape.expert_hidden, shared_hidden=shape.shared_hidden,
                vocab=shape.vocab, rope_base=shape.rope_base, rms_eps=shape.rms_eps,
                temperature=temperature, canvas=canvas, max_batch=max_batch, max_seq=max_seq,
                prefill_rows=prefill_rows)


def lmhead_argmax_static(z, embed, temperature, argmax=None, lse=None, conf=None, stream=None) -> int:
    """dg_lmhead_argmax_static on torch CUDA tensors; returns the dg_status
    code (0 = launched).  No device memory is allocated by the library.

    The library sees raw pointers and sizes only, so the tensors are checked
    here first and DG_ERR_INVALID_ARG (1) is returned, with nothing launched,
    when z or embed is not a contiguous bf16 CUDA matrix, their widths differ,
    or an output is not a contiguous CUDA tensor of its type (int32 argmax,
    float32 lse / conf) with at least one element per row of z."""
    import torch
    lib = load_library()

    def dense_cuda(t, dtype, ndim=None):
        return (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == dtype and t.is_contiguous()
                and (ndim is None or t.dim() == ndim))
    if not (dense_cuda(z, torch.bfloat16, 2) and dense_cuda(embed, torch.bfloat16, 2)):
        return 1
    n_rows, d = z.shape
    if embed.shape[1] != d or embed.device != z.device:
        return 1
    for t, dtype in ((argmax, torch.int32), (lse, torch.float32), (conf, torch.float32)):
        if t is not None and not (dense_cuda(t, dtype) and t.numel() >= n_rows and t.device == z.device):
            return 1
    return lib.dg_lmhead_argmax_static(_ptr(z), n_rows, d, _ptr(embed), embed.shape[0], float(temperature),
                                       _ptr(argmax), _ptr(lse), _ptr(conf), stream)


def anneal_temperature(step: int, max_steps: int = 48, t_first: float = 0.8, t_last: float = 0.4) -> float:
    """Temperature of step `step` of a block: linear from 0.8 at the first
    step to 0.4 at step max_steps - 1 (codemajin.net "DiffusionGemma
    architecture", section 3.3)."""
    if max_steps <= 1:
        return t_first
    return t_first + (t_last - t_first) * step / (max_steps - 1)


def generate_blocks(ctx: Context, prefix, init_canvas, n_blocks: int, max_steps: int, tau, seed: int,
                    commit_last: bool = False, before_step=None, after_step=None, entropy=None) -> dict:
    """Block-autoregressive generation through the C ABI (codemajin.net
    "DiffusionGemma architecture", section 3.2, block-AR; aibars.net, block
    commit): prefill the prompt causally, then for each block start from
    init_canvas(k) (an int32 CUDA tensor [batch, canvas], e.g. uniform noise),
    run up to max_steps denoising steps, stop as soon as every position of
    every sequence is settled (conf >= tau, read from the all-settled flags),
    and commit the block to the KV cache.  The last block is committed only
    with commit_last, matching the K - 1 commit forwards that codemajin.net
    section 5.1 counts in TPF.

    tau is a float or a function of the step index.  With entropy =
    {"gamma": ..., "stop_entropy": ...} the steps use the entropy-constrained
    sampler instead (dg_denoise_step_entropy) at the temperatures of
    anneal_temperature(step, max_steps), and a block ends when every sequence
    reports the adaptive stop (section 3.3).  before_step(k, s) and
    after_step(k, s, canvas_in, canvas_out, conf, settled) are optional hooks
    (tests use them to record a step; with the entropy sampler conf holds the
    entropies and settled the stop flags).  Host control only: every step of the
    path runs in the library's kernels; the one device-to-host read per step is
    the batch's all-settled flags.

    Returns {"blocks": [final canvas of each block], "steps": [steps taken per
    block], "settled": [whether each block stopped early]}."""
    import torch
    B, C = int(prefix.shape[0]), int(ctx.cfg["canvas"])
    ctx.prefill(prefix)
    out = {"blocks": [], "steps": [], "settled": []}
    for k in range(n_blocks):
        cur = init_canvas(k).to(torch.int32).contiguous()
        nxt = torch.empty_like(cur)
        conf = torch.empty(B, C, dtype=torch.float32, device=cur.device)
        settled = torch.empty(B, dtype=torch.int32, device=cur.device)
        argmax = torch.empty(B, C, dtype=torch.int32, device=cur.device)
        steps, done = 0, False
        for s in range(max_steps):
            if before_step is not None:
                before_step(k, s)
            if entropy is not None:
                ctx.denoise_step_entropy(cur, s, seed, anneal_temperature(s, max_steps), entropy["gamma"],
                                         entropy["stop_entropy"], nxt, prev_argmax=argmax if s > 0 else None,
                                         argmax_out=argmax, entropy=conf, stopped=settled)
            else:
                t = tau(s) if callable(tau) else tau
                ctx.denoise_step(cur, s, seed, t, nxt, conf, settled)
            if after_step is not None:
                after_step(k, s, cur, nxt, conf, settled)
            cur, nxt = nxt, cur
            steps += 1
            ctx.sync()                       # the flags are written on the context's stream
            if bool((settled.cpu() != 0).all()):
                done = True
                break
        out["blocks"].append(cur.clone())
        out["steps"].append(steps)
        out["settled"].append(done)
        if k + 1 < n_blocks or commit_last:
            ctx.commit_block(cur)
    return out


def timeline_launches(records):
    """Rebuild the launch sequence from timeline records: launches on one
    stream run one after another, so after sorting by start time a new launch
    begins wherever the kernel id changes or a CTA starts after every CTA so
    far has ended.  Returns a list of dicts {kernel, name, t0_ns, t1_ns, ctas}."""
    import numpy as np
    if len(records) == 0:
        return []
    r = records[np.argsort(records["t0_ns"], kind="stable")]
    out = []
    cur = None
    for t0, t1, k in zip(r["t0_ns"].tolist(), r["t1_ns"].tolist(), r["kernel"].tolist()):
        if cur is None or k != cur["kernel"] or t0 > cur["t1_ns"]:
            cur = {"kernel": k, "name": TIMELINE_KERNELS.get(k, str(k)), "t0_ns": t0, "t1_ns": t1, "ctas": 0}
            out.append(cur)
        cur["t1_ns"] = max(cur["t1_ns"], t1)
        cur["ctas"] += 1
    return out


def timeline_summary(launches) -> dict:
    """Per-kernel totals of a launch sequence: launches, summed span (us),
    mean span, share of the wall time, and the idle gaps before each kernel's
    launches; plus the wall time and the summed gaps."""
    if not launches:
        return {"wall_us": 0.0, "gaps_us": 0.0, "launches": 0, "kernels": {}}
    wall = (max(l["t1_ns"] for l in launches) - launches[0]["t0_ns"]) / 1e3
    kernels, gaps, prev_end = {}, 0.0, launches[0]["t0_ns"]
    for l in launches:
        gap = max(0.0, (l["t0_ns"] - prev_end) / 1e3)
        span = (l["t1_ns"] - l["t0_ns"]) / 1e3
        k = kernels.setdefault(l["name"], {"launches": 0, "total_us": 0.0, "gaps_before_us": 0.0})
        k["launches"] += 1
        k["total_us"] += span
        k["gaps_before_us"] += gap
        gaps += gap
        prev_end = max(prev_end, l["t1_ns"])
    for k in kernels.values():
        k["avg_us"] = k["total_us"] / k["launches"]
        k["share"] = k["total_us"] / wall if wall > 0 else 0.0
    return {"wall_us": wall, "gaps_us": gaps, "launches": len(launches), "kernels": kernels}
