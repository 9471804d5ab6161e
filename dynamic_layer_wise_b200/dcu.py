"""Thin Python binding of libdcu (``include/dcu.h``): argument marshalling only.

Every step of the DCU path runs in the CUDA kernels of ``libdcu.so``; this
module converts torch tensors to device pointers and raises ``DcuError`` on a
non-zero return code.  It fails loudly when the library is missing: there is
no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdcu.so")

# ---- constants mirrored from include/dcu.h
DCU_OK, DCU_EINVAL, DCU_ENOMEM, DCU_ECUDA, DCU_ECAPACITY, DCU_ESTATE, DCU_EDEVICE = 0, -1, -2, -3, -4, -5, -6
DCU_ST_BAD_KEY, DCU_ST_BAD_TOKEN, DCU_ST_TIMEOUT = 1, 2, 4
DCU_F32, DCU_BF16 = 0, 1
DCU_FRECHET, DCU_THRESHOLD, DCU_FACTOR, DCU_APD = 0, 1, 2, 3
DCU_WINDOW_INCLUSIVE, DCU_WINDOW_HALFOPEN = 0, 1
(DCU_T_H, DCU_T_K, DCU_T_V, DCU_T_D, DCU_T_S, DCU_T_S_PREV, DCU_T_BUDGET, DCU_T_SEL, DCU_T_SEL_COUNT,
 DCU_T_CONF, DCU_T_ARGMAX, DCU_T_ATTN, DCU_T_STALE, DCU_T_APD_TAU, DCU_T_APD_C, DCU_T_APD_H) = range(16)
DCU_SELECT_INPUT, DCU_SELECT_VALUE = 0, 1
DCU_OPT_FUSED_EPILOGUE, DCU_OPT_L2_PREFETCH, DCU_OPT_ATTENTION, DCU_OPT_GEMM_SMEM_KB = 1, 2, 3, 4
DCU_OPT_GEMM_PASS_SWEEP = 5
DCU_ATTN_TCGEN05, DCU_ATTN_MMA_SYNC = 0, 1
(DCU_K_REFRESH, DCU_K_BUDGET, DCU_K_SELECT, DCU_K_GATHER, DCU_K_GEMM, DCU_K_EPILOGUE, DCU_K_ATTN, DCU_K_SCATTER,
 DCU_K_LMHEAD, DCU_K_COMMIT, DCU_K_COUNT) = range(11)

_i32, _i64, _f32, _f64, _vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_void_p


class dcu_cfg(ctypes.Structure):
    _fields_ = [("n_layers", _i32), ("d_model", _i32), ("n_heads", _i32), ("n_kv_heads", _i32),
                ("head_dim", _i32), ("d_ffn", _i32), ("vocab", _i32), ("mask_id", _i32),
                ("max_batch", _i32), ("max_seq", _i32), ("dtype", _i32), ("rms_eps", _f32),
                ("rope_theta", _f32), ("window_mode", _i32)]


_PP = ctypes.POINTER(_vp)


class dcu_weights(ctypes.Structure):
    _fields_ = [("embed", _vp), ("final_norm", _vp), ("lm_head", _vp),
                ("attn_norm", _PP), ("wq", _PP), ("wk", _PP), ("wv", _PP), ("wo", _PP),
                ("ffn_norm", _PP), ("w_gate", _PP), ("w_up", _PP), ("w_down", _PP)]


class DcuError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libdcu error {code}: {msg}")
        self.code = code


_LIB = None

# name -> (restype, argtypes)
_SIGS = {
    "dcu_create": (_i32, [ctypes.POINTER(dcu_weights), ctypes.POINTER(dcu_cfg), ctypes.POINTER(_vp)]),
    "dcu_destroy": (None, [_vp]),
    "dcu_last_error": (ctypes.c_char_p, [_vp]),
    "dcu_full_forward": (_i32, [_vp, _vp, _i32, _i32, _vp]),
    "dcu_step": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _vp]),
    "commit_select": (_i32, [_vp, _i32, _f32, _vp, _vp, _vp, _vp, _vp]),
    "commit_select_block": (_i32, [_vp, _i32, _f32, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "dcu_status": (_i32, [_vp, _vp, ctypes.POINTER(_i32)]),
    "dcu_budget_split": (_i32, [_vp, _i32, _i32, _i32, _i32, _vp, _vp]),
    "dcu_select_tokens": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "dcu_cosine_distance": (_i32, [_vp, _vp, _vp, _i64, _i32, _i32, _vp, _vp]),
    "dcu_commit_rule": (_i32, [_i32, _f32, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp]),
    "dcu_commit_rule_block": (_i32, [_i32, _f32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp]),
    "dcu_selftest_wait_timeout": (_i32, [_vp, _vp]),
    "dcu_tensor_bytes": (_i32, [_vp, _i32, ctypes.POINTER(_i64)]),
    "dcu_get_tensor": (_i32, [_vp, _i32, _i32, _vp, _i64, _vp]),
    "dcu_set_tensor": (_i32, [_vp, _i32, _i32, _vp, _i64, _vp]),
    "dcu_profile_enable": (_i32, [_vp, _i32]),
    "dcu_profile_read": (_i32, [_vp, _i32, ctypes.POINTER(_f64), ctypes.POINTER(_i64), _i32]),
    "dcu_kernel_class_name": (ctypes.c_char_p, [_i32]),
    "dcu_launch_count": (_i64, [_vp]),
    "dcu_set_graphs": (_i32, [_vp, _i32]),
    "dcu_set_refresh": (_i32, [_vp, _i32, _i32, _i32]),
    "dcu_set_select_from": (_i32, [_vp, _i32]),
    "dcu_set_option": (_i32, [_vp, _i32, _i32]),
    "dcu_set_apd": (_i32, [_vp, _f32, _f32, _f32]),
    "dcu_linear": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp]),
    "dcu_lm_confidence_noalloc": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp]),
}


def lib():
    """Loads libdcu.so (raises if it is not built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run `python -m dynamic_layer_wise_b200.build` "
                               "(the DCU path has no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _err(handle) -> str:
    m = lib().dcu_last_error(handle)
    return m.decode() if m else ""


def _check(rc: int, handle=None):
    if rc != DCU_OK:
        raise DcuError(rc, _err(handle))


def _ptr(t) -> _vp:
    if t is None:
        return _vp(0)
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return _vp(t.data_ptr())


def _stream(stream) -> _vp:
    if stream is None:
        return _vp(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return _vp(stream.cuda_stream)
    return _vp(int(stream))


_LAYER_KEYS = ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down")


class Context:
    """Owns a dcu_ctx handle and keeps the weight tensors it points to alive."""

    def __init__(self, handle, weights, arrays, cfg: dict):
        self.handle = handle
        self._weights = weights
        self._arrays = arrays
        self.cfg = dict(cfg)

    def close(self):
        if self.handle:
            lib().dcu_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def dcu_create(weights: dict, cfg: dict) -> Context:
    """weights: {'embed', 'final_norm', 'lm_head', 'layers': [ {attn_norm, wq, ...}, ... ]} of CUDA
    tensors; cfg: the fields of dcu_cfg (dtype as 'bf16' | 'f32' or DCU_*)."""
    c = dict(cfg)
    if isinstance(c.get("dtype"), str):
        c["dtype"] = {"bf16": DCU_BF16, "f32": DCU_F32}[c["dtype"]]
    c.setdefault("mask_id", c["vocab"] - 1)
    c.setdefault("rms_eps", 1e-5)
    c.setdefault("rope_theta", 10000.0)
    c.setdefault("window_mode", DCU_WINDOW_INCLUSIVE)
    cs = dcu_cfg(**{k: c[k] for k, _ in dcu_cfg._fields_})
    L = c["n_layers"]
    layers = weights["layers"]
    if len(layers) != L:
        raise ValueError("weights['layers'] must have n_layers entries")
    arrays = {}
    for k in _LAYER_KEYS:
        arr = (_vp * L)(*[_ptr(layers[l][k]).value for l in range(L)])
        arrays[k] = arr
    w = dcu_weights(_ptr(weights["embed"]), _ptr(weights["final_norm"]), _ptr(weights["lm_head"]),
                    *[ctypes.cast(arrays[k], _PP) for k in _LAYER_KEYS])
    h = _vp(0)
    rc = lib().dcu_create(ctypes.byref(w), ctypes.byref(cs), ctypes.byref(h))
    _check(rc, None)
    return Context(h, weights, arrays, c)


def dcu_full_forward(ctx: Context, token_ids, stream=None):
    B, N = token_ids.shape
    assert token_ids.dtype == torch.int32
    _check(lib().dcu_full_forward(ctx.handle, _ptr(token_ids), B, N, _stream(stream)), ctx.handle)


def dcu_step(ctx: Context, token_ids, key_positions, n_keys, B_layer: int, B_window: int, stream=None):
    for t in (token_ids, key_positions, n_keys):
        assert t.dtype == torch.int32
    _check(lib().dcu_step(ctx.handle, _ptr(token_ids), _ptr(key_positions), _ptr(n_keys), int(B_layer),
                          int(B_window), _stream(stream)), ctx.handle)


def commit_select(ctx: Context, rule: int, param: float, masked, token_ids, out_positions, out_count, stream=None):
    assert masked.dtype == torch.uint8 and token_ids.dtype == torch.int32
    assert out_positions.dtype == torch.int32 and out_count.dtype == torch.int32
    _check(lib().commit_select(ctx.handle, int(rule), float(param), _ptr(masked), _ptr(token_ids),
                               _ptr(out_positions), _ptr(out_count), _stream(stream)), ctx.handle)


def commit_select_block(ctx: Context, rule: int, param: float, gen_start: int, block_len: int, masked, token_ids,
                        out_positions, out_count, stream=None):
    assert masked.dtype == torch.uint8 and token_ids.dtype == torch.int32
    assert out_positions.dtype == torch.int32 and out_count.dtype == torch.int32
    _check(lib().commit_select_block(ctx.handle, int(rule), float(param), int(gen_start), int(block_len),
                                     _ptr(masked), _ptr(token_ids), _ptr(out_positions), _ptr(out_count),
                                     _stream(stream)), ctx.handle)


def dcu_status(ctx: Context, stream=None) -> int:
    bits = _i32(0)
    rc = lib().dcu_status(ctx.handle, _stream(stream), ctypes.byref(bits))
    if rc not in (DCU_OK, DCU_EDEVICE):
        _check(rc, ctx.handle)
    return int(bits.value)


def dcu_budget_split(s_prev, B_layer: int, uniform: bool, budgets=None, stream=None):
    B, L = s_prev.shape
    if budgets is None:
        budgets = torch.empty((B, L), dtype=torch.int32, device=s_prev.device)
    _check(lib().dcu_budget_split(_ptr(s_prev), B, L, int(B_layer), int(bool(uniform)), _ptr(budgets),
                                  _stream(stream)))
    return budgets


def dcu_select_tokens(d, key_positions, n_keys, budgets, B_window: int, window_mode: int = 0, status=None,
                      stream=None):
    B, N = d.shape
    idx = torch.empty((B, N), dtype=torch.int32, device=d.device)
    count = torch.empty((B,), dtype=torch.int32, device=d.device)
    s = torch.empty((B,), dtype=torch.float32, device=d.device)
    _check(lib().dcu_select_tokens(_ptr(d), _ptr(key_positions), _ptr(n_keys), _ptr(budgets), B, N, int(B_window),
                                   int(window_mode), _ptr(idx), _ptr(count), _ptr(s), _ptr(status),
                                   _stream(stream)))
    return idx, count, s


def dcu_cosine_distance(x, y, gain, stream=None):
    rows, D = x.shape
    dt = {torch.bfloat16: DCU_BF16, torch.float32: DCU_F32}[x.dtype]
    d = torch.empty((rows,), dtype=torch.float32, device=x.device)
    _check(lib().dcu_cosine_distance(_ptr(x), _ptr(y), _ptr(gain), rows, D, dt, _ptr(d), _stream(stream)))
    return d


def dcu_commit_rule(rule: int, param: float, conf, argmax, masked, token_ids, out_positions, out_count, stream=None):
    B, N = conf.shape
    _check(lib().dcu_commit_rule(int(rule), float(param), _ptr(conf), _ptr(argmax), _ptr(masked), _ptr(token_ids),
                                 B, N, _ptr(out_positions), _ptr(out_count), _stream(stream)))


def dcu_commit_rule_block(rule: int, param: float, gen_start: int, block_len: int, conf, argmax, masked, token_ids,
                          out_positions, out_count, stream=None):
    B, N = conf.shape
    _check(lib().dcu_commit_rule_block(int(rule), float(param), int(gen_start), int(block_len), _ptr(conf),
                                       _ptr(argmax), _ptr(masked), _ptr(token_ids), B, N, _ptr(out_positions),
                                       _ptr(out_count), _stream(stream)))


def dcu_selftest_wait_timeout(status, stream=None):
    """One bounded device wait that must expire: sets DCU_ST_TIMEOUT in status."""
    assert status.dtype == torch.int32
    _check(lib().dcu_selftest_wait_timeout(_ptr(status), _stream(stream)))


_KIND_DTYPE = {DCU_T_D: torch.float32, DCU_T_S: torch.float32, DCU_T_S_PREV: torch.float32,
               DCU_T_BUDGET: torch.int32, DCU_T_SEL: torch.int32, DCU_T_SEL_COUNT: torch.int32,
               DCU_T_CONF: torch.float32, DCU_T_ARGMAX: torch.int32, DCU_T_STALE: torch.uint8,
               DCU_T_APD_TAU: torch.float32, DCU_T_APD_C: torch.float32, DCU_T_APD_H: torch.float32}


def _kind_dtype(ctx: Context, kind: int):
    if kind in (DCU_T_H, DCU_T_K, DCU_T_V, DCU_T_ATTN):
        return torch.bfloat16 if ctx.cfg["dtype"] == DCU_BF16 else torch.float32
    return _KIND_DTYPE[kind]


def dcu_get_tensor(ctx: Context, kind: int, layer: int = 0, stream=None):
    n = _i64(0)
    _check(lib().dcu_tensor_bytes(ctx.handle, kind, ctypes.byref(n)), ctx.handle)
    dt = _kind_dtype(ctx, kind)
    out = torch.empty(n.value // torch.tensor([], dtype=dt).element_size(), dtype=dt, device="cuda")
    _check(lib().dcu_get_tensor(ctx.handle, kind, layer, _ptr(out), n.value, _stream(stream)), ctx.handle)
    return out


def dcu_set_tensor(ctx: Context, kind: int, layer: int, src, stream=None):
    src = src.contiguous()
    _check(lib().dcu_set_tensor(ctx.handle, kind, layer, _ptr(src), src.numel() * src.element_size(),
                                _stream(stream)), ctx.handle)


def dcu_profile_enable(ctx: Context, max_launches: int):
    _check(lib().dcu_profile_enable(ctx.handle, int(max_launches)), ctx.handle)


def dcu_profile_read(ctx: Context, kernel_class: int, reset: bool = True):
    ms, n = _f64(0.0), _i64(0)
    _check(lib().dcu_profile_read(ctx.handle, kernel_class, ctypes.byref(ms), ctypes.byref(n), int(reset)),
           ctx.handle)
    return ms.value, n.value


def dcu_kernel_class_name(k: int) -> str:
    return lib().dcu_kernel_class_name(k).decode()


def dcu_launch_count(ctx: Context) -> int:
    return int(lib().dcu_launch_count(ctx.handle))


def dcu_lm_confidence_noalloc(h_rows, final_norm, lm_head, rms_eps: float = 1e-5, stream=None):
    """Confidence and argmax of final-layer rows with no device allocation by the
    library (the outputs are allocated here, by the caller side)."""
    m, D = h_rows.shape
    V = lm_head.shape[0]
    dt = {torch.bfloat16: DCU_BF16, torch.float32: DCU_F32}[h_rows.dtype]
    if lm_head.dtype != h_rows.dtype or lm_head.dim() != 2 or lm_head.shape[1] != D:
        raise ValueError("lm_head must be [V][D] in the dtype of h_rows")
    if final_norm.dtype != torch.float32 or final_norm.numel() != D:
        raise ValueError("final_norm must be float32 [D]")
    conf = torch.empty(m, dtype=torch.float32, device=h_rows.device)
    amax = torch.empty(m, dtype=torch.int32, device=h_rows.device)
    _check(lib().dcu_lm_confidence_noalloc(_ptr(h_rows), _ptr(final_norm), _ptr(lm_head), m, D, V, dt,
                                           float(rms_eps), _ptr(conf), _ptr(amax), _stream(stream)))
    return conf, amax


def dcu_linear(X, W, stream=None):
    """Y = X W^T in fp32 (X [M][K], W [Nout][K], bf16 or float32)."""
    M, K = X.shape
    Nout = W.shape[0]
    dt = {torch.bfloat16: DCU_BF16, torch.float32: DCU_F32}[X.dtype]
    Y = torch.empty((M, Nout), dtype=torch.float32, device=X.device)
    _check(lib().dcu_linear(_ptr(X), _ptr(W), M, K, Nout, dt, _ptr(Y), _stream(stream)))
    return Y


def dcu_set_graphs(ctx: Context, on: bool):
    _check(lib().dcu_set_graphs(ctx.handle, int(bool(on))), ctx.handle)


def dcu_set_refresh(ctx: Context, gen_start: int, prompt_interval: int, gen_interval: int):
    """Periodic full refresh of the prompt / generated positions (0 disables an interval)."""
    _check(lib().dcu_set_refresh(ctx.handle, int(gen_start), int(prompt_interval), int(gen_interval)), ctx.handle)


def dcu_set_select_from(ctx: Context, source: int):
    """DCU_SELECT_INPUT (layer-input distance, default) or DCU_SELECT_VALUE (Value distance)."""
    _check(lib().dcu_set_select_from(ctx.handle, int(source)), ctx.handle)


def dcu_set_option(ctx: Context, option: int, value: int):
    """Performance option of the context (DCU_OPT_FUSED_EPILOGUE, DCU_OPT_L2_PREFETCH, DCU_OPT_ATTENTION)."""
    _check(lib().dcu_set_option(ctx.handle, int(option), int(value)), ctx.handle)


def dcu_set_apd(ctx: Context, alpha: float, beta: float, tau0: float = 0.9):
    """Adaptive parallel decoding: enables rule DCU_APD with its alpha, beta and initial tau."""
    _check(lib().dcu_set_apd(ctx.handle, float(alpha), float(beta), float(tau0)), ctx.handle)
