"""Seeded synthetic inputs shared by the CUDA path, the oracle tests and the bench.

This module holds no arithmetic of the DCU method itself: it only turns
(seed, tensor id, element index) into numbers.  The same definition is
implemented twice, here in numpy for the host and in ``csrc/gen.cu`` for the
device (``libdcugen.so``); a GPU test checks that both give identical bits.

Definition (all integer arithmetic is modulo 2**64):

* Stream base: ``base(seed, tid) = mix((seed << 32) ^ tid)``.
* Element hash: ``h(seed, tid, i) = mix(base + (i + 1) * GOLDEN)`` -- the
  ``i``-th output of a SplitMix64 generator started at ``base``
  (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
  OOPSLA 2014), whose finaliser ``mix`` is given below.
* Normal-like value: the four 16-bit lanes of ``h`` are summed
  (Irwin-Hall with n = 4, variance-matched):
  ``z = (S - 131070) * sqrt(3) / 65536`` with ``S = sum of the four lanes``;
  the value is ``std * z`` evaluated as ``(S - 131070) * scale`` with
  ``scale = (std * SQRT3) / 65536`` in IEEE binary64.  It needs no
  transcendental function, so host and device agree bit for bit.
* bf16 values are rounded from binary64 to nearest-even on the bit pattern
  (the 45 low mantissa bits are dropped); fp32 values by the IEEE conversion.
* Uniform integers in ``[0, n)``: ``((h >> 32) * n) >> 32`` (multiply-shift).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

GOLDEN = 0x9E3779B97F4A7C15
_M64 = (1 << 64) - 1
SQRT3 = 1.7320508075688772

# Tensor ids of the synthetic model and sequences.
TID_EMBED = 1
TID_LM_HEAD = 2
TID_PROMPT = 1000      # + sequence index
TID_UNMASK_POS = 2000  # + sequence index
TID_UNMASK_IDS = 3000  # + sequence index
LAYER_TENSORS = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down")


def layer_tid(layer: int, name: str) -> int:
    return 16 + 16 * layer + LAYER_TENSORS.index(name)


def _mix(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=False)
    z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def _mix_int(z: int) -> int:
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def stream_base(seed: int, tid: int) -> int:
    return _mix_int(((seed & 0xFFFFFFFF) << 32) ^ (tid & 0xFFFFFFFF))


def hashes(seed: int, tid: int, start: int, count: int) -> np.ndarray:
    base = np.uint64(stream_base(seed, tid))
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(base + i * np.uint64(GOLDEN))


def normal_f64(seed: int, tid: int, start: int, count: int, std: float) -> np.ndarray:
    h = hashes(seed, tid, start, count)
    m = np.uint64(0xFFFF)
    s = ((h & m) + ((h >> np.uint64(16)) & m) + ((h >> np.uint64(32)) & m)
         + ((h >> np.uint64(48)) & m)).astype(np.int64)
    scale = (float(std) * SQRT3) / 65536.0
    return (s - 131070).astype(np.float64) * scale


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round binary64 to bfloat16 (nearest, ties to even) on the bit pattern."""
    b = np.ascontiguousarray(x, dtype=np.float64).view(np.uint64)
    with np.errstate(over="ignore"):
        b = b + np.uint64((1 << 44) - 1) + ((b >> np.uint64(45)) & np.uint64(1))
    b = b & np.uint64(~((1 << 45) - 1) & _M64)
    f = b.view(np.float64).astype(np.float32)  # exact: value already has 8 significant bits
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_values(seed: int, tid: int, start: int, count: int, std: float, dtype: str) -> np.ndarray:
    """Seeded N(0, std)-like values, as uint16 bf16 bits ('bf16') or float32 ('f32')."""
    v = normal_f64(seed, tid, start, count, std)
    if dtype == "bf16":
        return f64_to_bf16_bits(v)
    if dtype == "f32":
        return v.astype(np.float32)
    raise ValueError(dtype)


def uniform_ints(seed: int, tid: int, start: int, count: int, n: int) -> np.ndarray:
    h = hashes(seed, tid, start, count)
    with np.errstate(over="ignore"):
        return (((h >> np.uint64(32)) * np.uint64(n)) >> np.uint64(32)).astype(np.int64)


# ---------------------------------------------------------------- model shapes

@dataclass(frozen=True)
class ModelShape:
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    d_ffn: int
    vocab: int
    dtype: str = "bf16"          # 'bf16' or 'f32'
    rms_eps: float = 1e-5
    rope_theta: float = 10000.0
    init_std: float = 0.02

    @property
    def mask_id(self) -> int:
        return self.vocab - 1

    def weight_shapes(self) -> dict:
        D, F, hd = self.d_model, self.d_ffn, self.head_dim
        return {"wq": (self.n_heads * hd, D), "wk": (self.n_kv_heads * hd, D),
                "wv": (self.n_kv_heads * hd, D), "wo": (D, self.n_heads * hd),
                "w_gate": (F, D), "w_up": (F, D), "w_down": (D, F)}


TOY = ModelShape(n_layers=4, d_model=256, n_heads=4, n_kv_heads=4, head_dim=64, d_ffn=1024,
                 vocab=1024, dtype="f32")
LLADA_8B = ModelShape(n_layers=32, d_model=4096, n_heads=32, n_kv_heads=32, head_dim=128,
                      d_ffn=12288, vocab=126464, dtype="bf16")
DREAM_7B = ModelShape(n_layers=28, d_model=3584, n_heads=28, n_kv_heads=4, head_dim=128,
                      d_ffn=18944, vocab=152064, dtype="bf16")


def weight_values(shape: ModelShape, seed: int, name: str, layer: int | None = None,
                  rows: np.ndarray | None = None) -> np.ndarray:
    """Host copy of one weight tensor (or selected rows of it) in its storage dtype.

    Row-major ``[out][in]``; ``embed`` and ``lm_head`` are ``[vocab][d_model]``.
    Norm gains are all ones and are not drawn.
    """
    if name in ("embed", "lm_head"):
        tid = TID_EMBED if name == "embed" else TID_LM_HEAD
        n_rows, n_cols = shape.vocab, shape.d_model
    else:
        tid = layer_tid(layer, name)
        n_rows, n_cols = shape.weight_shapes()[name]
    if rows is None:
        return normal_values(seed, tid, 0, n_rows * n_cols, shape.init_std, shape.dtype).reshape(n_rows, n_cols)
    out = [normal_values(seed, tid, int(r) * n_cols, n_cols, shape.init_std, shape.dtype) for r in rows]
    return np.stack(out) if out else np.zeros((0, n_cols), dtype=np.uint16 if shape.dtype == "bf16" else np.float32)


def weight_rows(shape: ModelShape, seed: int, name: str, row0: int, row1: int, layer: int | None = None,
                threads: int = 8) -> np.ndarray:
    """Rows [row0, row1) of a weight tensor in its storage dtype (generated in
    parallel chunks)."""
    from concurrent.futures import ThreadPoolExecutor
    if name in ("embed", "lm_head"):
        tid = TID_EMBED if name == "embed" else TID_LM_HEAD
        n_cols = shape.d_model
    else:
        tid = layer_tid(layer, name)
        n_cols = shape.weight_shapes()[name][1]
    step = max(1, (row1 - row0 + threads - 1) // threads)
    parts = [(r, min(row1, r + step)) for r in range(row0, row1, step)]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        out = list(ex.map(lambda ab: normal_values(seed, tid, ab[0] * n_cols, (ab[1] - ab[0]) * n_cols,
                                                    shape.init_std, shape.dtype), parts))
    return np.concatenate(out).reshape(row1 - row0, n_cols) if out else np.zeros((0, n_cols))


def as_f64(values: np.ndarray, dtype: str) -> np.ndarray:
    """Exact conversion of stored values (bf16 bits or float32) to float64."""
    if dtype == "bf16":
        return bf16_bits_to_f32(values).astype(np.float64)
    return values.astype(np.float64)


def prompt_ids(seed: int, b: int, n_prompt: int, vocab: int) -> np.ndarray:
    """Prompt token ids, uniform in [0, vocab - 1) (the last id is the mask id)."""
    return uniform_ints(seed, TID_PROMPT + b, 0, n_prompt, vocab - 1)


def sequence_ids(seed: int, b: int, n_prompt: int, n_gen: int, vocab: int) -> np.ndarray:
    ids = np.full(n_prompt + n_gen, vocab - 1, dtype=np.int64)
    ids[:n_prompt] = prompt_ids(seed, b, n_prompt, vocab)
    return ids


def unmask_draw(seed: int, b: int, gen_positions: np.ndarray, count: int, vocab: int):
    """Draw ``count`` positions without replacement from ``gen_positions`` (the
    ones with the smallest hashes) and new ids uniform in [0, vocab - 1)."""
    h = hashes(seed, TID_UNMASK_POS + b, 0, len(gen_positions))
    order = np.argsort(h, kind="stable")[:count]
    pos = np.sort(np.asarray(gen_positions)[order])
    new_ids = uniform_ints(seed, TID_UNMASK_IDS + b, 0, count, vocab - 1)
    return pos.astype(np.int64), new_ids


# ------------------------------------------------------- device generator binding

_GEN = None


def _gen_lib():
    global _GEN
    if _GEN is None:
        path = os.path.join(os.path.dirname(__file__), "libdcugen.so")
        if not os.path.exists(path):
            raise RuntimeError(f"device input generator not built: {path} (run __graft_entry__.build())")
        lib = ctypes.CDLL(path)
        lib.dcugen_normal.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32,
                                      ctypes.c_uint64, ctypes.c_double, ctypes.c_int32, ctypes.c_void_p]
        lib.dcugen_normal.restype = ctypes.c_int
        lib.dcugen_fill.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int32,
                                    ctypes.c_void_p]
        lib.dcugen_fill.restype = ctypes.c_int
        _GEN = lib
    return _GEN


def device_normal_(t, seed: int, tid: int, std: float, start: int = 0, stream=None):
    """Fill a CUDA tensor (bfloat16 or float32) with the seeded values in place."""
    import torch
    assert t.is_cuda and t.is_contiguous()
    dt = {torch.bfloat16: 0, torch.float32: 1}[t.dtype]
    s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    rc = _gen_lib().dcugen_normal(ctypes.c_void_p(t.data_ptr()), t.numel(), seed, tid, start, std, dt,
                                  ctypes.c_void_p(s))
    if rc != 0:
        raise RuntimeError(f"dcugen_normal failed ({rc})")
    return t


def device_fill_(t, value: float, stream=None):
    import torch
    assert t.is_cuda and t.is_contiguous()
    dt = {torch.bfloat16: 0, torch.float32: 1}[t.dtype]
    s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    rc = _gen_lib().dcugen_fill(ctypes.c_void_p(t.data_ptr()), t.numel(), value, dt, ctypes.c_void_p(s))
    if rc != 0:
        raise RuntimeError(f"dcugen_fill failed ({rc})")
    return t


def device_weights(shape: ModelShape, seed: int, device: str = "cuda") -> dict:
    """The seeded synthetic model on the device, in the layout of include/dcu.h
    (norm gains float32 ones), filled by the device generator."""
    import torch
    dt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32

    def rnd(tid, rows, cols):
        t = torch.empty((rows, cols), dtype=dt, device=device)
        return device_normal_(t, seed, tid, shape.init_std)

    def ones():
        return torch.ones(shape.d_model, dtype=torch.float32, device=device)

    ws = shape.weight_shapes()
    layers = []
    for l in range(shape.n_layers):
        lw = {"attn_norm": ones(), "ffn_norm": ones()}
        for name in LAYER_TENSORS:
            lw[name] = rnd(layer_tid(l, name), *ws[name])
        layers.append(lw)
    return {"embed": rnd(TID_EMBED, shape.vocab, shape.d_model),
            "lm_head": rnd(TID_LM_HEAD, shape.vocab, shape.d_model),
            "final_norm": ones(), "layers": layers}


def cfg_dict(shape: ModelShape, max_batch: int, max_seq: int, window_mode: int = 0) -> dict:
    return dict(n_layers=shape.n_layers, d_model=shape.d_model, n_heads=shape.n_heads, n_kv_heads=shape.n_kv_heads,
                head_dim=shape.head_dim, d_ffn=shape.d_ffn, vocab=shape.vocab, mask_id=shape.mask_id,
                max_batch=max_batch, max_seq=max_seq, dtype=shape.dtype, rms_eps=shape.rms_eps,
                rope_theta=shape.rope_theta, window_mode=window_mode)
