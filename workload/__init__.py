"""Seeded synthetic workloads for the expert-parallel dispatch path.

Inputs only: router logits -> top-K ids and gate weights (the model's gate,
upstream of the EP layer), hidden rows x, the stand-in expert's per-expert
scale, and replica/home gradients.  Nothing here computes any step of the
method under test; the CPU oracle and the CUDA path both read what this
module writes.

The five workloads follow the MoE settings the source pages describe:
MoonEP's public benchmark defaults (S=8192, E=384, H=7168, K=8; the twodots.gr
MoonEP article, section on what the benchmarks show) at UltraEP's 64-rank
expert-parallel scale (the remio.ai UltraEP article), a DeepSeek-V3-shaped
layer (E=256, K=8, H=7168), a moderate 8-rank case, an adversarial prefill
case, and a tiny case.  Their skew recipes are stated per entry of CONFIGS.

Random numbers: Philox4x32-10 with key (seed, stream) and a sum-of-twelve-
uniforms normal; see gen.c.  Host (libgen.so) and device (libgen_dev.so)
produce bit-identical values.
"""
import ctypes
import os

import numpy as np

from . import build as _build

STREAM_LOGITS = 0x100  # + layer
STREAM_BIAS = 0x200    # + layer (per-layer bias redraw), else + 0
STREAM_X = 0x300       # + layer
STREAM_GHOME = 0x400
STREAM_GREP = 0x500

# name, R ranks, S tokens/rank, E experts, K top-k, H hidden, block_m, bias recipe,
# gradient elements per expert (n) and replica-gradient dtype, layers
CONFIGS = {
    1: dict(name="tiny", R=4, S=64, E=16, K=2, H=128, block_m=4, bias="zipf",
            grad_n=128, grad_dtype="f32", layers=1),
    2: dict(name="moderate_ep8", R=8, S=4096, E=64, K=6, H=2048, block_m=64, bias="normal_sigma0.5",
            grad_n=3 * 2048 * 1024, grad_dtype="f32", layers=1),
    3: dict(name="deepseek_v3_ep32", R=32, S=4096, E=256, K=8, H=7168, block_m=128, bias="lognormal_minus1",
            grad_n=3 * 7168 * 2048, grad_dtype="bf16", layers=1),
    4: dict(name="fine_grained_ep64_8layers", R=64, S=8192, E=384, K=8, H=7168, block_m=128,
            bias="normal_per_layer", grad_n=None, grad_dtype=None, layers=8),
    5: dict(name="adversarial_prefill_ep16", R=16, S=16384, E=256, K=8, H=4096, block_m=128, bias="hot0",
            grad_n=3 * 4096 * 1536, grad_dtype="f32", layers=1),
}


def shape(cfg):
    """Dict with T = R*S tokens, P = T*K pairs and the rest of cfg."""
    c = dict(CONFIGS[cfg]) if isinstance(cfg, int) else dict(cfg)
    c["T"] = c["R"] * c["S"]
    c["P"] = c["T"] * c["K"]
    return c


_lib = None
_dev = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build_host()
        L = ctypes.CDLL(path)
        L.gen_normal12_at.restype = ctypes.c_float
        L.gen_normal12_at.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64]
        L.gen_fill_normal_f32.restype = None
        L.gen_fill_normal_f32.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int64,
                                          ctypes.c_void_p, ctypes.c_int]
        L.gen_fill_normal_bf16.restype = None
        L.gen_fill_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int64,
                                           ctypes.c_void_p, ctypes.c_int]
        L.gen_routing.restype = None
        L.gen_routing.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_int]
        _lib = L
    return _lib


def dev_lib():
    global _dev
    if _dev is None:
        path = _build.build_device()
        L = ctypes.CDLL(path)
        for name in ("gen_dev_fill_normal_f32", "gen_dev_fill_normal_bf16"):
            f = getattr(L, name)
            f.restype = ctypes.c_int
            f.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p,
                          ctypes.c_void_p]
        _dev = L
    return _dev


def nthreads():
    return max(1, min(64, os.cpu_count() or 1))


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def normal_f32(seed, stream, offset, n, threads=None):
    out = np.empty(n, dtype=np.float32)
    lib().gen_fill_normal_f32(seed, stream, offset, n, _ptr(out), threads or nthreads())
    return out


def normal_bf16(seed, stream, offset, n, threads=None):
    """bf16 bit patterns (uint16)."""
    out = np.empty(n, dtype=np.uint16)
    lib().gen_fill_normal_bf16(seed, stream, offset, n, _ptr(out), threads or nthreads())
    return out


def bias(cfg, seed, layer=0, variant="default"):
    """Per-expert router bias b_e (fp32) of the workload's skew recipe."""
    c = shape(cfg)
    E = c["E"]
    kind = c["bias"]
    if variant in ("uniform",):
        return np.zeros(E, dtype=np.float32)
    if kind == "zipf":  # b_e = 1.2 * ln(1/(e+1))
        return np.array([1.2 * np.log(1.0 / (e + 1)) for e in range(E)], dtype=np.float32)
    if kind == "normal_sigma0.5":  # b_e ~ N(0, 0.5^2), drawn once per seed
        return (np.float32(0.5) * normal_f32(seed, STREAM_BIAS, 0, E)).astype(np.float32)
    if kind == "lognormal_minus1":  # b_e ~ lognormal(0, 1) - 1
        return (np.exp(normal_f32(seed, STREAM_BIAS, 0, E).astype(np.float64)) - 1.0).astype(np.float32)
    if kind == "normal_per_layer":  # b_e ~ N(0, 1), redrawn for every layer
        return normal_f32(seed, STREAM_BIAS + layer, 0, E)
    if kind == "hot0":  # b_0 = +4, the rest N(0, 1)
        b = normal_f32(seed, STREAM_BIAS, 0, E)
        b[0] = 4.0
        return b
    raise ValueError(kind)


def routing(cfg, seed, layer=0, variant="default"):
    """(topk_ids int32 [T,K], w fp32 [T,K]).

    variant: "default" -- logits = N(0,1) + b_e, top-K with ties to the lower id,
    w = softmax over the K chosen logits; "uniform" -- ids (t*K+k) mod E and w =
    softmax over N(0,1) logits at those ids; "single_expert" -- the default
    logits with logit[t,0] raised to (row max) + 1, so every token's top-1 is
    expert 0.
    """
    c = shape(cfg)
    T, E, K = c["T"], c["E"], c["K"]
    b = bias(c, seed, layer, variant)
    topk = np.empty((T, K), dtype=np.int32)
    w = np.empty((T, K), dtype=np.float32)
    lib().gen_routing(seed, STREAM_LOGITS + layer, T, E, K, _ptr(b), int(variant == "single_expert"),
                      int(variant == "uniform"), _ptr(topk), _ptr(w), nthreads())
    return topk, w


def routing_from(T, E, K, seed, bias_e=None, stream=STREAM_LOGITS, uniform=False, force_expert0=False):
    """Routing for an arbitrary (T, E, K) shape, for small test cases."""
    b = np.zeros(E, dtype=np.float32) if bias_e is None else np.ascontiguousarray(bias_e, dtype=np.float32)
    topk = np.empty((T, K), dtype=np.int32)
    w = np.empty((T, K), dtype=np.float32)
    lib().gen_routing(seed, stream, T, E, K, _ptr(b), int(force_expert0), int(uniform), _ptr(topk), _ptr(w),
                      nthreads())
    return topk, w


def hidden(T, H, seed, layer=0, t0=0, threads=None):
    """x rows [t0, t0+T) of a [*, H] bf16 hidden matrix, as uint16 bits."""
    return normal_bf16(seed, STREAM_X + layer, t0 * H, T * H, threads).reshape(T, H)


def hidden_rows(H, seed, layer, tokens):
    """x[tokens] (bf16 bits) without generating the whole matrix."""
    out = np.empty((len(tokens), H), dtype=np.uint16)
    for i, t in enumerate(tokens):
        lib().gen_fill_normal_bf16(seed, STREAM_X + layer, int(t) * H, H, _ptr(out[i]), 1)
    return out


def expert_scale(E):
    """Stand-in expert parameter s_e = 1 + e/E, in fp32."""
    e = np.arange(E, dtype=np.float32)
    return (np.float32(1.0) + e / np.float32(E)).astype(np.float32)


def grad_rows(seed, stream, n, rows, dtype="f32"):
    """rows x n gradient block; row r is normal12 at offset r*n."""
    if dtype == "f32":
        return normal_f32(seed, stream, 0, rows * n).reshape(rows, n)
    return normal_bf16(seed, stream, 0, rows * n).reshape(rows, n)


def grad_elements(seed, stream, n, row, cols, dtype="f32"):
    """Selected elements g[row, cols] of a gradient block (sampled checks)."""
    L = lib()
    vals = np.array([L.gen_normal12_at(seed, stream, int(row) * n + int(j)) for j in cols], dtype=np.float32)
    if dtype == "f32":
        return vals
    u = vals.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def fill_device(tensor, seed, stream, offset=0):
    """Fill a contiguous CUDA fp32 or bf16 tensor with normal12 values."""
    import torch
    L = dev_lib()
    st = torch.cuda.current_stream(tensor.device).cuda_stream
    n = tensor.numel()
    if tensor.dtype == torch.float32:
        rc = L.gen_dev_fill_normal_f32(seed, stream, offset, n, ctypes.c_void_p(tensor.data_ptr()),
                                       ctypes.c_void_p(st))
    elif tensor.dtype in (torch.bfloat16, torch.int16, torch.uint16):
        rc = L.gen_dev_fill_normal_bf16(seed, stream, offset, n, ctypes.c_void_p(tensor.data_ptr()),
                                        ctypes.c_void_p(st))
    else:
        raise TypeError(tensor.dtype)
    if rc != 0:
        raise RuntimeError(f"device generator failed: {rc}")
