"""Seeded synthetic inputs for the HGA attention layer.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark.  It holds no step of the method itself: it only draws numbers and
rounds them to the storage type.

Recipe (one counter-based generator, defined here so both sides see the same
bytes):

* splitmix64: the n-th output (n = 0, 1, ...) of a generator seeded with
  ``key`` is ``mix(key + (n + 1) * 0x9E3779B97F4A7C15)`` where ``mix`` is the
  splitmix64 finaliser (xor-shift 30, multiply 0xBF58476D1CE4E5B9, xor-shift 27,
  multiply 0x94D049BB133111EB, xor-shift 31), all modulo 2**64.
* A uniform in (0, 1) is ``((r >> 11) + 0.5) * 2**-53``.
* A standard normal for logical element n is Box-Muller on the uniforms of
  outputs 2n and 2n+1: ``sqrt(-2 ln u0) * cos(2 pi u1)``.
* Every tensor has its own stream key ``mix(seed * 0x9E3779B97F4A7C15 + tag)``
  with the tags below, and element n is its row-major flat index in the
  *whole-sequence* tensor, so any slice (one segment, one head) can be drawn
  on its own and agrees with the full draw.
* Keys get a per-chunk offset: for each (batch, kv head, 64-token chunk) a
  vector u ~ N(0, I_D) (stream OFFSET, flat index over [B][Hkv][L/c][D]) is
  scaled to norm 2 and added to every key of that chunk.
* Values are computed in float64, rounded to float32 (nearest-even) and, for
  bf16 workloads, to bfloat16 (nearest-even).  Both sides receive exactly
  these numbers.

The five workloads are the ones the HGA layer is measured on: a tiny fp32
case and Qwen3-8B-shaped layers (32 query heads, 8 KV heads, head_dim 128) at
16K and 128K tokens of context.
"""
from __future__ import annotations

import dataclasses
import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
M1 = np.uint64(0xBF58476D1CE4E5B9)
M2 = np.uint64(0x94D049BB133111EB)

TAG_Q, TAG_K, TAG_V, TAG_DO, TAG_OFFSET = 1, 2, 3, 4, 5


def _mix(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    z ^= z >> np.uint64(30)
    z *= M1
    z ^= z >> np.uint64(27)
    z *= M2
    z ^= z >> np.uint64(31)
    return z


def stream_key(seed: int, tag: int) -> np.uint64:
    with np.errstate(over="ignore"):
        base = np.array([seed], dtype=np.uint64) * GAMMA + np.uint64(tag)
    return _mix(base)[0]


def splitmix_outputs(key: np.uint64, n: np.ndarray) -> np.ndarray:
    """n-th outputs (uint64) of the splitmix64 generator seeded with key."""
    with np.errstate(over="ignore"):
        x = key + (n.astype(np.uint64) + np.uint64(1)) * GAMMA
    return _mix(x)


def _uniform(r: np.ndarray) -> np.ndarray:
    return ((r >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normals(key: np.uint64, flat_index: np.ndarray) -> np.ndarray:
    """Standard normals (float64) for the given logical element indices."""
    n = flat_index.astype(np.uint64)
    u0 = _uniform(splitmix_outputs(key, n * np.uint64(2)))
    u1 = _uniform(splitmix_outputs(key, n * np.uint64(2) + np.uint64(1)))
    return np.sqrt(-2.0 * np.log(u0)) * np.cos(2.0 * np.pi * u1)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float64/float32 -> float32 holding the nearest-even bfloat16 value."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> np.uint64(16)) & np.uint64(1)
    rounded = (bits + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    out = (rounded << np.uint64(16)).astype(np.uint32)
    return out.view(np.float32)


def bf16_bits(x_f32: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are already bf16-exact."""
    return (np.ascontiguousarray(x_f32, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one HGA attention layer workload.

    ``seg_starts`` lists the history length T at which each processed segment
    begins; the layer's whole sequence is ``seq_len`` tokens.
    """
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    chunk: int
    q_block: int
    topk: int
    seg_len: int
    seq_len: int
    seg_starts: tuple
    dtype: str  # "fp32" or "bf16"
    seed: int
    backward: bool = False
    tiered: bool = False
    sink_chunks: int = 0  # attention-sink window: history chunks always routed
    decode: bool = False  # one new token per sequence; seg_len is then its local window

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


def _segs(first_t: int, seg: int, n: int) -> tuple:
    return tuple(first_t + s * seg for s in range(n))


WORKLOADS = {
    # tiny fp32 layer: 2 q heads / 1 kv head, D 64, T 1024 + S 256, k 4
    "tiny_fp32": Workload("tiny_fp32", 1, 2, 1, 64, 64, 64, 4, 256, 1280, (1024,), "fp32", 0),
    # Qwen3-8B-shaped layer at 16K context, forward of the last 2,048-token segment
    "qwen3_16k_fwd": Workload("qwen3_16k_fwd", 1, 32, 8, 128, 64, 64, 16, 2048, 16384, (14336,), "bf16", 1),
    # the same layer trained segment-wise: 8 consecutive 2,048-token segments
    "qwen3_16k_train": Workload("qwen3_16k_train", 1, 32, 8, 128, 64, 64, 16, 2048, 16384,
                                _segs(0, 2048, 8), "bf16", 2, backward=True),
    # 131,072-token evaluation forward as 32 segments of 4,096 tokens, k 32
    "qwen3_128k_eval": Workload("qwen3_128k_eval", 1, 32, 8, 128, 64, 64, 32, 4096, 131072,
                                _segs(0, 4096, 32), "bf16", 3),
    # the same evaluation with detached history K/V in pinned host memory
    "qwen3_128k_tiered": Workload("qwen3_128k_tiered", 1, 32, 8, 128, 64, 64, 32, 4096, 131072,
                                  _segs(0, 4096, 32), "bf16", 3, tiered=True),
    # decode at 128K context: 16 sequences, each adds one token after 131,008 detached history
    # tokens and closes a 64-token local window; top-32 chunks
    "qwen3_128k_decode": Workload("qwen3_128k_decode", 16, 32, 8, 128, 64, 64, 32, 64, 131072, (131008,),
                                  "bf16", 4, decode=True),
    # the same decode at 32K context (same grid and routed-chunk count; 2.1 GB of K/V on the
    # device, the size used for counter captures)
    "qwen3_32k_decode": Workload("qwen3_32k_decode", 16, 32, 8, 128, 64, 64, 32, 64, 32768, (32704,),
                                 "bf16", 4, decode=True),
    # the 16K forward with a one-chunk attention-sink window (chunk 0 always routed)
    "qwen3_16k_fwd_sink": Workload("qwen3_16k_fwd_sink", 1, 32, 8, 128, 64, 64, 16, 2048, 16384, (14336,),
                                   "bf16", 1, sink_chunks=1),
}


def _finish(x: np.ndarray, dtype: str) -> np.ndarray:
    x32 = x.astype(np.float32)
    return round_bf16(x32) if dtype == "bf16" else x32


def draw(seed: int, tag: int, shape_full: tuple, t_axis_slice: slice | None = None,
         t_axis: int = 2) -> np.ndarray:
    """Standard normals of a [*, *, L, D]-shaped logical tensor, optionally one token slice."""
    key = stream_key(seed, tag)
    dims = list(shape_full)
    t0, t1 = 0, dims[t_axis]
    if t_axis_slice is not None:
        t0, t1 = t_axis_slice.start, t_axis_slice.stop
    idx_axes = [np.arange(d, dtype=np.int64) for d in dims]
    idx_axes[t_axis] = np.arange(t0, t1, dtype=np.int64)
    strides = np.cumprod([1] + dims[::-1][:-1])[::-1]
    flat = np.zeros([len(a) for a in idx_axes], dtype=np.int64)
    for ax, (a, st) in enumerate(zip(idx_axes, strides)):
        shape = [1] * len(dims)
        shape[ax] = len(a)
        flat = flat + (a * int(st)).reshape(shape)
    return normals(key, flat)


def chunk_offsets(w: Workload, chunk_lo: int, chunk_hi: int) -> np.ndarray:
    """Per-chunk key offsets of norm 2, shape [B][Hkv][chunk_hi-chunk_lo][D] (float64)."""
    n_chunks = w.seq_len // w.chunk
    u = draw(w.seed, TAG_OFFSET, (w.batch, w.n_kv_heads, n_chunks, w.head_dim),
             slice(chunk_lo, chunk_hi))
    return 2.0 * u / np.linalg.norm(u, axis=-1, keepdims=True)


PIECE = 2048  # tokens drawn per piece, to bound host memory on long sequences


def _pieces(fn, t0: int, t1: int) -> np.ndarray:
    parts = [fn(a, min(a + PIECE, t1)) for a in range(t0, t1, PIECE)]
    if not parts:
        return fn(t0, t0)
    return parts[0] if len(parts) == 1 else np.concatenate(parts, axis=2)


def keys(w: Workload, t0: int, t1: int) -> np.ndarray:
    """Keys for tokens [t0, t1) of the whole sequence, [B][Hkv][t1-t0][D] float32."""
    c = w.chunk
    assert t0 % c == 0 and t1 % c == 0

    def piece(a, b):
        k = draw(w.seed, TAG_K, (w.batch, w.n_kv_heads, w.seq_len, w.head_dim), slice(a, b))
        off = chunk_offsets(w, a // c, b // c)
        return _finish(k + np.repeat(off, c, axis=2), w.dtype)
    return _pieces(piece, t0, t1)


def values(w: Workload, t0: int, t1: int) -> np.ndarray:
    return _pieces(lambda a, b: _finish(draw(w.seed, TAG_V, (w.batch, w.n_kv_heads, w.seq_len,
                                                            w.head_dim), slice(a, b)), w.dtype), t0, t1)


def queries(w: Workload, t0: int, t1: int) -> np.ndarray:
    return _pieces(lambda a, b: _finish(draw(w.seed, TAG_Q, (w.batch, w.n_q_heads, w.seq_len,
                                                            w.head_dim), slice(a, b)), w.dtype), t0, t1)


def grad_out(w: Workload, t0: int, t1: int) -> np.ndarray:
    return _pieces(lambda a, b: _finish(draw(w.seed, TAG_DO, (w.batch, w.n_q_heads, w.seq_len,
                                                             w.head_dim), slice(a, b)), w.dtype), t0, t1)


def custom(name: str, **kw) -> Workload:
    """A smaller workload with the same recipe (used for fast parity sweeps)."""
    base = dict(batch=1, n_q_heads=2, n_kv_heads=1, head_dim=64, chunk=64, q_block=64, topk=4,
                seg_len=256, seq_len=1280, seg_starts=(1024,), dtype="fp32", seed=0)
    base.update(kw)
    return Workload(name=name, **base)


# ---------------------------------------------------------------------------
# The same recipe drawn with torch (int64 arithmetic wraps modulo 2**64), so a
# benchmark can draw long sequences directly on the GPU.  Logical right shifts
# are arithmetic shifts with the sign-extended top bits masked off.  float64
# log/cos may differ from numpy's in the last bit, which almost never survives
# the rounding to float32/bf16.

def _to_i64(u: int) -> int:
    return u - (1 << 64) if u >= (1 << 63) else u


_GAMMA_I = _to_i64(0x9E3779B97F4A7C15)
_M1_I = _to_i64(0xBF58476D1CE4E5B9)
_M2_I = _to_i64(0x94D049BB133111EB)


def _shr(z, k: int):
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix_t(z):
    z = z ^ _shr(z, 30)
    z = z * _M1_I
    z = z ^ _shr(z, 27)
    z = z * _M2_I
    return z ^ _shr(z, 31)


def draw_torch(seed: int, tag: int, shape_full: tuple, t0: int, t1: int, device):
    """torch (float64) version of ``draw`` for tokens [t0, t1) of axis 2."""
    import torch
    key = _to_i64(int(stream_key(seed, tag)))
    dims = list(shape_full)
    strides = [int(s) for s in np.cumprod([1] + dims[::-1][:-1])[::-1]]
    ar = lambda n, s, ax: (torch.arange(n[0], n[1], device=device, dtype=torch.int64) * s).reshape(
        [-1 if a == ax else 1 for a in range(len(dims))])
    flat = ar((0, dims[0]), strides[0], 0) + ar((0, dims[1]), strides[1], 1) + ar((t0, t1), strides[2], 2) + \
        ar((0, dims[3]), strides[3], 3)
    n2 = flat * 2

    def uni(n):
        r = _mix_t(key + (n + 1) * _GAMMA_I)
        return (_shr(r, 11).to(torch.float64) + 0.5) * (2.0 ** -53)
    return torch.sqrt(-2.0 * torch.log(uni(n2))) * torch.cos(2.0 * np.pi * uni(n2 + 1))


def _finish_t(x, dtype: str):
    import torch
    x32 = x.to(torch.float32)
    return x32.to(torch.bfloat16) if dtype == "bf16" else x32


def keys_torch(w: Workload, t0: int, t1: int, device):
    c = w.chunk
    nck = w.seq_len // c
    parts = []
    for a in range(t0, t1, PIECE):
        b = min(a + PIECE, t1)
        k = draw_torch(w.seed, TAG_K, (w.batch, w.n_kv_heads, w.seq_len, w.head_dim), a, b, device)
        u = draw_torch(w.seed, TAG_OFFSET, (w.batch, w.n_kv_heads, nck, w.head_dim), a // c, b // c, device)
        off = 2.0 * u / u.norm(dim=-1, keepdim=True)
        parts.append(_finish_t(k + off.repeat_interleave(c, dim=2), w.dtype))
    import torch
    return torch.cat(parts, dim=2)


def _plain_torch(w: Workload, tag: int, heads: int, t0: int, t1: int, device):
    import torch
    return torch.cat([_finish_t(draw_torch(w.seed, tag, (w.batch, heads, w.seq_len, w.head_dim), a,
                                           min(a + PIECE, t1), device), w.dtype)
                      for a in range(t0, t1, PIECE)], dim=2)


def values_torch(w: Workload, t0: int, t1: int, device):
    return _plain_torch(w, TAG_V, w.n_kv_heads, t0, t1, device)


def queries_torch(w: Workload, t0: int, t1: int, device):
    return _plain_torch(w, TAG_Q, w.n_q_heads, t0, t1, device)


def grad_out_torch(w: Workload, t0: int, t1: int, device):
    return _plain_torch(w, TAG_DO, w.n_q_heads, t0, t1, device)
