"""Seeded synthetic inputs for the MoonEP hot path.

This module only draws inputs: router output (top-K ids and weights), hidden
states, per-expert scales, expert weights and replica gradients.  It holds
none of the method's arithmetic (no keep/spill split, no planning, no
destination rows, no reduction), so the CUDA path and the CPU oracle can both
consume what it produces without sharing any code with each other.

Router skew follows the workload statement used throughout this library: a
per-expert logit bias b_e = alpha * 2 * log(1 / (rank_e + 1)), where rank_e is
the expert's position in a seeded random permutation (a Zipf-like skew), added
to N(0, 1) noise; top-K by logit; the K softmax probabilities renormalised to
sum to one.  This stands in for the lognormal-sigma routing generator that
"The Busiest Rank Sets Your Step Time: Running MoonEP's Planning Code
Ourselves" (section "What we measured") ran but did not print.

Large tensors (hidden states, weights, gradients) come from a counter-based
generator (SplitMix64, Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) so that any element can be regenerated on the
host by index, identically to the device copy: four 16-bit uniforms per
element, summed (an Irwin-Hall(4) variate, exact in fp32) and scaled by sqrt(3)
to unit variance.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# ----------------------------------------------------------------------------
# Workloads
# ----------------------------------------------------------------------------


@dataclass(frozen=True)
class Workload:
    """One synthetic workload.  L = experts per rank, N = R*L experts in total,
    C = S*K rows per rank, C_max = C or the headroom size, I = FFN intermediate
    size; weights per expert are P*H*I bf16 values, gradients H*I fp32."""
    name: str
    R: int
    L: int
    S: int
    K: int
    H: int
    B: int
    I: int
    P: int = 2
    headroom: float = 0.0          # C_max = floor((1 + headroom) * C)
    maxvio: tuple = ()             # target input maxvio values (empty: use alpha)
    alpha: float | None = None     # fixed bias scale when maxvio is not targeted
    seeds: tuple = (0, 1, 2, 3, 4)

    @property
    def N(self):
        return self.R * self.L

    @property
    def T(self):
        return self.R * self.S

    @property
    def C(self):
        return self.S * self.K

    @property
    def C_max(self):
        return int(math.floor((1.0 + self.headroom) * self.C))

    @property
    def w_elems(self):
        return self.P * self.H * self.I

    @property
    def g_elems(self):
        return self.H * self.I

    def cfg(self):
        return dict(R=self.R, L=self.L, S=self.S, K=self.K, H=self.H, B=self.B,
                    C=self.C, C_max=self.C_max)


WORKLOADS = {
    "tiny": Workload("tiny", R=4, L=4, S=64, K=2, H=128, B=4, I=256, alpha=1.0),
    "mid": Workload("mid", R=8, L=8, S=4096, K=8, H=7168, B=8, I=2048, maxvio=(2.0,)),
    "skew": Workload("skew", R=8, L=32, S=8192, K=8, H=7168, B=32, I=2048,
                     maxvio=(0.0, 1.0, 2.0, 4.0, 8.0)),
    "inference": Workload("inference", R=16, L=24, S=2048, K=8, H=7168, B=4, I=2048,
                          headroom=0.25, maxvio=(4.0,)),
    "training": Workload("training", R=16, L=16, S=8192, K=8, H=7168, B=16, I=2048,
                         maxvio=(8.0,)),
    # the mid shapes at a quarter of the tokens and an eighth of the FFN size:
    # about 3 GB on the device, still far above L2, for profiler captures
    "profile": Workload("profile", R=8, L=8, S=1024, K=8, H=7168, B=8, I=256, maxvio=(2.0,)),
    # the full FFN size (I = 2048, 58.7 MB of fp32 gradient per expert) over
    # 16 experts, for captures of the weight and gradient kernels: at seed 0,
    # 3 replicated experts with 3, 3 and 2 pieces (the mid workload has 3, 4
    # and 1); prefetch moves 0.94 GB and reduce_grad 1.29 GB (as on mid), far
    # above L2, while the weights or gradients take about 1.9 GB
    "profile_w": Workload("profile_w", R=8, L=2, S=4096, K=2, H=7168, B=2, I=2048, maxvio=(2.0,)),
}


# ----------------------------------------------------------------------------
# Router output
# ----------------------------------------------------------------------------


def input_maxvio(topk_idx: np.ndarray, N: int) -> float:
    """Per-expert input imbalance: max expert load / mean expert load - 1."""
    ids = np.asarray(topk_idx).reshape(-1)
    if ids.size == 0:
        return 0.0
    cnt = np.bincount(ids, minlength=N)
    return float(cnt.max()) / (ids.size / N) - 1.0


def _topk(logits: np.ndarray, K: int):
    """Top-K of each row by descending logit.  Returns (ids int64, logits)."""
    import torch
    v, i = torch.topk(torch.from_numpy(logits), K, dim=1, largest=True, sorted=True)
    return i.numpy(), v.numpy()


def _renorm_weights(sel_logits: np.ndarray) -> np.ndarray:
    """Softmax probabilities of the chosen K, renormalised to sum to 1 (equal to
    a softmax over the chosen logits); computed in fp64, stored as fp32."""
    z = sel_logits.astype(np.float64)
    z = z - z.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    return p.astype(np.float32)


@dataclass
class Routing:
    topk_idx: np.ndarray      # int32 [R, S, K]
    topk_w: np.ndarray        # fp32  [R, S, K]
    alpha: float
    maxvio: float             # achieved input maxvio
    target: float | None = None
    info: dict = field(default_factory=dict)


def routing(R, L, S, K, seed, alpha=None, maxvio=None, tol=0.05, balanced=False):
    """Router output for R ranks x S tokens, K of N=R*L experts.

    alpha: bias scale.  maxvio: if given, alpha is bisected until the achieved
    input maxvio is within +-tol (relative) of the target.  maxvio == 0 (or
    balanced=True) gives exactly balanced routing: global token t picks experts
    (t*K + k) mod N, weights renormalised from the same random logits.
    """
    N, T = R * L, R * S
    if K > N:
        raise ValueError("K must not exceed the number of experts")
    rng = np.random.Generator(np.random.PCG64(seed))
    perm = rng.permutation(N)
    pos = np.empty(N, np.int64)
    pos[perm] = np.arange(N)
    bias = 2.0 * np.log(1.0 / (pos + 1.0))          # fp64, <= 0
    z = rng.standard_normal((T, N)) if T > 0 else np.zeros((0, N))

    if balanced or (maxvio is not None and maxvio == 0.0):
        t = np.arange(T, dtype=np.int64)[:, None]
        ids = (t * K + np.arange(K, dtype=np.int64)[None, :]) % N
        sel = np.take_along_axis(z.astype(np.float32), ids, axis=1)
        order = np.lexsort((ids, -sel), axis=1) if T > 0 else np.zeros((0, K), np.int64)
        ids = np.take_along_axis(ids, order, axis=1)
        sel = np.take_along_axis(sel, order, axis=1)
        w = _renorm_weights(sel) if T > 0 else np.zeros((0, K), np.float32)
        r = Routing(ids.astype(np.int32).reshape(R, S, K), w.reshape(R, S, K), 0.0,
                    input_maxvio(ids, N), 0.0)
        return r

    def draw(a):
        logits = (z + a * bias[None, :]).astype(np.float32)
        if T == 0:
            return np.zeros((0, K), np.int64), np.zeros((0, K), np.float32)
        return _topk(logits, K)

    if maxvio is None:
        a = 1.0 if alpha is None else float(alpha)
        ids, sel = draw(a)
    else:
        target = float(maxvio)
        lo, hi = 0.0, 1.0
        ids, sel = draw(hi)
        while input_maxvio(ids, N) < target and hi < 64.0:
            lo, hi = hi, hi * 2.0
            ids, sel = draw(hi)
        a = hi
        for _ in range(40):
            mv = input_maxvio(ids, N)
            if abs(mv - target) <= tol * target:
                break
            if mv < target:
                lo = a
            else:
                hi = a
            a = 0.5 * (lo + hi)
            ids, sel = draw(a)
    w = _renorm_weights(sel) if T > 0 else np.zeros((0, K), np.float32)
    return Routing(ids.astype(np.int32).reshape(R, S, K), w.reshape(R, S, K), float(a),
                   input_maxvio(ids, N), maxvio)


def lognormal_routing(R, L, S, K, seed, sigma):
    """Router output with a lognormal per-expert popularity: expert e gets
    sampling weight exp(sigma * n_e), n_e ~ N(0,1); each token draws K distinct
    experts in proportion to it (Gumbel top-K).  A stand-in for the sigma-knob
    generator of the planning-balance table in "The Busiest Rank Sets Your Step
    Time" (section "What we measured"), whose code is not printed."""
    N, T = R * L, R * S
    rng = np.random.Generator(np.random.PCG64(seed))
    logpop = sigma * rng.standard_normal(N)
    g = rng.gumbel(size=(T, N))
    logits = (g + logpop[None, :]).astype(np.float32)
    ids, sel = _topk(logits, K)
    w = _renorm_weights(sel)
    return Routing(ids.astype(np.int32).reshape(R, S, K), w.reshape(R, S, K), sigma,
                   input_maxvio(ids, N), None)


def expert_scales(N, seed):
    """Per-expert fp32 scale ~ U(0.5, 1.5) for the stand-in expert."""
    rng = np.random.Generator(np.random.PCG64(seed + 7919))
    return rng.uniform(0.5, 1.5, N).astype(np.float32)


# ----------------------------------------------------------------------------
# Counter-based generator for large tensors (host: numpy, device: torch)
# ----------------------------------------------------------------------------

_GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_SQRT3 = np.float32(1.7320508075688772)

# stream ids keep the tensors of one workload independent of each other
STREAM_X, STREAM_W, STREAM_G_HOME, STREAM_G_REP, STREAM_Y = 1, 2, 3, 4, 5


def _key(seed: int, stream: int) -> int:
    return ((seed * 0x100000001B3) ^ (stream << 48) ^ 0x5851F42D4C957F2D) & 0xFFFFFFFFFFFFFFFF


def _splitmix_np(x):
    x = x + np.uint64(_GOLDEN)
    x = (x ^ (x >> np.uint64(30))) * np.uint64(_M1)
    x = (x ^ (x >> np.uint64(27))) * np.uint64(_M2)
    return x ^ (x >> np.uint64(31))


def cb_f32_np(seed: int, stream: int, idx) -> np.ndarray:
    """fp32 value of element(s) idx of the counter-based stream."""
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        h = _splitmix_np(idx + np.uint64(_key(seed, stream)))
    mask = np.uint64(0xFFFF)
    s = ((h & mask).astype(np.float32) + ((h >> np.uint64(16)) & mask).astype(np.float32)
         + ((h >> np.uint64(32)) & mask).astype(np.float32)
         + ((h >> np.uint64(48)) & mask).astype(np.float32))
    # s is a sum of four integers < 2^16: exact in fp32; /2^16 is exact
    u = s * np.float32(1.0 / 65536.0) - np.float32(2.0)
    return (u * _SQRT3).astype(np.float32)


def f32_to_bf16_bits_np(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = ((b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    return r


def bf16_bits_to_f32_np(u: np.ndarray) -> np.ndarray:
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def cb_bf16_np(seed: int, stream: int, idx) -> np.ndarray:
    """bf16 bit patterns (uint16) of element(s) idx."""
    return f32_to_bf16_bits_np(cb_f32_np(seed, stream, idx))


def _lsr(x, s):
    """Logical right shift of torch int64 (torch's >> is arithmetic)."""
    return (x >> s) & ((1 << (64 - s)) - 1)


def _wrap_i64(v: int) -> int:
    v &= 0xFFFFFFFFFFFFFFFF
    return v - (1 << 64) if v >= (1 << 63) else v


def cb_fill_torch(out, seed: int, stream: int, offset: int = 0, chunk: int = 1 << 25):
    """Fill a contiguous torch tensor (float32 or bfloat16, any device) with the
    counter-based stream: element i of out gets value cb_f32(seed, stream,
    offset + i) (rounded to nearest-even for bfloat16)."""
    import torch
    flat = out.view(-1)
    n = flat.numel()
    key = _key(seed, stream)
    g, m1, m2 = _wrap_i64(_GOLDEN), _wrap_i64(_M1), _wrap_i64(_M2)
    for start in range(0, n, chunk):
        cnt = min(chunk, n - start)
        x = torch.arange(start + offset, start + offset + cnt, dtype=torch.int64, device=out.device)
        x = x + _wrap_i64(key)
        x = x + g
        x = (x ^ _lsr(x, 30)) * m1
        x = (x ^ _lsr(x, 27)) * m2
        x = x ^ _lsr(x, 31)
        s = ((x & 0xFFFF).float() + (_lsr(x, 16) & 0xFFFF).float()
             + (_lsr(x, 32) & 0xFFFF).float() + (_lsr(x, 48) & 0xFFFF).float())
        u = s * (1.0 / 65536.0) - 2.0
        v = u * float(_SQRT3)
        flat[start:start + cnt] = v.to(flat.dtype)
        del x, s, u, v
    return out
