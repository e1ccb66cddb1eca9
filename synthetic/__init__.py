"""Seeded synthetic inputs for the NVFP4 quantized linear layer.

This module is shared by the parity tests, the smoke check and the benchmark.
It holds none of the layer's arithmetic (no quantization, no scale rule, no
matmul): only a counter-based generator, the rounding of its draws to BF16,
and the workload recipes (shapes, value distributions, injected outliers and
calibration streams).

Generator.  SplitMix64 in counter form: draw i of stream `seed` is
mix(seed + (i + 1) * 0x9E3779B97F4A7C15), where mix is SplitMix64's output
function.  Uniforms are (u >> 11 + 0.5) * 2^-53, strictly inside (0, 1).
Normals come from Box-Muller on uniform pairs (2j, 2j + 1): element 2j takes
the cosine branch and 2j + 1 the sine branch, in binary64.  Draws are rounded
to BF16 with round-to-nearest-even directly from binary64.

Workloads stand in for the pages' activations (FastH3 Trim, comfyui-wiki news,
"What the ComfyUI repack contains": every NVFP4 layer calibrated on 1,000
prompts; FastH3 thread digest, farwalk.ai, tweet 6/8: uncalibrated scales clip
up to 137x the limit).  The prompts, weights and activations themselves are
not available, so the activations are seeded draws with the distributions
below, and an evaluation batch is always a PREFIX of its layer's calibration
stream, so "a calibrated scale clips nothing" holds by construction.
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, field

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

#: Clip limit L of the recipes: no body draw reaches it (bodies are N(0,1)
#: truncated at 8), and injected outliers are multiples of it up to 137 L.
CLIP_LIMIT = 8.0
OUTLIER_MAX_FACTOR = 137.0


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def derive_seed(*keys) -> int:
    """Fold a tuple of ints / strings into one 64-bit stream seed."""
    z = np.array([0x5EED5EED5EED5EED], dtype=np.uint64)
    with np.errstate(over="ignore"):
        for k in keys:
            if isinstance(k, (tuple, list)):
                v = derive_seed(*k)
            else:
                v = zlib.crc32(k.encode()) if isinstance(k, str) else int(k)
            z = _mix(z + np.uint64(v & 0xFFFFFFFFFFFFFFFF) * _GAMMA + _GAMMA)
    return int(z[0])


def u64(seed: int, start: int, n: int) -> np.ndarray:
    """Draws start .. start+n-1 of stream `seed` as uint64."""
    idx = np.arange(start + 1, start + 1 + n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(np.uint64(seed) + idx * _GAMMA)


def uniform(seed: int, start: int, n: int) -> np.ndarray:
    u = u64(seed, start, n) >> np.uint64(11)
    return (u.astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, start: int, n: int) -> np.ndarray:
    """Standard normals start .. start+n-1 of stream `seed` (Box-Muller)."""
    p0, p1 = start // 2, (start + n + 1) // 2
    u = uniform(seed, 2 * p0, 2 * (p1 - p0)).reshape(-1, 2)
    r = np.sqrt(-2.0 * np.log(u[:, 0]))
    t = 2.0 * np.pi * u[:, 1]
    z = np.empty(2 * (p1 - p0), dtype=np.float64)
    z[0::2] = r * np.cos(t)
    z[1::2] = r * np.sin(t)
    off = start - 2 * p0
    return z[off:off + n]


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round binary64 values to BF16 (nearest, ties to even), as uint16 bits.

    Values must be finite and inside the BF16 normal range or zero."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                    # x = m * 2^e, 0.5 <= |m| < 1
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)   # 8 significant bits, RNE
    f = r.astype(np.float32)              # exact: r has 8 significant bits
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def truncated_normal(seed: int, start: int, n: int, bound: float = CLIP_LIMIT) -> np.ndarray:
    """Normals with |z| < bound; a draw at or beyond it is redrawn from the
    stream's redraw sub-streams (attempt 1, 2, ...) at the same index."""
    z = normal(seed, start, n)
    bad = np.nonzero(np.abs(z) >= bound)[0]
    attempt = 0
    while bad.size:
        attempt += 1
        rs = derive_seed(seed, "redraw", attempt)
        for i in bad:
            z[i] = normal(rs, start + int(i), 1)[0]
        bad = bad[np.abs(z[bad]) >= bound]
    return z


# ---------------------------------------------------------------------------
# Workload recipes
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class Layer:
    """One quantized linear layer of a workload: y[M, N] = x[M, K] . W[N, K]^T + b."""
    name: str
    M: int
    K: int
    N: int
    batch: int                 # tokens per calibration batch
    n_calib: int               # calibration batches; the input is batches 0 .. M/batch - 1
    outlier_rate: float = 0.0  # fraction of elements replaced by outliers, per batch
    outlier_mode: str = "fixed"    # "fixed": all +-137 L; "uniform": L * U[1, 137], one exactly 137 L
    channel_lognormal: bool = False  # per-channel std exp(N(0, 1)), drawn once per layer
    key: tuple = field(default=())  # seed key of the layer

    @property
    def n_eval_batches(self) -> int:
        return self.M // self.batch

    def outliers_per_batch(self) -> int:
        return int(round(self.outlier_rate * self.batch * self.K))


def workloads() -> dict:
    """The five synthetic workloads, by name.

    tiny         128 x 256 -> 256; N(0,1) with 0.1% outliers at +-137 L; 16 calibration batches of 128 tokens.
    attn_proj    8192 x 2688 -> 2688; N(0,1) with 0.01% outliers L * U[1,137]; 1000 batches of 64 tokens.
    qkv          32768 x 2688 -> 8064; N(0,1) times a log-normal (sigma 1) std per channel; 1000 x 64.
    ffn          up 32768 x 2688 -> 10752 (attn_proj's distribution), GELU, down 32768 x 10752 -> 2688
                 (its input is the GELU output of the up layer, so it has no recipe of its own).
    block_sweep  42 blocks x {qkv 2688->8064, out 2688->2688, up 2688->10752, down 10752->2688} at M=49152,
                 qkv/out/up inputs drawn like qkv, each layer with its own seeds.
    """
    w = {
        "tiny": [Layer("tiny", 128, 256, 256, 128, 16, 1e-3, "fixed", key=("tiny", 0))],
        "attn_proj": [Layer("attn_proj", 8192, 2688, 2688, 64, 1000, 1e-4, "uniform", key=("attn_proj", 0))],
        "qkv": [Layer("qkv", 32768, 2688, 8064, 64, 1000, channel_lognormal=True, key=("qkv", 0))],
        "ffn": [Layer("ffn_up", 32768, 2688, 10752, 64, 1000, 1e-4, "uniform", key=("ffn", "up")),
                Layer("ffn_down", 32768, 10752, 2688, 64, 1000, key=("ffn", "down"))],
    }
    sweep = []
    for b in range(42):
        sweep += [Layer(f"b{b}.qkv", 49152, 2688, 8064, 64, 1000, channel_lognormal=True, key=("sweep", b, "qkv")),
                  Layer(f"b{b}.out", 49152, 2688, 2688, 64, 1000, channel_lognormal=True, key=("sweep", b, "out")),
                  Layer(f"b{b}.up", 49152, 2688, 10752, 64, 1000, channel_lognormal=True, key=("sweep", b, "up")),
                  Layer(f"b{b}.down", 49152, 10752, 2688, 64, 1000, key=("sweep", b, "down"))]
    w["block_sweep"] = sweep
    return w


def channel_std(layer: Layer) -> np.ndarray:
    return np.exp(normal(derive_seed(*layer.key, "channel_std"), 0, layer.K))


def activation_batches(layer: Layer, b0: int, nb: int, uncalibrated_body: bool = False,
                       bound: float = CLIP_LIMIT) -> np.ndarray:
    """Calibration-stream batches b0 .. b0+nb-1 of `layer` as BF16 bits [nb * batch, K]
    (`bound`: the truncation of the body draws; the recipes use CLIP_LIMIT)."""
    B, K = layer.batch, layer.K
    out = np.empty((nb * B, K), dtype=np.uint16)
    std = channel_std(layer) if layer.channel_lognormal else None
    n_out = layer.outliers_per_batch()
    for j in range(nb):
        b = b0 + j
        s = derive_seed(*layer.key, "x", b)
        z = truncated_normal(s, 0, B * K, bound)
        if std is not None:
            z = (z.reshape(B, K) * std[None, :]).reshape(-1)
        if n_out and not uncalibrated_body:
            keys = u64(derive_seed(s, "outlier_pos"), 0, B * K)
            pos = np.argpartition(keys, n_out)[:n_out]
            pos = pos[np.argsort(keys[pos])]           # the lowest key first
            sign = np.where(uniform(derive_seed(s, "outlier_sign"), 0, n_out) < 0.5, -1.0, 1.0)
            if layer.outlier_mode == "fixed":
                mag = np.full(n_out, OUTLIER_MAX_FACTOR * CLIP_LIMIT)
            else:
                u = 1.0 + (OUTLIER_MAX_FACTOR - 1.0) * uniform(derive_seed(s, "outlier_mag"), 0, n_out)
                mag = CLIP_LIMIT * u
                mag[0] = OUTLIER_MAX_FACTOR * CLIP_LIMIT
            z[pos] = sign * mag
        out[j * B:(j + 1) * B] = to_bf16_bits(z).reshape(B, K)
    return out


def outlier_positions(layer: Layer, b: int) -> np.ndarray:
    """Flat positions (within batch b, row-major [batch, K]) of the injected outliers."""
    n_out = layer.outliers_per_batch()
    s = derive_seed(*layer.key, "x", b)
    keys = u64(derive_seed(s, "outlier_pos"), 0, layer.batch * layer.K)
    pos = np.argpartition(keys, n_out)[:n_out]
    return np.sort(pos)


def activations(layer: Layer) -> np.ndarray:
    """The layer's input x [M, K]: calibration batches 0 .. M/batch - 1."""
    return activation_batches(layer, 0, layer.n_eval_batches)


def weights(layer: Layer) -> np.ndarray:
    """W [N, K] ~ N(0, 0.02^2) as BF16 bits."""
    z = normal(derive_seed(*layer.key, "w"), 0, layer.N * layer.K) * 0.02
    return to_bf16_bits(z).reshape(layer.N, layer.K)


def bias(layer: Layer) -> np.ndarray:
    """b [N] ~ N(0, 0.01^2) as BF16 bits."""
    return to_bf16_bits(normal(derive_seed(*layer.key, "b"), 0, layer.N) * 0.01)


def random_bf16(seed_key, shape, std: float = 1.0) -> np.ndarray:
    """Plain N(0, std^2) BF16 bits of any shape (edge-case tests)."""
    n = int(np.prod(shape))
    return to_bf16_bits(normal(derive_seed(*seed_key), 0, n) * std).reshape(shape)


def attention_qk(heads: int, tokens: int, d: int, which: str, seed: int = 0) -> np.ndarray:
    """Query or key activations of shape [heads, tokens, d] as BF16 bits.

    Each (head, channel) has its own spread, exp(N(0, 0.5^2)), and one channel
    in 32 of every head is an outlier channel with 8x that spread; that is the
    channel-wise outlier structure of attention queries and keys that
    per-token INT8 scales must absorb.  Every tenth token is scaled by 4, so
    rows differ in range as well."""
    n = heads * tokens * d
    z = normal(derive_seed("attn", which, seed, heads, tokens, d), 0, n).reshape(heads, tokens, d)
    spread = np.exp(0.5 * normal(derive_seed("attn-spread", which, seed, heads, d), 0, heads * d)).reshape(heads, 1, d)
    outlier = (u64(derive_seed("attn-outlier", which, seed, heads, d), 0, heads * d) % 32 == 0).reshape(heads, 1, d)
    spread = spread * np.where(outlier, 8.0, 1.0)
    row = np.where(np.arange(tokens) % 10 == 0, 4.0, 1.0).reshape(1, tokens, 1)
    return to_bf16_bits(z * spread * row)


def to_f16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> IEEE half bits (numpy's conversion, round to nearest even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


# The eight timesteps of the distilled sampler (FastH3 Trim, "What Trim changes").
SAMPLER_TIMESTEPS = (999, 874, 749, 624, 500, 375, 250, 125)


def adaln_inputs(blocks: int, n: int, d: int, r: int, timesteps, seed: int = 0):
    """Synthetic stand-ins for the AdaLN basis projection (no trained weights exist here):
    time embeddings e [bt, d] BF16 ~ N(0, 1), one seeded row per timestep; shared basis
    [r, d] FP16 ~ N(0, 1/d) (rows of about unit norm); per-block projections [blocks, n, r]
    FP16 ~ N(0, 0.05^2); per-block biases [blocks, n] FP16 ~ N(0, 0.01^2)."""
    e = np.stack([normal(derive_seed("temb", seed, int(t), d), 0, d) for t in timesteps]) if len(timesteps) \
        else np.zeros((0, d))
    basis = normal(derive_seed("adaln-basis", seed, r, d), 0, r * d).reshape(r, d) / np.sqrt(d)
    proj = normal(derive_seed("adaln-proj", seed, blocks, n, r), 0, blocks * n * r).reshape(blocks, n, r) * 0.05
    bias = normal(derive_seed("adaln-bias", seed, blocks, n), 0, blocks * n).reshape(blocks, n) * 0.01
    return to_bf16_bits(e), to_f16_bits(basis), to_f16_bits(proj), to_f16_bits(bias)


# ---------------------------------------------------------------------------
# The same recipes evaluated with torch on any device
# ---------------------------------------------------------------------------
#
# Full-size workloads (the 168-layer block sweep draws ~50 G normals) are far
# too large for numpy on the host, so the recipes are also written with torch
# tensor operations that run where the tensors live.  The arithmetic is the
# same step for step: SplitMix64 in uint64 arithmetic (held in int64 tensors;
# multiplication wraps modulo 2^64, right shifts are made logical by masking),
# the same uniform and Box-Muller formulas in binary64, and BF16
# round-to-nearest-even straight from binary64.  The only possible difference
# from the numpy path is the last-ulp rounding of log, cos and sin in the
# device's libraries, which changes the BF16 result only when a draw lies
# within ~1e-16 (relative) of a BF16 rounding boundary: about 1e-13 of draws.
# Tests that consume these tensors always hand the oracle the very bytes the
# GPU consumed, so parity never depends on the two paths agreeing.

def _s64(v: int) -> int:
    """uint64 value -> the int64 with the same bits."""
    return v - (1 << 64) if v >= (1 << 63) else v


_GAMMA_S = _s64(0x9E3779B97F4A7C15)
_M1_S = _s64(0xBF58476D1CE4E5B9)
_M2_S = _s64(0x94D049BB133111EB)


def _srl(z, s: int):
    """Logical right shift of int64 tensors holding uint64 bits."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix_t(z):
    z = (z ^ _srl(z, 30)) * _M1_S
    z = (z ^ _srl(z, 27)) * _M2_S
    return z ^ _srl(z, 31)


def u64_t(seed: int, start: int, n: int, device):
    """Draws start .. start+n-1 of stream `seed` (int64 tensor of uint64 bits)."""
    import torch
    idx = torch.arange(start + 1, start + 1 + n, dtype=torch.int64, device=device)
    return _mix_t(idx * _GAMMA_S + _s64(seed & 0xFFFFFFFFFFFFFFFF))


def uniform_t(seed: int, start: int, n: int, device):
    import torch
    u = _srl(u64_t(seed, start, n, device), 11)
    return (u.to(torch.float64) + 0.5) * (2.0 ** -53)


def normal_t(seed: int, start: int, n: int, device):
    """Standard normals start .. start+n-1 of stream `seed` (float64 tensor), as normal()."""
    import torch
    p0, p1 = start // 2, (start + n + 1) // 2
    u = uniform_t(seed, 2 * p0, 2 * (p1 - p0), device).view(-1, 2)
    r = torch.sqrt(-2.0 * torch.log(u[:, 0]))
    t = (2.0 * np.pi) * u[:, 1]
    z = torch.stack((r * torch.cos(t), r * torch.sin(t)), dim=1).view(-1)
    off = start - 2 * p0
    return z[off:off + n]


def to_bf16_bits_t(x):
    """Round a float64 tensor to BF16 (nearest, ties to even) directly from
    binary64, as to_bf16_bits; returns int16 bits (view as torch.bfloat16)."""
    import torch
    m, e = torch.frexp(x)
    r = torch.ldexp(torch.round(torch.ldexp(m, torch.full_like(e, 8))), e - 8)
    return (r.to(torch.float32).view(torch.int32) >> 16).to(torch.int16)


def truncated_normal_t(seed: int, start: int, n: int, device, bound: float = CLIP_LIMIT):
    """truncated_normal() on `device`: draws at or beyond `bound` are redrawn
    from the redraw sub-streams (rare: ~1e-15 of draws), on the host."""
    import torch
    z = normal_t(seed, start, n, device)
    bad = torch.nonzero(z.abs() >= bound).view(-1)
    if bad.numel():
        idx = bad.cpu().numpy()
        fix = np.empty(idx.size)
        for j, i in enumerate(idx):
            v, attempt = float(z[int(i)]), 0
            while abs(v) >= bound:
                attempt += 1
                v = normal(derive_seed(seed, "redraw", attempt), start + int(i), 1)[0]
            fix[j] = v
        z[bad] = torch.from_numpy(fix).to(device)
    return z


def _normal_rows_t(seeds, n: int, device):
    """Row j = normal(seeds[j], 0, n) for an even n, all rows at once ([len(seeds), n] float64)."""
    import torch
    sd = torch.tensor([_s64(v & 0xFFFFFFFFFFFFFFFF) for v in seeds], dtype=torch.int64, device=device)
    idx = torch.arange(1, n + 1, dtype=torch.int64, device=device)
    u = (_srl(_mix_t(idx[None, :] * _GAMMA_S + sd[:, None]), 11).to(torch.float64) + 0.5) * (2.0 ** -53)
    u = u.view(len(seeds), n // 2, 2)
    r = torch.sqrt(-2.0 * torch.log(u[:, :, 0]))
    t = (2.0 * np.pi) * u[:, :, 1]
    return torch.stack((r * torch.cos(t), r * torch.sin(t)), dim=2).view(len(seeds), n)


def activation_batches_t(layer: Layer, b0: int, nb: int, device, chunk: int = 32, bound: float = CLIP_LIMIT):
    """activation_batches() on `device`: calibration-stream batches b0 ..
    b0+nb-1 as int16 BF16 bits [nb * batch, K], `chunk` batches per pass
    (every recipe: log-normal channel spreads and injected outliers)."""
    import torch
    B, K = layer.batch, layer.K
    n_out = layer.outliers_per_batch()
    std = torch.from_numpy(channel_std(layer)).to(device) if layer.channel_lognormal else None
    out = torch.empty((nb * B, K), dtype=torch.int16, device=device)
    for j0 in range(0, nb, chunk):
        seeds = [derive_seed(*layer.key, "x", b0 + j) for j in range(j0, min(nb, j0 + chunk))]
        z = _normal_rows_t(seeds, B * K, device)
        bad = torch.nonzero(z.abs() >= bound)
        for r, i in bad.cpu().tolist():             # truncation redraws: ~1e-15 of draws at bound 8
            v, attempt = float(z[r, i]), 0
            while abs(v) >= bound:
                attempt += 1
                v = normal(derive_seed(seeds[r], "redraw", attempt), i, 1)[0]
            z[r, i] = v
        if std is not None:
            z = (z.view(len(seeds), B, K) * std[None, None, :]).view(len(seeds), B * K)
        if n_out:
            # The n_out positions with the lowest keys (keys compared as uint64:
            # flipping the sign bit makes the int64 order the unsigned one).
            keys = _normal_keys_t([derive_seed(s, "outlier_pos") for s in seeds], B * K, device)
            pos = torch.topk(keys ^ _s64(1 << 63), n_out, dim=1, largest=False, sorted=True).indices
            sign_u = torch.stack([uniform_t(derive_seed(s, "outlier_sign"), 0, n_out, device) for s in seeds])
            sign = torch.where(sign_u < 0.5, -1.0, 1.0).to(torch.float64)
            if layer.outlier_mode == "fixed":
                mag = torch.full((len(seeds), n_out), OUTLIER_MAX_FACTOR * CLIP_LIMIT, dtype=torch.float64,
                                 device=device)
            else:
                u = torch.stack([uniform_t(derive_seed(s, "outlier_mag"), 0, n_out, device) for s in seeds])
                mag = CLIP_LIMIT * (1.0 + (OUTLIER_MAX_FACTOR - 1.0) * u)
                mag[:, 0] = OUTLIER_MAX_FACTOR * CLIP_LIMIT
            z.scatter_(1, pos, sign * mag)
        out[j0 * B:(j0 + len(seeds)) * B] = to_bf16_bits_t(z).view(len(seeds) * B, K)
    return out


def _normal_keys_t(seeds, n: int, device):
    """Row j = u64(seeds[j], 0, n) (int64 tensor of uint64 bits), all rows at once."""
    import torch
    sd = torch.tensor([_s64(v & 0xFFFFFFFFFFFFFFFF) for v in seeds], dtype=torch.int64, device=device)
    idx = torch.arange(1, n + 1, dtype=torch.int64, device=device)
    return _mix_t(idx[None, :] * _GAMMA_S + sd[:, None])


def weights_t(layer: Layer, device):
    """weights() on `device` as int16 BF16 bits [N, K]."""
    return to_bf16_bits_t(normal_t(derive_seed(*layer.key, "w"), 0, layer.N * layer.K, device) * 0.02) \
        .view(layer.N, layer.K)


def bias_t(layer: Layer, device):
    """bias() on `device` as int16 BF16 bits [N]."""
    return to_bf16_bits_t(normal_t(derive_seed(*layer.key, "b"), 0, layer.N, device) * 0.01)
