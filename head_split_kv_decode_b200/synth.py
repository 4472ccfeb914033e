"""Seeded synthetic inputs: the one module both the CUDA path and the oracle use.

It holds none of the attention arithmetic, only value generation:

* ``normal_at`` / ``kv_field``: a counter-based generator.  Element ``idx`` of
  stream ``seed`` is a function of (seed, idx) alone, so any slice can be
  produced on any device, in any order, with the same bits.  The key
  ``seed * 2**40 + idx`` goes through the SplitMix64 finaliser (Steele, Lea and
  Flood, "Fast Splittable Pseudorandom Number Generators", OOPSLA 2014) twice
  (keys 2k and 2k+1); the eight 16-bit fields of the two outputs are summed
  (Irwin-Hall, n = 8) and standardised.  Only integer operations and one IEEE
  fp32 multiply are involved, so CPU and CUDA produce identical values.  The
  result is approximately N(0, 1) (bounded at about +-4.9 sigma).
* head masks: a seeded permutation per layer marks exactly round(frac * Hkv)
  KV heads as retrieval heads.
* planted structure (needle keys, outlier channels) is computed on the CPU in
  float64 and handed to both sides.

Canonical indexing of a KV history tensor [B, positions, Hkv, d]: element
(b, p, h, c) has index ((b * P_MAX + p) * Hkv + h) * d + c, independent of how
many positions a caller materialises.
"""

import math
from dataclasses import dataclass, field

import torch

P_MAX = 1 << 22           # positions per sequence in the canonical index
_GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_IH_MEAN = 4 * 65535
_IH_INV_STD = 1.0 / math.sqrt(8.0 * (65536.0 ** 2 - 1.0) / 12.0)

# tensor ids inside a (workload, layer) seed block
T_K, T_V, T_Q, T_MASK, T_NEEDLE, T_OUTLIER, T_KNEW, T_VNEW = range(8)


def _s64(c):
    """Unsigned 64-bit constant -> the int64 with the same bits."""
    return c - (1 << 64) if c >= (1 << 63) else c


def _shr(z, k):
    """Logical right shift of int64 tensors."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def _splitmix64(z):
    z = z + _s64(_GOLDEN)
    z = (z ^ _shr(z, 30)) * _s64(_M1)
    z = (z ^ _shr(z, 27)) * _s64(_M2)
    return z ^ _shr(z, 31)


def normal_at(seed, index):
    """Approximately N(0,1) float32 values of stream ``seed`` at int64 ``index``."""
    if not (0 <= seed < (1 << 22)):
        raise ValueError("seed out of range")
    key = index.to(torch.int64) + (int(seed) << 40)
    acc = torch.zeros_like(key)
    for half in (0, 1):
        h = _splitmix64(key * 2 + half)
        for sh in (0, 16, 32, 48):
            acc += (h >> sh) & 0xFFFF
    centred = (acc - _IH_MEAN).to(torch.float32)
    return centred * torch.tensor(_IH_INV_STD, dtype=torch.float32,
                                  device=centred.device)


def normal(seed, shape, device="cpu", chunk=1 << 25):
    """Dense tensor of ``shape`` whose element k is ``normal_at(seed, k)``."""
    numel = math.prod(shape)
    out = torch.empty(numel, dtype=torch.float32, device=device)
    for s in range(0, numel, chunk):
        e = min(numel, s + chunk)
        out[s:e] = normal_at(seed, torch.arange(s, e, device=device))
    return out.view(*shape)


def kv_field(seed, batch_ids, positions, Hkv, d, heads=None, device="cpu"):
    """Values of the canonical [B, P, Hkv, d] stream for the given batch rows,
    positions and (optionally) a subset of heads.

    Returns float32 [len(batch_ids), len(positions), len(heads), d].
    """
    heads = torch.arange(Hkv) if heads is None else torch.as_tensor(heads)
    b = torch.as_tensor(batch_ids, dtype=torch.int64, device=device)
    p = torch.as_tensor(positions, dtype=torch.int64, device=device)
    h = heads.to(dtype=torch.int64, device=device)
    c = torch.arange(d, dtype=torch.int64, device=device)
    idx = ((b[:, None, None, None] * P_MAX + p[None, :, None, None]) * Hkv
           + h[None, None, :, None]) * d + c[None, None, None, :]
    return normal_at(seed, idx.reshape(-1)).view(idx.shape)


def head_mask(seed, layers, n_kv_heads, frac):
    """uint8 [layers, n_kv_heads]: exactly round(frac * Hkv) retrieval heads
    per layer, chosen by a seeded permutation."""
    n_ret = int(round(frac * n_kv_heads))
    mask = torch.zeros(layers, n_kv_heads, dtype=torch.uint8)
    for layer in range(layers):
        g = torch.Generator().manual_seed(seed * 1009 + layer)
        perm = torch.randperm(n_kv_heads, generator=g)
        mask[layer, perm[:n_ret]] = 1
    return mask


def layer_seed(workload_id, layer, tensor_id):
    """Seed of one tensor of one layer of one workload."""
    return 1000 * workload_id + 10 * layer + tensor_id


def outlier_channels(seed, d, frac=0.01):
    """Seeded channel subset (at least one) that is scaled as outliers."""
    k = max(1, int(round(frac * d)))
    g = torch.Generator().manual_seed(seed)
    return torch.randperm(d, generator=g)[:k].sort().values


def needle_position(seed, lo, hi):
    """Seeded position in [lo, hi)."""
    g = torch.Generator().manual_seed(seed)
    return int(torch.randint(lo, hi, (1,), generator=g).item())


def needle_key(q_row, sigma_mult, kv_scale):
    """A key whose dot product with ``q_row`` is ``sigma_mult`` standard
    deviations of q.k for k ~ kv_scale * N(0, I): k = sigma_mult * kv_scale *
    q / |q| (computed in float64 on the CPU)."""
    q = q_row.to(torch.float64).cpu()
    return (sigma_mult * kv_scale * q / q.norm()).to(torch.float32)


@dataclass(frozen=True)
class Workload:
    """Shape and value recipe of one synthetic workload."""
    wid: int
    name: str
    kv_dtype: str            # "f32", "bf16" or "int4"
    layers: int
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    context: int             # tokens already in the cache before decoding
    S: int
    R: int
    retrieval_frac: float
    steps: int = 1           # decode steps (append + attend) per layer
    chunk: int = 0           # pre-fill chunk length (0 = decode workload)
    kv_scale: float = 1.0
    needle_sigma: float = 0.0
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0
    batches: tuple = field(default=())
    row_lengths: tuple = field(default=())  # per-row contexts of a mixed-length batch

    @property
    def group(self):
        return self.n_q_heads // self.n_kv_heads


def mixed_lengths(seed, n, lo, hi):
    """n seeded context lengths, log-uniform in [lo, hi]: the length mix of a
    serving batch whose sequences arrived at different times."""
    g = torch.Generator().manual_seed(seed)
    u = torch.rand(n, generator=g, dtype=torch.float64)
    return tuple(int(round(lo * (hi / lo) ** x)) for x in u.tolist())


WORKLOADS = {
    "tiny_mha_f32": Workload(
        1, "tiny MHA decode fp32: 8/8 heads, d64, ctx 512, S4+R64",
        "f32", 1, 1, 8, 8, 64, 512, 4, 64, 0.5, steps=1),
    "llama2_7b_mha_32k": Workload(
        2, "Llama-2-7B-shaped MHA decode bf16: 32 layers, 32/32 heads, d128, ctx 32768, 25% retrieval, S64+R256",
        "bf16", 32, 1, 32, 32, 128, 32768, 64, 256, 0.25, steps=128,
        kv_scale=0.5, needle_sigma=8.0),
    "llama3_8b_gqa_128k": Workload(
        3, "Llama-3-8B-shaped GQA decode bf16: 32 layers, 32/8 heads, d128, ctx 131072, 50% retrieval, S64+R256",
        "bf16", 32, 1, 32, 8, 128, 131072, 64, 256, 0.5, steps=128,
        batches=(1, 4)),
    "llama3_8b_gqa_prefill_32k": Workload(
        4, "Llama-3-8B-shaped GQA chunked pre-fill bf16: 32/8 heads, d128, 32768-token prompt in 4096-token chunks, 50% retrieval, S64+R256",
        "bf16", 32, 1, 32, 8, 128, 32768, 64, 256, 0.5, chunk=4096),
    "llama3_8b_gqa_paged_mixed": Workload(
        6, "Llama-3-8B-shaped GQA decode bf16, paged KV: 32 layers, 32/8 heads, d128, 8 sequences of 2K-64K tokens (log-uniform), 50% retrieval, S64+R256",
        "bf16", 32, 8, 32, 8, 128, 65536, 64, 256, 0.5, steps=64,
        row_lengths=mixed_lengths(6001, 8, 2048, 65536)),
    "llama3_8b_gqa_int4_1m": Workload(
        5, "Llama-3-8B-shaped GQA decode with INT4 KV: 32 layers, 32/8 heads, d128, ctx 1048576, 25% retrieval, S64+R256",
        "int4", 32, 1, 32, 8, 128, 1048576, 64, 256, 0.25, steps=64,
        outlier_frac=0.01, outlier_mult=10.0),
}


# ---------------------------------------------------------------- materialisers
#
# One consistent stream per (workload, layer, K or V): the K/V of position p is
# the same whether it is part of the pre-filled context or appended by a decode
# step, and the query of a decode step sits at the position of the token that
# step appends.


def history(w, layer, which, batch_ids, positions, heads=None, device="cpu", mask_row=None):
    """K (which="k") or V (which="v") values, float32
    [len(batch_ids), len(positions), len(heads), d], with the workload's planted
    structure: scale, outlier channels, and (K only) one needle key per
    retrieval head placed at a seeded position in [S, context - R)."""
    heads = list(range(w.n_kv_heads)) if heads is None else list(heads)
    tid = T_K if which == "k" else T_V
    x = kv_field(layer_seed(w.wid, layer, tid), batch_ids, positions, w.n_kv_heads,
                 w.head_dim, heads=heads, device=device)
    if w.kv_scale != 1.0:
        x = x * w.kv_scale
    if w.outlier_frac > 0:
        for j, h in enumerate(heads):
            ch = outlier_channels(layer_seed(w.wid, layer, T_OUTLIER) * 128 + h, w.head_dim,
                                  w.outlier_frac).to(device)
            x[:, :, j, ch] = x[:, :, j, ch] * w.outlier_mult
    if which == "k" and w.needle_sigma > 0 and mask_row is not None:
        pos_t = torch.as_tensor(positions)
        for j, h in enumerate(heads):
            if not int(mask_row[h]):
                continue
            for bi, b in enumerate(batch_ids):
                p = needle_position(layer_seed(w.wid, layer, T_NEEDLE) * 4096 + int(b) * 64 + h,
                                    w.S, w.context - w.R)
                hit = (pos_t == p).nonzero()
                if len(hit):
                    q0 = queries(w, layer, [b], [w.context], heads=[h * w.group])[0, 0, 0]
                    x[bi, int(hit[0]), j] = needle_key(q0, w.needle_sigma, w.kv_scale).to(device)
    return x


def queries(w, layer, batch_ids, positions, heads=None, device="cpu"):
    """Query values float32 [len(batch_ids), len(positions), len(heads), d]."""
    return kv_field(layer_seed(w.wid, layer, T_Q), batch_ids, positions, w.n_q_heads,
                    w.head_dim, heads=heads, device=device)


def workload_mask(w):
    """The workload's retrieval-head mask, uint8 [layers, n_kv_heads]."""
    return head_mask(layer_seed(w.wid, 0, T_MASK), w.layers, w.n_kv_heads, w.retrieval_frac)


def io_dtype(w):
    return torch.float32 if w.kv_dtype == "f32" else torch.bfloat16
