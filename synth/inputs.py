"""Seeded synthetic inputs with the shapes and value distributions of the indexer workloads.

Everything here is input preparation: random draws (torch's counter-based Philox
generator, seeded per call), the per-token FP8 E4M3 quantisation that produces the
codes and fp32 scales the indexer consumes, the layer-to-layer correlation recipe,
and the paged key-cache layout for decode. Nothing here scores, selects or compares.

Quantisation reading (the pages only say "FP8", IndexShare deep-dive report §1.1):
one fp32 scale per token (per query token over all heads x dims, per key token over
dims), scale = absmax / 448 (1.0 for an all-zero token), codes = round-to-nearest-even
of x / scale saturated to +-448, written as OCP E4M3 bytes.
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Iterator, List, Optional, Sequence, Tuple

import torch

E4M3_MAX = 448.0

# The 1/4-retention F/S pattern that greedy search found for the 47-layer 30B model
# (IndexShare deep-dive report, §3.1 "Training-Free: greedy layer selection"). The
# extracted page shows a stray space after the 25th character; it is not part of
# the pattern.
SEARCHED_QUARTER_PATTERN = "FSFSFSSSSFSSSFSSFFSSFSSFS" + "SSSFSSSFSSSSFSSSSSSSSS"

_QUANT_ROWS_PER_CHUNK = 1 << 14


def _generator(seed: int, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    return g


def quantize_e4m3_per_token(x: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-token E4M3 quantisation: returns (uint8 codes shaped like x, fp32 scale[x.shape[0]])."""
    t = x.shape[0]
    flat = x.reshape(t, -1)
    codes = torch.empty(flat.shape, dtype=torch.uint8, device=x.device)
    scale = torch.empty(t, dtype=torch.float32, device=x.device)
    for r0 in range(0, t, _QUANT_ROWS_PER_CHUNK):
        r1 = min(t, r0 + _QUANT_ROWS_PER_CHUNK)
        blk = flat[r0:r1].to(torch.float32)
        absmax = blk.abs().amax(dim=1)
        sc = torch.where(absmax > 0, absmax / E4M3_MAX, torch.ones_like(absmax))
        y = (blk / sc[:, None]).clamp_(-E4M3_MAX, E4M3_MAX)
        codes[r0:r1] = y.to(torch.float8_e4m3fn).view(torch.uint8)
        scale[r0:r1] = sc
    return codes.reshape(x.shape).contiguous(), scale


def _exact_codes(values: torch.Tensor) -> torch.Tensor:
    """E4M3 codes of values that E4M3 represents exactly (small integers, halves)."""
    return values.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).contiguous()


@dataclass
class PrefillLayer:
    """One layer's indexer inputs for L tokens (queries = keys, causal).

    q[L][H][d] u8 E4M3, q_scale[L] f32, w[L][H] f32, k[L][d] u8 E4M3, k_scale[L] f32.
    """

    q: torch.Tensor
    q_scale: torch.Tensor
    w: torch.Tensor
    k: torch.Tensor
    k_scale: torch.Tensor

    @property
    def L(self) -> int:
        return int(self.q.shape[0])

    @property
    def H(self) -> int:
        return int(self.q.shape[1])

    @property
    def d(self) -> int:
        return int(self.q.shape[2])

    def to(self, device) -> "PrefillLayer":
        return PrefillLayer(*(getattr(self, f).to(device).contiguous() for f in
                              ("q", "q_scale", "w", "k", "k_scale")))

    def numpy(self) -> dict:
        return {f: getattr(self, f).detach().cpu().numpy() for f in
                ("q", "q_scale", "w", "k", "k_scale")}


@dataclass
class DecodeLayer:
    """One layer's decode inputs: one query per request and a paged key cache.

    q[B][H][d] u8, q_scale[B] f32, w[B][H] f32, k_cache[nblk][bs][d] u8,
    k_scale_cache[nblk][bs] f32. The block table and lengths are shared by all layers.
    """

    q: torch.Tensor
    q_scale: torch.Tensor
    w: torch.Tensor
    k_cache: torch.Tensor
    k_scale_cache: torch.Tensor

    def to(self, device) -> "DecodeLayer":
        return DecodeLayer(*(getattr(self, f).to(device).contiguous() for f in
                             ("q", "q_scale", "w", "k_cache", "k_scale_cache")))

    def numpy(self) -> dict:
        return {f: getattr(self, f).detach().cpu().numpy() for f in
                ("q", "q_scale", "w", "k_cache", "k_scale_cache")}


def _layer_from_real(xq, xk, xw) -> PrefillLayer:
    q, qs = quantize_e4m3_per_token(xq)
    k, ks = quantize_e4m3_per_token(xk)
    return PrefillLayer(q, qs, xw.to(torch.float32).contiguous(), k, ks)


def gaussian_layer(L: int, H: int, d: int, seed: int, w_std: Optional[float] = None,
                   device="cpu") -> PrefillLayer:
    """q, k ~ N(0,1) per element; w ~ N(0,1) * w_std (default 1/sqrt(H))."""
    g = _generator(seed, device)
    xq = torch.randn(L, H, d, generator=g, device=device)
    xk = torch.randn(L, d, generator=g, device=device)
    ws = (1.0 / math.sqrt(H)) if w_std is None else w_std
    xw = torch.randn(L, H, generator=g, device=device) * ws
    return _layer_from_real(xq, xk, xw)


def planted_layer(L: int, H: int, d: int, topk: int, seed: int, n_plants: int = 8,
                  device="cpu") -> Tuple[PrefillLayer, List[Tuple[int, int]]]:
    """Gaussian layer with `n_plants` keys that copy a query head's direction.

    For each plant: a query row t_p uniform in [topk, L), a key s_p uniform in
    [0, t_p] (distinct over plants), j* = the head with the largest weight of row
    t_p (resampled until that weight is positive), and key s_p is overwritten with
    4*sqrt(d) * q[t_p, j*] / |q[t_p, j*]| before quantisation. Returns the layer and
    the (t_p, s_p) list.
    """
    if L <= topk:
        raise ValueError("planted keys need L > topk")
    g = _generator(seed, device)
    xq = torch.randn(L, H, d, generator=g, device=device)
    xk = torch.randn(L, d, generator=g, device=device)
    xw = torch.randn(L, H, generator=g, device=device) * (1.0 / math.sqrt(H))
    pick = _generator(seed + 7919, "cpu")
    plants: List[Tuple[int, int]] = []
    used_s = set()
    used_t = set()
    while len(plants) < n_plants:
        t_p = int(torch.randint(topk, L, (1,), generator=pick))
        s_p = int(torch.randint(0, t_p + 1, (1,), generator=pick))
        if t_p in used_t or s_p in used_s:
            continue
        j_star = int(torch.argmax(xw[t_p]).item())
        if float(xw[t_p, j_star]) <= 0.0:
            continue
        direction = xq[t_p, j_star]
        xk[s_p] = 4.0 * math.sqrt(d) * direction / direction.norm()
        used_s.add(s_p)
        used_t.add(t_p)
        plants.append((t_p, s_p))
    return _layer_from_real(xq, xk, xw), plants


def gmm_layer(L: int, H: int, d: int, seed: int, n_comp: int = 64, comp_std: float = 0.5,
              w_std: float = 1.0 / 8.0, device="cpu") -> PrefillLayer:
    """Keys from a Gaussian mixture (centres ~ N(0, I_d), component uniform, spread
    `comp_std`); q ~ N(0,1); w ~ N(0,1) * w_std."""
    g = _generator(seed, device)
    centres = torch.randn(n_comp, d, generator=g, device=device)
    comp = torch.randint(0, n_comp, (L,), generator=g, device=device)
    xk = centres[comp] + comp_std * torch.randn(L, d, generator=g, device=device)
    xq = torch.randn(L, H, d, generator=g, device=device)
    xw = torch.randn(L, H, generator=g, device=device) * w_std
    return _layer_from_real(xq, xk, xw)


def correlated_layers(L: int, H: int, d: int, n_layers: int, seed: int, rho: float = 0.9,
                      noise: float = 0.44, w_std: Optional[float] = None,
                      device="cpu") -> Iterator[PrefillLayer]:
    """Layer stack where layer l = (rho * layer(l-1) + noise * fresh N(0,1)) / sqrt(rho^2 + noise^2),
    applied elementwise to the real-valued q, k and w before per-layer quantisation."""
    g = _generator(seed, device)
    norm = math.sqrt(rho * rho + noise * noise)
    ws = (1.0 / math.sqrt(H)) if w_std is None else w_std
    xq = torch.randn(L, H, d, generator=g, device=device)
    xk = torch.randn(L, d, generator=g, device=device)
    xw = torch.randn(L, H, generator=g, device=device)
    for layer in range(n_layers):
        if layer > 0:
            xq.mul_(rho).add_(torch.randn(L, H, d, generator=g, device=device), alpha=noise).div_(norm)
            xk.mul_(rho).add_(torch.randn(L, d, generator=g, device=device), alpha=noise).div_(norm)
            xw.mul_(rho).add_(torch.randn(L, H, generator=g, device=device), alpha=noise).div_(norm)
        yield _layer_from_real(xq, xk, xw * ws)


def exact_layer(L: int, H: int, d: int, seed: int, device="cpu") -> PrefillLayer:
    """Inputs on which fp32 arithmetic in any order is exact, with many tied scores.

    q codes are integers in [-3, 3], key codes integers in [-2, 2] drawn from a small
    pool of distinct key rows (duplicated keys tie exactly), scales are powers of two
    and w takes values in {-1, -0.5, 0.5, 1}. Every dot product is an integer of
    magnitude <= 6d and every head-weighted sum stays far below 2^24.
    """
    g = _generator(seed, "cpu")
    pool = max(4, L // 8)
    qv = torch.randint(-3, 4, (L, H, d), generator=g).to(torch.float32)
    kpool = torch.randint(-2, 3, (pool, d), generator=g).to(torch.float32)
    kscale_pool = torch.tensor([0.5, 1.0, 2.0])[torch.randint(0, 3, (pool,), generator=g)]
    pick = torch.randint(0, pool, (L,), generator=g)
    kv = kpool[pick]
    ks = kscale_pool[pick].to(torch.float32)
    qs = torch.tensor([0.25, 0.5, 1.0, 2.0])[torch.randint(0, 4, (L,), generator=g)].to(torch.float32)
    w = torch.tensor([-1.0, -0.5, 0.5, 1.0])[torch.randint(0, 4, (L, H), generator=g)].to(torch.float32)
    layer = PrefillLayer(_exact_codes(qv), qs.contiguous(), w.contiguous(), _exact_codes(kv),
                         ks.contiguous())
    return layer.to(device)


def ordered_stream_layer(L: int, H: int, d: int, order: str, device="cpu") -> PrefillLayer:
    """Key streams whose score order is fixed by construction (no randomness).

    Every q and k code is E4M3 1.0, q scales are 1 and every head weight is 1/H, so each
    head dot product equals d and the score of (t, s) is d * k_scale[s] * (sum of weights),
    the same for every query. order = "increasing": k_scale[s] = 1 + s/1024 (strictly
    increasing along s, exact in fp32), so every new key beats all earlier ones;
    "decreasing": k_scale[s] = 1 + (L - s)/1024; "constant": all q codes are 0, so every
    score is exactly 0 and only the index breaks ties.
    """
    one = _exact_codes(torch.ones(1))[0]
    q = torch.full((L, H, d), int(one), dtype=torch.uint8)
    if order == "constant":
        q.zero_()
    k = torch.full((L, d), int(one), dtype=torch.uint8)
    s = torch.arange(L, dtype=torch.float64)
    if order == "decreasing":
        s = L - s
    ks = (1.0 + s / 1024.0).to(torch.float32)
    layer = PrefillLayer(q, torch.ones(L, dtype=torch.float32), torch.full((L, H), 1.0 / H, dtype=torch.float32),
                         k, ks.contiguous())
    return layer.to(device)


def periodic_stream_layer(L: int, H: int, d: int, period: int, high_on_multiples: bool,
                          device="cpu") -> PrefillLayer:
    """Like ordered_stream_layer("increasing"), with every period-th key (s % period == 0) four
    times as strong as the rest (high_on_multiples) or every other key four times as strong.

    k_scale[s] = (1 + s/2^20) * (4 or 1), exact in fp32, so all scores are distinct and the
    top-k order is fixed: the strong keys newest first, then the weak keys newest first.
    """
    layer = ordered_stream_layer(L, H, d, "increasing")
    s = torch.arange(L, dtype=torch.float64)
    on = (torch.arange(L) % period) == 0
    strong = on if high_on_multiples else ~on
    ks = (1.0 + s / 2.0 ** 20) * torch.where(strong, 4.0, 1.0).to(torch.float64)
    layer = PrefillLayer(layer.q, layer.q_scale, layer.w, layer.k, ks.to(torch.float32).contiguous())
    return layer.to(device)


def decode_lengths(B: int, lo: int, hi: int, seed: int) -> List[int]:
    """Per-request cache lengths, uniform integers in [lo, hi]."""
    g = _generator(seed, "cpu")
    return [int(x) for x in torch.randint(lo, hi + 1, (B,), generator=g)]


def paged_decode_layers(lens: Sequence[int], H: int, d: int, n_layers: int, seed: int,
                        block_size: int = 64, rho: float = 0.9, noise: float = 0.44,
                        w_std: Optional[float] = None, device="cpu"
                        ) -> Tuple[torch.Tensor, torch.Tensor, Iterator[DecodeLayer]]:
    """Paged decode inputs for len(lens) requests, one new query each.

    Request b owns ceil(lens[b] / block_size) physical blocks, taken in order from a
    random permutation of all physical blocks; its block table row lists them and is
    padded with -1. Keys of every physical slot (including the unused tail of a last
    block) are drawn and quantised per slot. Layers are correlated like
    `correlated_layers`. Returns (block_table[B][max_blocks] i32, seq_lens[B] i32,
    iterator of DecodeLayer).
    """
    B = len(lens)
    nb = [(int(n) + block_size - 1) // block_size for n in lens]
    nblk = sum(nb)
    max_blocks = max(nb) if nb else 0
    g_cpu = _generator(seed, "cpu")
    perm = torch.randperm(nblk, generator=g_cpu).to(torch.int32)
    table = torch.full((B, max(1, max_blocks)), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        table[b, :nb[b]] = perm[off:off + nb[b]]
        off += nb[b]
    seq_lens = torch.tensor([int(n) for n in lens], dtype=torch.int32)

    def layers() -> Iterator[DecodeLayer]:
        g = _generator(seed + 1, device)
        norm = math.sqrt(rho * rho + noise * noise)
        ws = (1.0 / math.sqrt(H)) if w_std is None else w_std
        xq = torch.randn(B, H, d, generator=g, device=device)
        xw = torch.randn(B, H, generator=g, device=device)
        xk = torch.randn(nblk * block_size, d, generator=g, device=device)
        for layer in range(n_layers):
            if layer > 0:
                xq.mul_(rho).add_(torch.randn(B, H, d, generator=g, device=device), alpha=noise).div_(norm)
                xw.mul_(rho).add_(torch.randn(B, H, generator=g, device=device), alpha=noise).div_(norm)
                xk.mul_(rho).add_(torch.randn(nblk * block_size, d, generator=g, device=device),
                                  alpha=noise).div_(norm)
            q, qs = quantize_e4m3_per_token(xq)
            kc, ks = quantize_e4m3_per_token(xk)
            yield DecodeLayer(q, qs, (xw * ws).to(torch.float32).contiguous(),
                              kc.reshape(nblk, block_size, d).contiguous(),
                              ks.reshape(nblk, block_size).contiguous())

    return table.to(device), seq_lens.to(device), layers()


@dataclass
class LatentDecodeInputs:
    """Inputs of the sparse-attention consumer for one decode step: bf16 queries q[B][Hq][dqk],
    a bf16 latent cache latent[n_blocks * block_size][dqk] laid out in the same physical blocks
    as `block_table`, and selected logical positions idx[B][topk] (-1: none)."""
    q: torch.Tensor
    latent: torch.Tensor
    block_table: torch.Tensor
    seq_lens: torch.Tensor
    idx: torch.Tensor


def latent_decode_inputs(lens: Sequence[int], topk: int, seed: int, Hq: int = 128, dqk: int = 576,
                         block_size: int = 64, device="cpu") -> LatentDecodeInputs:
    """Random bf16 queries and latents (N(0, 1) rounded to bf16), a random block table as in
    `paged_decode_layers`, and per request min(topk, len) distinct positions drawn uniformly
    from [0, len) in random order, padded with -1."""
    B = len(lens)
    nb = [(int(n) + block_size - 1) // block_size for n in lens]
    nblk = sum(nb)
    g = _generator(seed, "cpu")
    perm = torch.randperm(nblk, generator=g).to(torch.int32)
    table = torch.full((B, max(1, max(nb) if nb else 1)), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        table[b, :nb[b]] = perm[off:off + nb[b]]
        off += nb[b]
    idx = torch.full((B, topk), -1, dtype=torch.int32)
    for b, n in enumerate(lens):
        m = min(topk, int(n))
        idx[b, :m] = torch.randperm(int(n), generator=g)[:m].to(torch.int32)
    gd = _generator(seed + 1, device)
    q = torch.randn(B, Hq, dqk, generator=gd, device=device).to(torch.bfloat16)
    latent = torch.randn(nblk * block_size, dqk, generator=gd, device=device).to(torch.bfloat16)
    seq = torch.tensor([int(n) for n in lens], dtype=torch.int32)
    return LatentDecodeInputs(q, latent, table.to(device), seq.to(device), idx.to(device))
