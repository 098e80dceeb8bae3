"""Seeded synthetic inputs for the DSA layer, shared by the tests, the
benchmark and the smoke check.

This module draws random numbers and packs them into the layouts the library
and the oracle read; it holds none of the layer's arithmetic (no indexer, no
top-k, no attention).  The FP8 packing below is input preparation: the pages
only say the indexer runs in FP8 ("Kwai Keye-VL-2.0 Technical Report" review,
DSA section: "FP8实现"; report translation section 2.3.1), so the format
(OCP e4m3fn) and granularity (one scale per token, absmax / 448) are a reading
of ours.  Both the oracle and the CUDA path consume the same bytes and scales.

Workload shapes (attention: Hq query heads, Hkv KV heads, head dim D; indexer:
HI heads of dim dI; top-k budget k):

====  ======================  =====================================================
id    name                    shape
====  ======================  =====================================================
0     tiny                    L=512, Hq=8, Hkv=2, D=64, HI=4, dI=32, k=64
1     prefill-32k             L=32768, Hq=32, Hkv=4, D=128, HI=32, dI=64, k=2048
2     prefill-128k            L=131072, same layer
3     decode-b32              B=32 sequences, cached lengths U[32768, 262144],
                              page 64, same layer
4     multimodal-256k         L=262144, 16 frames x 256 tokens then 64 text tokens
====  ======================  =====================================================
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

PAGE = 64
E4M3_MAX = 448.0

# e4m3fn encodings of the small integers used by the exact-arithmetic inputs.
_E4M3_SMALL_INT = {0: 0x00, 1: 0x38, 2: 0x40, 3: 0x44, 4: 0x48}


@dataclass(frozen=True)
class Config:
    name: str
    L: int = 0
    Hq: int = 32
    Hkv: int = 4
    D: int = 128
    HI: int = 32
    dI: int = 64
    k: int = 2048
    B: int = 0
    len_lo: int = 0
    len_hi: int = 0
    seed: int = 0
    tiny: bool = False
    multimodal: bool = False

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


CONFIGS = {
    0: Config("tiny", L=512, Hq=8, Hkv=2, D=64, HI=4, dI=32, k=64, seed=1000, tiny=True),
    1: Config("prefill-32k", L=32768, seed=1001),
    2: Config("prefill-128k", L=131072, seed=1002),
    3: Config("decode-b32", B=32, len_lo=32768, len_hi=262144, seed=1003),
    4: Config("multimodal-256k", L=262144, seed=1004, multimodal=True),
}

# Structure of the multimodal workload: a period of 16 video frames of 256
# tokens each followed by a 64-token text segment, repeated from t = 0.
FRAME_TOKENS = 256
FRAMES_PER_GROUP = 16
TEXT_TOKENS = 64
PERIOD = FRAME_TOKENS * FRAMES_PER_GROUP + TEXT_TOKENS
FRAME_NOISE_STD = 0.05


def config(i: int, **over) -> Config:
    c = CONFIGS[i]
    return replace(c, **over) if over else c


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def quantize_e4m3_per_token(x: torch.Tensor):
    """Per-token e4m3fn packing: scale = absmax / 448 over all dims after the
    first (1 when the token is all zeros); bytes = round-to-nearest-even of
    x / scale.  Returns (uint8 bytes shaped like x, float32 scales [x.shape[0]])."""
    flat = x.reshape(x.shape[0], -1).float()
    amax = flat.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (flat / scale[:, None]).clamp_(-E4M3_MAX, E4M3_MAX)
    q = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(x.shape)
    return q.contiguous(), scale.contiguous()


def _frame_structured(L: int, width: tuple, g: torch.Generator, device) -> torch.Tensor:
    """Rows of a multimodal sequence: frame tokens are their frame's mean
    vector (N(0,1)) plus N(0, 0.05) noise, text tokens are N(0,1)."""
    t = torch.arange(L, device=device)
    p = t % PERIOD
    is_frame = p < FRAME_TOKENS * FRAMES_PER_GROUP
    frame_id = (t // PERIOD) * FRAMES_PER_GROUP + torch.div(p, FRAME_TOKENS, rounding_mode="floor")
    n_frames = int(frame_id.max().item()) + 1
    means = torch.randn((n_frames,) + width, generator=g, device=device)
    noise = torch.randn((L,) + width, generator=g, device=device)
    out = torch.where(is_frame.view((L,) + (1,) * len(width)),
                      means[frame_id.clamp(max=n_frames - 1)] + FRAME_NOISE_STD * noise, noise)
    return out


def prefill_inputs(cfg: Config, device="cpu", seed: int | None = None, L: int | None = None) -> dict:
    """Seeded prefill inputs.

    Returns a dict of tensors on ``device``:
      q8 [L,HI,dI] uint8 (e4m3fn), sq [L] f32, w [L,HI] f32,
      k8 [L,dI] uint8 (e4m3fn), sk [L] f32,
      Q [L,Hq,D], K [L,Hkv,D], V [L,Hkv,D] bfloat16.
    """
    L = cfg.L if L is None else L
    g = _gen(device, cfg.seed if seed is None else seed)
    qI = torch.randn(L, cfg.HI, cfg.dI, generator=g, device=device)
    if cfg.multimodal:
        kI = _frame_structured(L, (cfg.dI,), g, device)
    else:
        kI = torch.randn(L, cfg.dI, generator=g, device=device)
    if cfg.tiny:
        w = torch.rand(L, cfg.HI, generator=g, device=device)
    else:
        w = torch.rand(L, cfg.HI, generator=g, device=device) / cfg.HI
    q8, sq = quantize_e4m3_per_token(qI)
    del qI
    k8, sk = quantize_e4m3_per_token(kI)
    del kI
    std = 1.0 / math.sqrt(64.0) if cfg.tiny else 1.0
    Q = (torch.randn(L, cfg.Hq, cfg.D, generator=g, device=device) * std).to(torch.bfloat16)
    if cfg.multimodal:
        K = _frame_structured(L, (cfg.Hkv, cfg.D), g, device).to(torch.bfloat16)
        V = _frame_structured(L, (cfg.Hkv, cfg.D), g, device).to(torch.bfloat16)
    else:
        K = (torch.randn(L, cfg.Hkv, cfg.D, generator=g, device=device) * std).to(torch.bfloat16)
        V = (torch.randn(L, cfg.Hkv, cfg.D, generator=g, device=device) * std).to(torch.bfloat16)
    return dict(q8=q8, sq=sq, w=w.contiguous(), k8=k8, sk=sk, Q=Q, K=K, V=V)


def exact_indexer_inputs(L: int, HI: int, dI: int, seed: int, device="cpu",
                         key_pool: int | None = None) -> dict:
    """Indexer inputs on which every fp32 operation of any evaluation order is
    exact: e4m3 values in {0, +-1, +-2, +-3, +-4}, per-token scales in
    {1/2, 1, 2}, head weights in {2^-5, ..., 1}.  A dot product is an integer
    of magnitude <= 16*dI, each weighted term a multiple of 2^-5 * sq * sk, and
    the whole sum spans at most 24 bits, so the GPU's fp32 scores must equal
    the oracle's fp64 scores exactly.  With ``key_pool = n`` every key token
    (bytes and scale) is a copy of one of n distinct keys, so every row holds
    many exactly tied scores and the lower-index tie rule of the top-k decides
    which of them are selected."""
    g = _gen(device, seed)
    lut = torch.tensor([_E4M3_SMALL_INT[i] for i in range(5)], dtype=torch.uint8, device=device)

    def draw(shape):
        mag = torch.randint(0, 5, shape, generator=g, device=device)
        neg = torch.randint(0, 2, shape, generator=g, device=device).to(torch.uint8) * 0x80
        b = lut[mag] | neg
        return torch.where(mag == 0, torch.zeros_like(b), b)

    q8 = draw((L, HI, dI))
    k8 = draw((L, dI))
    sq = torch.pow(2.0, torch.randint(-1, 2, (L,), generator=g, device=device).float())
    sk = torch.pow(2.0, torch.randint(-1, 2, (L,), generator=g, device=device).float())
    w = torch.pow(2.0, -torch.randint(0, 6, (L, HI), generator=g, device=device).float())
    if key_pool:
        pick = torch.randint(0, key_pool, (L,), generator=g, device=device)
        k8 = k8[:key_pool][pick]
        sk = sk[:key_pool][pick]
    return dict(q8=q8.contiguous(), sq=sq, w=w.contiguous(), k8=k8.contiguous(), sk=sk)


def kl_targets(n_rows: int, G: int, width: int, seed: int, device="cpu", zero_frac: float = 0.3) -> torch.Tensor:
    """Non-negative target weights [n_rows, G, width] float32 for the
    indexer's distillation losses: U(0,1)^3 draws with a fraction of exact
    zeros (the loss normalises them; nothing here is normalised)."""
    g = _gen(device, seed)
    x = torch.rand(n_rows, G, width, generator=g, device=device) ** 3
    z = torch.rand(n_rows, G, width, generator=g, device=device) < zero_frac
    return torch.where(z, torch.zeros_like(x), x).contiguous()


def tie_heavy_scores(n_rows: int, width: int, seed: int, device="cpu") -> torch.Tensor:
    """fp32 score rows for exercising the top-k alone: a mix of clustered
    duplicates, signed zeros, negatives and a few large values."""
    g = _gen(device, seed)
    base = torch.randint(-8, 9, (n_rows, width), generator=g, device=device).float() * 0.25
    mode = torch.randint(0, 4, (n_rows, 1), generator=g, device=device)
    cont = torch.randn(n_rows, width, generator=g, device=device)
    x = torch.where(mode == 0, cont, base)
    zero_mask = torch.rand(n_rows, width, generator=g, device=device) < 0.1
    sign_mask = torch.rand(n_rows, width, generator=g, device=device) < 0.5
    zeros = torch.where(sign_mask, torch.tensor(-0.0, device=device), torch.tensor(0.0, device=device))
    x = torch.where(zero_mask, zeros, x)
    return x.contiguous()


def decode_inputs(cfg: Config, device="cpu", seed: int | None = None, B: int | None = None,
                  seq_lens=None, len_lo: int | None = None, len_hi: int | None = None,
                  spare_pages: int = 3) -> dict:
    """Seeded decode inputs over a paged cache (page = 64 tokens).

    Pages are dealt to sequences in a random order, so consecutive logical
    pages of one sequence are scattered through the cache.  Returns a dict:
      q [B,Hq,D] bf16, q8 [B,HI,dI] uint8, sq [B] f32, w [B,HI] f32,
      k8_cache [P,64,dI] uint8, sk_cache [P,64] f32,
      k_cache, v_cache [P,64,Hkv,D] bf16, block_table [B,max_pages] int32
      (-1 past the end), seq_lens [B] int32, max_seq_len (int), num_pages (int).
    The query token sits at position seq_len-1, already in the cache.
    """
    g = _gen(device, cfg.seed if seed is None else seed)
    if seq_lens is not None:
        B = len(seq_lens)
    B = cfg.B if B is None else B
    lo = cfg.len_lo if len_lo is None else len_lo
    hi = cfg.len_hi if len_hi is None else len_hi
    if seq_lens is None:
        lens = torch.randint(lo, hi + 1, (B,), generator=g, device=device).to(torch.int32)
    else:
        lens = torch.as_tensor(seq_lens, dtype=torch.int32, device=device)
    lens_host = [int(v) for v in lens.cpu()]
    pages = [(n + PAGE - 1) // PAGE for n in lens_host]
    max_pages = max(1, max(pages) if pages else 1)
    P = sum(pages) + spare_pages
    perm = torch.randperm(P, generator=g, device=device).to(torch.int32)
    bt = torch.full((B, max_pages), -1, dtype=torch.int32, device=device)
    off = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[off: off + n]
        off += n
    kI = torch.randn(P * PAGE, cfg.dI, generator=g, device=device)
    k8, sk = quantize_e4m3_per_token(kI)
    del kI
    std = 1.0 / math.sqrt(64.0) if cfg.tiny else 1.0
    k_cache = (torch.randn(P, PAGE, cfg.Hkv, cfg.D, generator=g, device=device) * std).to(torch.bfloat16)
    v_cache = (torch.randn(P, PAGE, cfg.Hkv, cfg.D, generator=g, device=device) * std).to(torch.bfloat16)
    qI = torch.randn(B, cfg.HI, cfg.dI, generator=g, device=device)
    q8, sq = quantize_e4m3_per_token(qI)
    if cfg.tiny:
        w = torch.rand(B, cfg.HI, generator=g, device=device)
    else:
        w = torch.rand(B, cfg.HI, generator=g, device=device) / cfg.HI
    q = (torch.randn(B, cfg.Hq, cfg.D, generator=g, device=device) * std).to(torch.bfloat16)
    return dict(q=q, q8=q8, sq=sq, w=w.contiguous(),
                k8_cache=k8.reshape(P, PAGE, cfg.dI).contiguous(), sk_cache=sk.reshape(P, PAGE).contiguous(),
                k_cache=k_cache, v_cache=v_cache, block_table=bt, seq_lens=lens,
                max_seq_len=max(lens_host) if lens_host else 0, num_pages=P)


def to_numpy_bits(t: torch.Tensor):
    """Host numpy view of a tensor; bf16 becomes its uint16 bit pattern."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()
