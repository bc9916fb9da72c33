"""Seeded synthetic inputs for the routed KV write and routed attention.

This module only draws random inputs; it holds none of the quantization or attention
arithmetic, and it serves both the CUDA path and the CPU oracle (which receive the same
bytes).

Workloads are shaped like the decoders in the TriRoute paper review page, section 5
(model table: 160M with d=768, H=12, head_dim 64; 1.3B with d=2048, H=16, head_dim 128;
sequence length 2048, long-context evaluation at 8k). The pages train on the Pile and
RedPajama; no dataset is read here: K/V/Q are i.i.d. normal fp16 values, with 1% of the
channels scaled by 8 in the outlier workloads, and bits / modes are i.i.d. categorical
draws with the stated probabilities.

Recipe (all draws from torch.Generator streams keyed by (seed, stream, sequence)):
  - values:  torch.randn in fp32, outlier channels multiplied by 8, rounded to fp16;
  - outlier channels: round(0.01 * H * D) distinct indices of the flattened (head,
    channel) axis, drawn once per tensor (Q, K, V separately) and fixed across tokens;
  - bits:    i.i.d. per (token, head) over {2, 4, 8, 16};
  - modes:   i.i.d. per (token, head) for prefill, per (sequence, head) for decode.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

BIT_VALUES = (2, 4, 8, 16)
MODE_SKIP, MODE_LOCAL, MODE_FULL = 0, 1, 2

# stream ids
_S_Q, _S_K, _S_V, _S_OQ, _S_OK, _S_OV, _S_BITS, _S_MODES, _S_DQ, _S_DMODES = range(1, 11)
_S_ZA, _S_ZB = 11, 12


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "prefill" or "decode"
    seqlens: tuple            # tokens per sequence (decode: cached context incl. the query token)
    heads: int
    head_dim: int
    w: int
    bits_p: tuple             # probabilities of 2/4/8/16 bits
    modes_p: tuple            # probabilities of skip/local/full
    outliers: bool
    seed: int
    note: str = ""

    @property
    def batch(self) -> int:
        return len(self.seqlens)

    @property
    def n_tok(self) -> int:
        return int(sum(self.seqlens))


WORKLOADS = {
    "tiny_prefill": Workload(
        "tiny_prefill", "prefill", (256,), 4, 64, 32, (0.25, 0.25, 0.25, 0.25),
        (1 / 3, 1 / 3, 1 / 3), False, 1001,
        "B=1, H=4, head_dim=64, T=256, w=32, bits and modes uniform"),
    "prefill_160m": Workload(
        "prefill_160m", "prefill", (2048,) * 8, 12, 64, 256, (0.3, 0.4, 0.2, 0.1),
        (0.2, 0.4, 0.4), True, 1002,
        "160M-like prefill: B=8, H=12, head_dim=64, T=2048, w=256, 1% outlier channels x8"),
    "decode_1p3b": Workload(
        "decode_1p3b", "decode", (8192,) * 64, 16, 128, 512, (0.25, 0.45, 0.2, 0.1),
        (0.15, 0.45, 0.4), False, 1003,
        "1.3B-like decode: batch 64, H=16, head_dim=128, context 8192, w=512"),
    "decode_long": Workload(
        "decode_long", "decode", (65536,) * 8, 16, 128, 1024, (0.5, 0.35, 0.1, 0.05),
        (0.1, 0.6, 0.3), False, 1004,
        "long-context decode: batch 8, H=16, head_dim=128, context 65536, w=1024"),
    "ragged_prefill": Workload(
        "ragged_prefill", "prefill", (1024, 3000, 8192, 5555), 16, 128, 512,
        (0.3, 0.4, 0.2, 0.1), (0.2, 0.4, 0.4), True, 1005,
        "ragged prefill + write: lengths {1024, 3000, 8192, 5555}, H=16, head_dim=128, "
        "w=512, 1% outlier channels x8"),
}


def _gen(seed: int, stream: int, index: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + stream * 65_537 + index) % (2**63 - 1))
    return g


def outlier_channels(heads: int, head_dim: int, seed: int, stream: int) -> torch.Tensor:
    """round(1% of heads*head_dim) distinct flattened channel indices (CPU int64)."""
    n = int(round(0.01 * heads * head_dim))
    g = _gen(seed, stream, 0, "cpu")
    return torch.randperm(heads * head_dim, generator=g)[:n]


def normal_fp16(shape, seed: int, stream: int, index: int, device,
                outlier_idx: torch.Tensor | None = None, outlier_scale: float = 8.0):
    """fp16 N(0,1) draws of shape [..., H, D]; listed flattened (H, D) channels scaled."""
    g = _gen(seed, stream, index, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if outlier_idx is not None and outlier_idx.numel() > 0:
        H, D = shape[-2], shape[-1]
        scale = torch.ones(H * D, device=device, dtype=torch.float32)
        scale[outlier_idx.to(device)] = outlier_scale
        x = x * scale.view(H, D)
    return x.to(torch.float16)


def categorical(shape, probs, values, seed: int, stream: int, index: int, device):
    """i.i.d. draws from `values` with probabilities `probs` (uint8 tensor)."""
    g = _gen(seed, stream, index, device)
    u = torch.rand(shape, generator=g, device=device, dtype=torch.float64)
    cum = torch.tensor(probs, dtype=torch.float64, device=device).cumsum(0)[:-1]
    idx = torch.bucketize(u, cum, right=True)
    table = torch.tensor(values, dtype=torch.uint8, device=device)
    return table[idx]


def cu_seqlens(seqlens, device="cpu") -> torch.Tensor:
    c = [0]
    for n in seqlens:
        c.append(c[-1] + int(n))
    return torch.tensor(c, dtype=torch.int32, device=device)


def kv_tokens(wl: Workload, device, seq_range=None):
    """K, V fp16 [n_tok, H, D] and bits uint8 [n_tok, H] for every token of the workload,
    drawn per sequence (so any subset of sequences can be regenerated alone)."""
    H, D = wl.heads, wl.head_dim
    ok = outlier_channels(H, D, wl.seed, _S_OK) if wl.outliers else None
    ov = outlier_channels(H, D, wl.seed, _S_OV) if wl.outliers else None
    seqs = range(wl.batch) if seq_range is None else seq_range
    ks, vs, bs = [], [], []
    for s in seqs:
        L = wl.seqlens[s]
        ks.append(normal_fp16((L, H, D), wl.seed, _S_K, s, device, ok))
        vs.append(normal_fp16((L, H, D), wl.seed, _S_V, s, device, ov))
        bs.append(categorical((L, H), wl.bits_p, BIT_VALUES, wl.seed, _S_BITS, s, device))
    return torch.cat(ks), torch.cat(vs), torch.cat(bs)


def widths(wl: Workload, s: int, device):
    """bits uint8 [L_s, H] of sequence s alone (the same draws as kv_tokens on `device`)."""
    return categorical((wl.seqlens[s], wl.heads), wl.bits_p, BIT_VALUES, wl.seed, _S_BITS, s, device)


def kv_sequence(wl: Workload, s: int, device):
    """K, V [L_s, H, D] and bits [L_s, H] of sequence s alone (same values as kv_tokens)."""
    return kv_tokens(wl, device, seq_range=[s])


def prefill_queries(wl: Workload, device, seq_range=None):
    """Q fp16 [n_tok, H, D] and per-(token, head) modes uint8 [n_tok, H]."""
    H, D = wl.heads, wl.head_dim
    oq = outlier_channels(H, D, wl.seed, _S_OQ) if wl.outliers else None
    seqs = range(wl.batch) if seq_range is None else seq_range
    qs, ms = [], []
    for s in seqs:
        L = wl.seqlens[s]
        qs.append(normal_fp16((L, H, D), wl.seed, _S_Q, s, device, oq))
        ms.append(categorical((L, H), wl.modes_p, (MODE_SKIP, MODE_LOCAL, MODE_FULL),
                              wl.seed, _S_MODES, s, device))
    return torch.cat(qs), torch.cat(ms)


def decode_queries(wl: Workload, device):
    """Q fp16 [B, H, D] N(0,1) and per-(sequence, head) modes uint8 [B, H]."""
    H, D = wl.heads, wl.head_dim
    q = normal_fp16((wl.batch, H, D), wl.seed, _S_DQ, 0, device)
    modes = categorical((wl.batch, H), wl.modes_p, (MODE_SKIP, MODE_LOCAL, MODE_FULL),
                        wl.seed, _S_DMODES, 0, device)
    return q, modes


def router_logits(wl: Workload, device, ties: bool = True):
    """Synthetic controller logits per (token, head): z_attn fp32 [n_tok, H, 3] and z_bits
    fp32 [n_tok, H, 4], N(0, 1). With ties=True every 8th row is rounded to multiples of
    0.5, so tied maxima occur. (Trained controller weights are not available; these only
    exercise the argmax.)"""
    out = []
    for stream, k in ((_S_ZA, 3), (_S_ZB, 4)):
        g = _gen(wl.seed, stream, 0, device)
        z = torch.randn((wl.n_tok, wl.heads, k), generator=g, device=device, dtype=torch.float32)
        if ties:
            z[::8] = torch.round(z[::8] * 2) / 2
        out.append(z)
    return out[0], out[1]


def scaled(wl: Workload, seqlens=None, heads=None, name=None) -> Workload:
    """Same distributions at other shapes (smaller parity cases of a workload)."""
    from dataclasses import replace
    return replace(wl, seqlens=tuple(seqlens) if seqlens is not None else wl.seqlens,
                   heads=heads if heads is not None else wl.heads,
                   name=name or wl.name + "_scaled")
