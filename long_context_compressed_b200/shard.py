"""Decode of one long sequence whose compressed entries are split over G GPUs.

Each GPU holds a contiguous range [lo, hi) of the compressed entries (index keys and
latent rows).  One decode step, on every GPU (all of its arithmetic runs in the
library's kernels; this module only orders the calls and the exchanges):

1. the indexer over the local entries, the local top-k (e4m3 scores of Hadamard-rotated
   queries and keys, exact bf16 rescoring of the kc = 2k candidates as in the single-GPU
   step), which also returns the exact scores of the local winners, and their global
   entry numbers;
2. one all-gather of the (score, global index) pairs, then the global top-k
   (csa_shard_select), the same on every GPU.  Every global winner is a local winner of
   its shard, so the gathered lists hold the whole-row top-k, and with the shards in
   entry order the lower-index tie rule still holds;
3. the winners inside [lo, hi) as local indices, and the attention over them without
   the sink (sparse_attn_partial); the SWA rows are attended on GPU 0 only;
4. one all-gather of the partial results (output and (m, l) in one buffer), then
   csa_attn_combine adds the sink once and every GPU holds the output.

The identity behind 3-4 is the attention-sink probability of "DeepSeek-V4 混合注意力：
从压缩记忆到百万上下文" §6 over a union of disjoint row sets.  The exchanges go through an
``exchange`` object with one method, ``all_gather(t) -> [G, *t.shape]``:
``TorchDistExchange`` uses torch.distributed (NCCL between GPUs).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


def shard_range(N: int, G: int, g: int) -> tuple[int, int]:
    """Contiguous entry range [lo, hi) of shard g when N entries are split over G shards."""
    if not (0 <= g < G):
        raise ValueError(f"shard {g} of {G}")
    return g * N // G, (g + 1) * N // G


class TorchDistExchange:
    """all_gather over a torch.distributed process group (NCCL for CUDA tensors)."""

    def __init__(self, group=None):
        self.group = group

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        import torch.distributed as dist
        G = dist.get_world_size(self.group)
        flat = torch.empty(G * t.numel(), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(flat, t.contiguous().view(-1), group=self.group)
        return flat.view((G,) + tuple(t.shape))


@dataclass
class Shard:
    """Resident state of one GPU's shard (B sequences, one query each)."""
    rank: int
    world: int
    lo: int
    hi: int
    kI: torch.Tensor          # [B, Ns, 128] bf16 index keys of the shard
    kv: torch.Tensor          # [B, Ns, D] bf16 latent rows (or [B, Ns, 608] KV8 entries)
    swa: torch.Tensor         # [B, W, D] bf16 raw SWA rows (used on rank 0 only)
    swa_pos0: torch.Tensor    # [B] int64
    q_pos: torch.Tensor       # [B, 1] int64
    sink: torch.Tensor        # [H] fp32
    n_valid: torch.Tensor     # [B, 1] int32, visible entries of this shard (csa_n_valid with [lo, hi))
    k8: torch.Tensor | None = None
    ks: torch.Tensor | None = None


class GpuKernels:
    """The library's calls for one shard; buffers are allocated on first use and kept."""

    def __init__(self, k: int, scale: float, hadamard: bool = True):
        self.k, self.scale, self.hadamard = k, scale, hadamard
        self.buf: dict = {}

    def _b(self, name, shape, dtype, device, zero=False):
        t = self.buf.get(name)
        if t is None or t.shape != torch.Size(shape) or t.dtype != dtype:
            t = (torch.zeros if zero else torch.empty)(shape, dtype=dtype, device=device)
            self.buf[name] = t
        return t

    def local_topk(self, sh: Shard, qI, w):
        """The shard's k best entries as (score, global index) pairs [B, k, 2] int32."""
        from . import csa
        B, Ns, dev, k = sh.kI.shape[0], sh.kI.shape[1], sh.kI.device, self.k
        if sh.k8 is None:
            sh.k8, sh.ks = csa.csa_quantize_e4m3(sh.kI, hadamard=self.hadamard)
        q8 = self._b("q8", qI.shape, torch.uint8, dev)
        qs = self._b("qs", qI.shape[:-1], torch.float32, dev)
        csa.csa_quantize_e4m3(qI, codes=q8, scale=qs, hadamard=self.hadamard)
        scores = self._b("scores", (B, 1, Ns), torch.float32, dev)
        ws = self.buf.get("select_ws")
        if ws is None:
            ws = self.buf["select_ws"] = csa.select_workspace(B, Ns, dev)
        csa.csa_index_scores(q8, w, sh.k8, sh.n_valid, q_scale=qs, k_scale=sh.ks, scores=scores, select_ws=ws)
        loc = self._b("loc", (B, 1, k), torch.int32, dev)
        exact = self._b("exact", (B, 1, k), torch.float32, dev)
        csa.csa_topk_select(scores, sh.n_valid, k, ws, kc=2 * k, qI=qI, w=w, kI=sh.kI, idx=loc, idx_scores=exact)
        pairs = csa.shard_pack(exact, loc, Ns, sh.lo, pairs=self._b("pairs", (B, k, 2), torch.int32, dev))
        return pairs

    def attend(self, sh: Shard, q, all_pairs):
        """This shard's part of the attention over the global top-k, written into one
        buffer (output, then (m, l)) -> uint8 [nbytes]."""
        from . import csa
        B, dev, k = q.shape[0], q.device, self.k
        g = csa.shard_select(all_pairs, k, idx=self._b("glob", (B, k), torch.int32, dev))
        loc = csa.shard_remap(g, sh.lo, sh.hi, 0, out=self._b("sel", (B, 1, k), torch.int32, dev))
        if "part" not in self.buf or self.buf["part"][1].shape != q.shape:
            self.buf["part"] = csa.pack_partial_views(tuple(q.shape), dev)
        buf, out, ml = self.buf["part"]
        csa.sparse_attn_partial(q, sh.kv, sh.swa, sh.swa_pos0, sh.q_pos, loc, self.scale, with_swa=(sh.rank == 0),
                                out=out, ml=ml)
        return buf

    def combine(self, sh: Shard, gathered, shape):
        from . import csa
        return csa.attn_combine_packed(gathered, shape, sh.sink)


def decode_step(sh: Shard, kernels, exchange, q, qI, w):
    """One decode step of the sharded sequence(s) on this GPU; returns the full output
    [B, 1, H, D] (identical on every GPU).  Two all-gathers per step."""
    pairs = kernels.local_topk(sh, qI, w)
    part = kernels.attend(sh, q, exchange.all_gather(pairs))
    return kernels.combine(sh, exchange.all_gather(part), tuple(q.shape))


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
