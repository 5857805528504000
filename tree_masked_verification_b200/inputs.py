"""Seeded synthetic inputs for Hybrid Tree Attention verification calls.

This module draws the random tensors and tree shapes that both the CUDA path
and the CPU oracle consume.  It holds none of the attention arithmetic: only
random draws, rounding to bf16 and the tree topology.

Recipe (every workload):
  * One ``torch.Generator('cpu')`` per (seed, stream, b, head), seeded from
    ``numpy.random.SeedSequence([seed, stream, b, head])``.  So one head's
    K/V can be regenerated alone (sampled parity at full size), and the bytes
    do not depend on the device.
  * Q, K, V drawn N(0, 1) in fp32 and rounded to bf16 (round to nearest even,
    by torch).  In "peaked" workloads each K row (prefix and tree keys alike)
    is multiplied in fp32 by one scalar 1 + |N(0, 1)| before the rounding.
  * Trees: "levels" -- node ids in breadth-first level order, level widths
    ``widths`` (4 16 16 16 16 -> 68 nodes, the ``--tree_shape`` of the LongSpec
    README's evaluation commands); level-1 nodes hang off the prefix end
    (parent -1) and each deeper node's parent is uniform over the previous
    level's ids.  "random" -- node 0 has parent -1, node i >= 1 a parent
    uniform over 0..i-1.  "chain" -- parent[i] = i - 1.
  * Prefix lengths: fixed L, or uniform integers in [lo, hi] per sequence.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional, Tuple

import numpy as np
import torch

# stream ids of the random draws
_S_Q, _S_KP, _S_VP, _S_KT, _S_VT, _S_KSCALE, _S_TREE, _S_LEN = range(8)

LONGSPEC_TREE_SHAPE = (4, 16, 16, 16, 16)


def _generator(seed: int, stream: int, b: int = 0, h: int = 0) -> torch.Generator:
    state = np.random.SeedSequence([int(seed), int(stream), int(b), int(h)])
    g = torch.Generator(device="cpu")
    g.manual_seed(int(state.generate_state(1, dtype=np.uint64)[0] & ((1 << 63) - 1)))
    return g


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (no copy of values' meaning)."""
    if t.dtype != torch.bfloat16:
        raise TypeError("expected a bf16 tensor")
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def tree_levels(widths, g: torch.Generator) -> np.ndarray:
    parent = []
    prev = []
    nid = 0
    for lvl, w in enumerate(widths):
        cur = list(range(nid, nid + w))
        for _ in cur:
            if lvl == 0:
                parent.append(-1)
            else:
                k = int(torch.randint(len(prev), (1,), generator=g).item())
                parent.append(prev[k])
        prev = cur
        nid += w
    return np.asarray(parent, dtype=np.int32)


def tree_random(T: int, g: torch.Generator) -> np.ndarray:
    parent = [-1] if T > 0 else []
    for i in range(1, T):
        parent.append(int(torch.randint(i, (1,), generator=g).item()))
    return np.asarray(parent, dtype=np.int32)


def tree_chain(T: int) -> np.ndarray:
    return np.arange(-1, T - 1, dtype=np.int32)


@dataclass(frozen=True)
class Workload:
    """Shapes and seed of one verification-attention call.

    q [B][Hq][T][D], k/v_prefix [B][Hkv][L_cap][D], k/v_tree [B][Hkv][T][D],
    prefix_len [B], parent [B][T]; bf16 tensors, int32 index arrays.
    """
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    T: int
    L_cap: int
    seed: int
    tree: str = "levels"                      # levels | random | chain
    widths: Tuple[int, ...] = LONGSPEC_TREE_SHAPE
    prefix_range: Optional[Tuple[int, int]] = None   # None -> every L_b = L_cap
    k_peaked: bool = False
    scale: float = 0.0                        # 0 -> 1/sqrt(D)
    # "verify": prefix + tree (longspec_hta_verify); "prefix": the T query
    # tokens attend to the prefix alone (longspec_hta_prefix_attention, the
    # draft model's cross-attention into the target's KV cache)
    kind: str = "verify"
    # "window": the draft model's sliding-window self-attention over the tree
    # (longspec_hta_window_verify): k/v_prefix is the ring of W = L_cap slots
    # and prefix_len the context length, which may exceed W
    # > 0: the prefix K/V in a paged cache of blocks of this many keys
    # (longspec_hta_verify_paged / _prefix_attention_paged)
    block_size: int = 0

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    # ---- index inputs -------------------------------------------------
    def prefix_lens(self) -> np.ndarray:
        if self.prefix_range is None:
            return np.full((self.B,), self.L_cap, dtype=np.int32)
        lo, hi = self.prefix_range
        g = _generator(self.seed, _S_LEN)
        return torch.randint(lo, hi + 1, (self.B,), generator=g).to(torch.int32).numpy()

    def visible_lens(self) -> np.ndarray:
        """Context keys a call must read per sequence: L_b, or for a
        sliding-window call the min(L_b, W - 1) positions in some row's window."""
        lens = self.prefix_lens()
        if self.kind == "window":
            return np.minimum(lens, self.L_cap - 1).astype(np.int32)
        return lens

    def parents(self) -> np.ndarray:
        out = np.zeros((self.B, self.T), dtype=np.int32)
        for b in range(self.B):
            g = _generator(self.seed, _S_TREE, b)
            if self.tree == "levels":
                if sum(self.widths) != self.T:
                    raise ValueError("level widths do not add up to T")
                out[b] = tree_levels(self.widths, g)
            elif self.tree == "random":
                out[b] = tree_random(self.T, g)
            elif self.tree == "chain":
                out[b] = tree_chain(self.T)
            else:
                raise ValueError(f"unknown tree kind {self.tree}")
        return out

    # ---- per-head random tensors ------------------------------------------
    def _key_scale(self, b: int, kvh: int) -> torch.Tensor:
        g = _generator(self.seed, _S_KSCALE, b, kvh)
        return 1.0 + torch.randn(self.L_cap + self.T, generator=g).abs()

    def q_head(self, b: int, h: int) -> torch.Tensor:
        g = _generator(self.seed, _S_Q, b, h)
        return torch.randn(self.T, self.D, generator=g).to(torch.bfloat16)

    def k_prefix_head(self, b: int, kvh: int) -> torch.Tensor:
        g = _generator(self.seed, _S_KP, b, kvh)
        k = torch.randn(self.L_cap, self.D, generator=g)
        if self.k_peaked:
            k *= self._key_scale(b, kvh)[: self.L_cap, None]
        return k.to(torch.bfloat16)

    def v_prefix_head(self, b: int, kvh: int) -> torch.Tensor:
        g = _generator(self.seed, _S_VP, b, kvh)
        return torch.randn(self.L_cap, self.D, generator=g).to(torch.bfloat16)

    def k_tree_head(self, b: int, kvh: int) -> torch.Tensor:
        g = _generator(self.seed, _S_KT, b, kvh)
        k = torch.randn(self.T, self.D, generator=g)
        if self.k_peaked:
            k *= self._key_scale(b, kvh)[self.L_cap:, None]
        return k.to(torch.bfloat16)

    def v_tree_head(self, b: int, kvh: int) -> torch.Tensor:
        g = _generator(self.seed, _S_VT, b, kvh)
        return torch.randn(self.T, self.D, generator=g).to(torch.bfloat16)

    # ---- whole tensors ------------------------------------------------
    def generate(self, with_prefix: bool = True) -> dict:
        """All inputs as CPU tensors (bf16 / int32)."""
        B, Hq, Hkv, D, T, L = self.B, self.Hq, self.Hkv, self.D, self.T, self.L_cap
        q = torch.empty(B, Hq, T, D, dtype=torch.bfloat16)
        kt = torch.empty(B, Hkv, T, D, dtype=torch.bfloat16)
        vt = torch.empty(B, Hkv, T, D, dtype=torch.bfloat16)
        for b in range(B):
            for h in range(Hq):
                q[b, h] = self.q_head(b, h)
            for h in range(Hkv):
                kt[b, h] = self.k_tree_head(b, h)
                vt[b, h] = self.v_tree_head(b, h)
        out = dict(q=q, k_tree=kt, v_tree=vt,
                   prefix_len=torch.from_numpy(self.prefix_lens()),
                   parent=torch.from_numpy(self.parents()))
        if with_prefix:
            kp = torch.empty(B, Hkv, L, D, dtype=torch.bfloat16)
            vp = torch.empty(B, Hkv, L, D, dtype=torch.bfloat16)
            for b in range(B):
                for h in range(Hkv):
                    kp[b, h] = self.k_prefix_head(b, h)
                    vp[b, h] = self.v_prefix_head(b, h)
            out["k_prefix"] = kp
            out["v_prefix"] = vp
        return out

    def generate_head(self, b: int, kvh: int) -> dict:
        """Inputs restricted to one (b, KV head): the G query heads of that
        group and that head's prefix/tree K, V, as a B=1, Hkv=1 problem."""
        G = self.Hq // self.Hkv
        q = torch.stack([self.q_head(b, kvh * G + g) for g in range(G)])[None]
        return dict(
            q=q,
            k_prefix=self.k_prefix_head(b, kvh)[None, None],
            v_prefix=self.v_prefix_head(b, kvh)[None, None],
            k_tree=self.k_tree_head(b, kvh)[None, None],
            v_tree=self.v_tree_head(b, kvh)[None, None],
            prefix_len=torch.from_numpy(self.prefix_lens()[b:b + 1].copy()),
            parent=torch.from_numpy(self.parents()[b:b + 1].copy()),
        )

    # ---- sizes ------------------------------------------------------------
    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def algorithmic_bytes(self) -> int:
        """Bytes one call must move at minimum: prefix K+V of the L_b keys
        actually present, Q, tree K+V, out (bf16), lse (fp32), parent and
        prefix_len (int32)."""
        lens = self.visible_lens().astype(np.int64)
        kv = int(2 * self.Hkv * self.D * 2 * lens.sum())
        q = self.B * self.Hq * self.T * self.D * 2
        tree = 2 * self.B * self.Hkv * self.T * self.D * 2
        out = self.B * self.Hq * self.T * self.D * 2
        lse = self.B * self.Hq * self.T * 4
        idx = self.B * self.T * 4 + self.B * 4
        if self.kind == "prefix":   # no tree K/V, no parent array
            return kv + q + out + lse + self.B * 4
        return kv + q + tree + out + lse + idx


# The attention shapes of the models the LongSpec pages evaluate, with the
# pages' 4/16/16/16/16 draft tree.  The datasets of the pages (LongBench,
# RepoBench-P, AIME24, MATH500) are not used: these draws stand in for them.
WORKLOADS = {
    "tiny": Workload("tiny", B=1, Hq=2, Hkv=1, D=64, T=8, L_cap=256, seed=0,
                     tree="random"),
    "llama3-8b-32k": Workload("llama3-8b-32k", B=1, Hq=32, Hkv=8, D=128,
                              T=68, L_cap=32768, seed=1),
    "vicuna-7b-b8": Workload("vicuna-7b-b8", B=8, Hq=32, Hkv=32, D=128, T=68,
                             L_cap=16384, seed=2, prefix_range=(8192, 16384)),
    "qwq-32b-32k-peaked": Workload("qwq-32b-32k-peaked", B=1, Hq=40, Hkv=8,
                                   D=128, T=68, L_cap=32768, seed=3,
                                   k_peaked=True),
    "ultra-256k": Workload("ultra-256k", B=1, Hq=32, Hkv=8, D=128, T=68,
                           L_cap=262144, seed=4),
    "ultra-256k-chain5": Workload("ultra-256k-chain5", B=1, Hq=32, Hkv=8,
                                  D=128, T=5, L_cap=262144, seed=5,
                                  tree="chain"),
    # the Llama-3-8B call with the prefix in a paged cache of 16-key blocks
    "llama3-8b-32k-paged16": Workload("llama3-8b-32k-paged16", B=1, Hq=32, Hkv=8, D=128,
                                      T=68, L_cap=32768, seed=1, block_size=16),
    # the draft model's cross-attention into the Llama-3-8B target's KV
    # cache: 4 draft tokens per head, no tree keys
    "draft-xattn-32k": Workload("draft-xattn-32k", B=1, Hq=32, Hkv=8, D=128,
                                T=4, L_cap=32768, seed=6, tree="chain",
                                kind="prefix"),
    # the draft model's sliding-window (512) self-attention over the tree,
    # 32k tokens of context, its K/V ring of 512 slots per KV head
    "draft-window-512": Workload("draft-window-512", B=1, Hq=32, Hkv=8, D=128,
                                 T=68, L_cap=512, seed=8, prefix_range=(32768, 32768),
                                 kind="window"),
}


def paged_cache(k_prefix: torch.Tensor, v_prefix: torch.Tensor, prefix_lens, block_size: int,
                seed: int, spare_blocks: int = 3, reserve: int = 0):
    """The contiguous prefix K/V [B][Hkv][L_cap][D] laid out as a paged cache:
    k/v_cache [num_blocks][Hkv][block_size][D] and block_table [B][max_blocks]
    (int32), the blocks of all sequences shuffled by a seeded permutation,
    with `spare_blocks` unused blocks of noise mixed in.  Each sequence gets
    blocks for its L_b keys plus `reserve` more positions (room for tokens
    appended later), capped at L_cap.  Table entries past a sequence's last
    block are -1 (never read).  Pure data movement."""
    B, Hkv, L_cap, D = k_prefix.shape
    max_blocks = -(-L_cap // block_size)
    lens = [int(x) for x in prefix_lens]
    used = [-(-min(L + reserve, L_cap) // block_size) for L in lens]
    n = sum(used) + spare_blocks
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n, generator=g)
    k_cache = torch.randn((n, Hkv, block_size, D), generator=g).to(torch.bfloat16)
    v_cache = torch.randn((n, Hkv, block_size, D), generator=g).to(torch.bfloat16)
    table = torch.full((B, max_blocks), -1, dtype=torch.int32)
    nxt = 0
    for b in range(B):
        for i in range(used[b]):
            blk = int(perm[nxt]); nxt += 1
            table[b, i] = blk
            k0, k1 = i * block_size, min((i + 1) * block_size, L_cap)
            k_cache[blk, :, :k1 - k0] = k_prefix[b, :, k0:k1]
            v_cache[blk, :, :k1 - k0] = v_prefix[b, :, k0:k1]
    return k_cache, v_cache, table



# greedy acceptance after a verification call: (B, T, V); T is the LongSpec
# tree's 68 nodes, V the target model's vocabulary
ACCEPT_WORKLOADS = {
    "accept-llama3-t68": (1, 68, 128256),
    "accept-vicuna-b8": (8, 68, 32000),
}


def accept_inputs(B: int, T: int, V: int, seed: int, tree: str = "levels",
                  widths: Tuple[int, ...] = LONGSPEC_TREE_SHAPE, p_match: float = 0.8):
    """Seeded inputs of greedy tree acceptance: logits bf16 [B][T+1][V]
    (row 0: the prefix end, row 1+i: after node i), draft_tokens and parent
    int32 [B][T].  Every row gets a planted top token (logit 8 among N(0,1)
    draws, so it is the row's unique maximum in practice); a node's draft
    token is its parent row's planted token with probability p_match, else a
    random token.  Also returns the planted tokens [B][T+1]."""
    g = torch.Generator().manual_seed(seed)
    logits = torch.randn((B, T + 1, V), generator=g)
    top = torch.randint(0, V, (B, T + 1), generator=g)
    logits.scatter_(2, top[..., None], 8.0)
    wl = Workload("accept", B=B, Hq=1, Hkv=1, D=64, T=T, L_cap=0, seed=seed, tree=tree,
                  widths=widths)
    parent = torch.from_numpy(wl.parents().copy())
    rows = torch.where(parent < 0, torch.zeros_like(parent), parent + 1).long()
    want = torch.gather(top, 1, rows)
    coin = torch.rand((B, T), generator=g) < p_match
    other = torch.randint(0, V, (B, T), generator=g)
    draft = torch.where(coin, want, other).to(torch.int32)
    return dict(logits=logits.to(torch.bfloat16), draft_tokens=draft, parent=parent.to(torch.int32),
                planted=top.to(torch.int32))


def commit_inputs(w: "Workload", seed: int, full_prefix: bool = False):
    """Seeded inputs of the KV commit after acceptance: the workload's
    prefix cache, prefix lengths and tree K/V (``w.generate()``), plus, per
    sequence, an accepted path: the root path of a node drawn uniformly from
    the tree (node ids from depth 1), or no path with probability 1/8.
    Returns the generate() dict plus accept_len int32 [B] and path int32
    [B][T] (-1 past accept_len)."""
    inp = w.generate()
    g = torch.Generator().manual_seed(seed)
    par = inp["parent"].numpy()
    B, T = par.shape
    path = np.full((B, T), -1, dtype=np.int32)
    n = np.zeros(B, dtype=np.int32)
    for b in range(B):
        if torch.rand((), generator=g).item() < 0.125:
            continue
        j = int(torch.randint(0, T, (), generator=g))
        chain = []
        while j != -1:
            chain.append(j)
            j = int(par[b, j])
        chain.reverse()
        n[b] = len(chain)
        path[b, :len(chain)] = chain
    inp["accept_len"] = torch.from_numpy(n)
    inp["path"] = torch.from_numpy(path)
    return inp


def window_ring(k_ctx: torch.Tensor, v_ctx: torch.Tensor, prefix_lens, W: int):
    """The last W positions of each sequence's context K/V [B][Hkv][L_max][D]
    as a ring [B][Hkv][W][D]: position p at slot p mod W, for p in
    [max(0, L_b - W), L_b); slots no position reaches are NaN (never read
    as keys).  Pure data movement."""
    B, Hkv, _, D = k_ctx.shape
    k = torch.full((B, Hkv, W, D), float("nan"), dtype=k_ctx.dtype)
    v = torch.full((B, Hkv, W, D), float("nan"), dtype=v_ctx.dtype)
    for b, L in enumerate(int(x) for x in prefix_lens):
        for p in range(max(0, L - W), L):
            k[b, :, p % W] = k_ctx[b, :, p]
            v[b, :, p % W] = v_ctx[b, :, p]
    return k, v
