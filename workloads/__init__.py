"""Seeded synthetic inputs for the block-sparse attention forward.

This module is shared by the parity tests, the benchmark and the oracle's
golden-value script.  It holds no attention arithmetic: it draws random
tensors, rounds them to bf16, and builds the integer index structures the
five workloads use (block tables, vertical/slash index sets, top-k block
selections, cu_seqlens).  Everything is a pure function of its seed.

Tensors are returned as numpy ``uint16`` arrays holding bf16 bit patterns, in
the (batch, seq, head, dim) layout used by the Incremental_FlashAttention
README ("Usage", section 1).  ``bf16_to_f64`` gives their exact values for a
CPU reference; ``to_torch_bf16`` hands the same bits to torch for the GPU.

Seeds: data = workload index (1..5), index structures = 1000 + index, the
gated workload's calibration data = 101.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

D_HEAD = 128


# ----------------------------------------------------------------------------
# bf16 helpers (round-to-nearest-even on the fp32 bit pattern)
# ----------------------------------------------------------------------------

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact values of bf16 bit patterns, widened to fp64."""
    return bf16_to_f32(bits).astype(np.float64)


def to_torch_bf16(bits: np.ndarray, device=None):
    """Same bits as a torch.bfloat16 tensor (optionally moved to ``device``)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device) if device is not None else t


def normal_f32(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    return bf16_bits(normal_f32(rng, shape))


# ----------------------------------------------------------------------------
# Workload containers
# ----------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    q: np.ndarray            # uint16 bf16 bits (B, Sq, Hq, D)
    k: np.ndarray            # uint16 bf16 bits (B, Sk, Hkv, D)
    v: np.ndarray
    causal: bool
    scale: float
    meta: dict = field(default_factory=dict)


def default_scale(d: int = D_HEAD) -> float:
    return 1.0 / math.sqrt(d)


# ----------------------------------------------------------------------------
# 1. Block-table forward (tiny): diagonal block + distinct random others
# ----------------------------------------------------------------------------

def block_table_diag_plus_random(rng, B, Hkv, n_qb, n_kb, nmax):
    """int32 [B, Hkv, n_qb, nmax]: entry 0 is the q-block's own (diagonal)
    key block i, entries 1.. are distinct random other key blocks."""
    tab = np.empty((B, Hkv, n_qb, nmax), dtype=np.int32)
    for b in range(B):
        for h in range(Hkv):
            for i in range(n_qb):
                others = np.array([j for j in range(n_kb) if j != i])
                pick = rng.choice(others, size=nmax - 1, replace=False)
                tab[b, h, i, 0] = i
                tab[b, h, i, 1:] = pick
    return tab


def make_block_table(B=1, H=2, Lq=256, Lk=1024, block=64, nmax=8, seed=1,
                     table_seed=1001) -> Workload:
    """The tiny block-table workload: non-causal, one table per
    (batch, kv-head, 64-row q-block)."""
    rng = np.random.default_rng(seed)
    q = normal_bf16(rng, (B, Lq, H, D_HEAD))
    k = normal_bf16(rng, (B, Lk, H, D_HEAD))
    v = normal_bf16(rng, (B, Lk, H, D_HEAD))
    trng = np.random.default_rng(table_seed)
    n_qb = -(-Lq // block)
    n_kb = Lk // block
    tab = block_table_diag_plus_random(trng, B, H, n_qb, n_kb, nmax)
    return Workload("block_table", q, k, v, causal=False, scale=default_scale(),
                    meta=dict(table=tab, q_block=block, kv_block=block, Hq=H, Hkv=H))


# ----------------------------------------------------------------------------
# 2. Speculative + sparse decode
# ----------------------------------------------------------------------------

def make_spec_decode(B=8, Hq=32, Hkv=8, Lq=1, Lk=32768, block=128, spec_len=2048,
                     n_missed=32, seed=2, table_seed=1002) -> Workload:
    """Pass A = dense over the last ``spec_len`` keys; pass B = ``n_missed``
    distinct random blocks (per batch and kv-head) from the blocks before it."""
    rng = np.random.default_rng(seed)
    q = normal_bf16(rng, (B, Lq, Hq, D_HEAD))
    k = normal_bf16(rng, (B, Lk, Hkv, D_HEAD))
    v = normal_bf16(rng, (B, Lk, Hkv, D_HEAD))
    n_rest = (Lk - spec_len) // block
    trng = np.random.default_rng(table_seed)
    tab = np.empty((B, Hkv, 1, n_missed), dtype=np.int32)
    for b in range(B):
        for h in range(Hkv):
            tab[b, h, 0] = trng.choice(n_rest, size=n_missed, replace=False)
    return Workload("spec_decode", q, k, v, causal=False, scale=default_scale(),
                    meta=dict(table=tab, kv_block=block, spec_begin=Lk - spec_len,
                              spec_end=Lk, Hq=Hq, Hkv=Hkv, causal_spec=True))


# ----------------------------------------------------------------------------
# 3. Gated prefill (BSFA): peaky scores from a shared shift direction
# ----------------------------------------------------------------------------

def make_gated(B=1, Hq=32, Hkv=8, L=32768, block=64, frac_shift=0.05, shift=3.0,
               seed=3) -> Workload:
    """q, k, v ~ N(0,1); per kv-head a random unit vector u; 5% of the key
    blocks of that kv-head get k += shift*u and every query of the heads in
    that group gets q += shift*u (one reading of 'shared with q')."""
    rng = np.random.default_rng(seed)
    q = normal_f32(rng, (B, L, Hq, D_HEAD))
    k = normal_f32(rng, (B, L, Hkv, D_HEAD))
    v = normal_f32(rng, (B, L, Hkv, D_HEAD))
    u = normal_f32(rng, (Hkv, D_HEAD)).astype(np.float64)
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    u = u.astype(np.float32)
    n_kb = L // block
    n_shift = int(math.ceil(frac_shift * n_kb))
    G = Hq // Hkv
    shifted = np.zeros((Hkv, n_shift), dtype=np.int64)
    for g in range(Hkv):
        shifted[g] = np.sort(rng.choice(n_kb, size=n_shift, replace=False))
        q[:, :, g * G:(g + 1) * G, :] += shift * u[g]
        for j in shifted[g]:
            k[:, j * block:(j + 1) * block, g, :] += shift * u[g]
    return Workload("gated", bf16_bits(q), bf16_bits(k), bf16_bits(v), causal=True,
                    scale=default_scale(),
                    meta=dict(block=block, Hq=Hq, Hkv=Hkv, shifted_blocks=shifted))


# ----------------------------------------------------------------------------
# 4. NSA-style selected attention, varlen
# ----------------------------------------------------------------------------

def nsa_selection(rng, seqlens, H, block=64, topk=16, n_init=1, n_local=2):
    """int32 [total, H, topk] of sequence-local key-block indices, -1 padded.

    For token t of a sequence and head h, with c = t // block: block 0 (the
    init block), the local blocks c and c-1, and distinct random blocks from
    the remaining causal-valid ones {1 .. c-2}, up to ``topk`` in all."""
    assert n_init == 1 and n_local == 2
    total = int(sum(seqlens))
    out = np.full((total, H, topk), -1, dtype=np.int32)
    n_rand = topk - n_init - n_local
    base = 0
    for L in seqlens:
        n_c = -(-L // block)
        for c in range(n_c):
            t0, t1 = base + c * block, base + min((c + 1) * block, L)
            rows = (t1 - t0) * H
            fixed = [0] + [b for b in (c, c - 1) if b >= 1]
            sel = np.full((rows, topk), -1, dtype=np.int32)
            sel[:, :len(fixed)] = fixed
            n_cand = max(c - 2, 0)          # candidates {1 .. c-2}
            take = min(n_rand, n_cand)
            if take > 0:
                if take == n_cand:
                    pick = np.broadcast_to(np.arange(1, c - 1), (rows, n_cand))
                else:
                    keys = rng.random((rows, n_cand))
                    pick = 1 + np.argpartition(keys, take - 1, axis=1)[:, :take]
                sel[:, len(fixed):len(fixed) + take] = pick
            out[t0:t1] = sel.reshape(t1 - t0, H, topk)
        base += L
    return out


def make_nsa_varlen(seqlens=(65536, 32768), H=4, block=64, topk=16, seed=4,
                    table_seed=1004) -> Workload:
    rng = np.random.default_rng(seed)
    total = int(sum(seqlens))
    q = normal_bf16(rng, (1, total, H, D_HEAD))
    k = normal_bf16(rng, (1, total, H, D_HEAD))
    v = normal_bf16(rng, (1, total, H, D_HEAD))
    cu = np.zeros(len(seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(seqlens)
    sel = nsa_selection(np.random.default_rng(table_seed), seqlens, H, block, topk)
    return Workload("nsa_varlen", q, k, v, causal=True, scale=default_scale(),
                    meta=dict(cu_seqlens=cu, seqlens=tuple(seqlens), sel=sel,
                              block=block, topk=topk, Hq=H, Hkv=H))


# ----------------------------------------------------------------------------
# 5. Vertical-slash sparse prefill
# ----------------------------------------------------------------------------

def vertical_slash_indices(rng, B, H, L, nnz_v, nnz_s, always=64):
    """Sorted distinct vertical columns and slash offsets per (b, h); each set
    always holds 0..always-1, the rest uniform over [always, L)."""
    vert = np.empty((B, H, nnz_v), dtype=np.int32)
    slash = np.empty((B, H, nnz_s), dtype=np.int32)
    base = np.arange(always)
    for b in range(B):
        for h in range(H):
            rv = always + rng.choice(L - always, size=nnz_v - always, replace=False)
            rs = always + rng.choice(L - always, size=nnz_s - always, replace=False)
            vert[b, h] = np.sort(np.concatenate([base, rv]))
            slash[b, h] = np.sort(np.concatenate([base, rs]))
    return vert, slash


def make_vertical_slash(B=1, H=32, L=131072, nnz_v=1000, nnz_s=6000, block=64,
                        seed=5, table_seed=1005) -> Workload:
    rng = np.random.default_rng(seed)
    q = normal_bf16(rng, (B, L, H, D_HEAD))
    k = normal_bf16(rng, (B, L, H, D_HEAD))
    v = normal_bf16(rng, (B, L, H, D_HEAD))
    vert, slash = vertical_slash_indices(np.random.default_rng(table_seed), B, H, L,
                                         nnz_v, nnz_s)
    return Workload("vertical_slash", q, k, v, causal=True, scale=default_scale(),
                    meta=dict(vertical=vert, slash=slash, block_M=block, block_N=block,
                              Hq=H, Hkv=H))


# ----------------------------------------------------------------------------
# Sampling of query rows for large-size parity checks
# ----------------------------------------------------------------------------

def sample_qblocks(rng, n_qb, n=4):
    """n distinct q-block indices, always including the last one."""
    if n_qb <= n:
        return np.arange(n_qb)
    rest = rng.choice(n_qb - 1, size=n - 1, replace=False)
    return np.sort(np.concatenate([rest, [n_qb - 1]]))
