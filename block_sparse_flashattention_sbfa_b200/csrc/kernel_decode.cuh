// Split-KV decode kernel: speculative + sparse decode (Incremental_FlashAttention
// README, Usage 2) and short-query block-table attention, fused with the LSE
// combine of the per-CTA pieces.
//
// Work: for every (batch b, kv-head g) pair the key set is a list of 64-key
// chunks -- the dense source A (k_spec/v_spec) cut into chunks, followed by
// the listed blocks of source B (k/v).  The chunks of all pairs are laid end
// to end and every CTA of the persistent grid takes an equal contiguous
// range of them (no load imbalance whatever the per-pair counts).  A CTA
// streams its chunks through a TMA pipeline; four consumer warps each take 16
// keys of a chunk and run QK^T and PV on mma.sync (the M = 16 tile carries
// the <= 16 query rows of the pair: Sq positions x G query heads).  At the end
// of its part of a pair the CTA merges its warps' running (m, l, O) and either
// writes the final row (the pair lies wholly inside the CTA's range) or an
// fp32 partial; the last CTA to finish a pair (atomic ticket) merges the
// partials with the LSE combine and resets the ticket.
#pragma once

#include "sbfa_ptx.cuh"

namespace sbfa {

constexpr int kDecChunk = 64;
constexpr int kDecGroupWarps = 4;                        // warps per consumer group
constexpr int kDecGroups = 2;                            // groups take alternate chunks
constexpr int kDecGroupThreads = kDecGroupWarps * 32;
constexpr int kDecThreads = kDecGroups * kDecGroupThreads;
constexpr int kDecWarpStages = 2;                        // cp.async double buffer per warp
constexpr int kDecSliceKeys = 16;                        // keys of a chunk one warp owns
constexpr int kDecSliceBytes = 2 * kDecSliceKeys * 128 * 2;  // K + V slice, bf16
constexpr int kDecMaxPairs = 4096;
constexpr int kDecMaxEntries = 1024;
constexpr int kDecMaxList = 2048;                        // chunks per window
constexpr int kDecMaxPieces = 256;                       // pair pieces per window
constexpr int kDecRows = 16;
constexpr int kDecD = 128;
constexpr int kDecStageBytes = 2 * kDecChunk * kDecD * 2;  // K + V, bf16

struct DecodeParams {
  int B, Sq, Hq, Hkv, G, rows;
  float scale_log2;
  const __nv_bfloat16* q;
  int64_t qsb, qss, qsh;
  __nv_bfloat16* o;
  int64_t osb, oss, osh;
  float* lse;
  int has_A, S_A, causal_A;
  int has_B, S_B, kv_block, nmax, n_kb;
  // key/value sources: A = dense range (k_spec/v_spec), B = table blocks
  const __nv_bfloat16* kA;
  const __nv_bfloat16* vA;
  const __nv_bfloat16* kB;
  const __nv_bfloat16* vB;
  int64_t kAsb, kAss, kAsh, vAsb, vAss, vAsh;
  int64_t kBsb, kBss, kBsh, vBsb, vBss, vBsh;
  const int* idx;
  int64_t tsb, tsh;
  int pair_mode;    // 1: every pair handled whole by one CTA (no workspace)
  int* ws_ticket;   // [B*Hkv]
  float* ws_part;   // [grid*2][rows][D]
  float* ws_lse;    // [grid*2][rows]
  int* status;
};

struct DecPiece {
  int pr, kbeg, kend, flags;  // list positions [kbeg, kend); flags: 1 = the CTA's
                              // part of pair pr starts in this window, 2 = ends in it
  int c_from;                 // pair-local chunk index of list position kbeg
};

struct DecSmem {
  alignas(1024) uint8_t slice[kDecGroups * kDecGroupWarps][kDecWarpStages][kDecSliceBytes];
  float mw[kDecGroupWarps][kDecRows];
  float lw[kDecGroupWarps][kDecRows];
  float ow[kDecGroupWarps][kDecRows][kDecD];
  int prefix[kDecMaxPairs + 1];
  int entries[kDecMaxEntries];
  int2 chunk[kDecMaxList];  // {key0, nkeys | src << 8}
  DecPiece piece[kDecMaxPieces];
  int n_pieces, n_list;
  int64_t next_x;           // window builder cursor (next global chunk of this CTA)
  int next_pr;
  int is_last;
  int n_split;
  int split_pr[2];  // pairs this CTA shares with others (stream-K: first and last)
};

static_assert(sizeof(DecSmem) + 1024 <= 232448, "decode shared memory exceeds 227 KB");

__device__ __forceinline__ int dec_chunks_per_entry(int kv_block) {
  return kv_block >= kDecChunk ? kv_block / kDecChunk : 1;
}

__device__ __forceinline__ int64_t dec_range_lo(int c, int64_t total, int grid) {
  return (total * c) / grid;
}

// CTA whose range holds global chunk x.
__device__ __forceinline__ int dec_cta_of(int64_t x, int64_t total, int grid) {
  int c = static_cast<int>((x * grid) / total);
  while (c + 1 < grid && dec_range_lo(c + 1, total, grid) <= x) ++c;
  while (c > 0 && dec_range_lo(c, total, grid) > x) --c;
  return c;
}

// Number of CTAs in [c_first, c_last] whose chunk range is not empty.
__device__ __forceinline__ int dec_nonempty_ctas(int c_first, int c_last, int64_t total, int grid) {
  int n = 0;
  for (int c = c_first; c <= c_last; ++c)
    n += dec_range_lo(c, total, grid) < dec_range_lo(c + 1, total, grid) ? 1 : 0;
  return n;
}

// Pair holding global chunk x (prefix is non-decreasing, prefix[n] = total).
__device__ __forceinline__ int dec_pair_of(const int* prefix, int npairs, int64_t x) {
  int lo = 0, hi = npairs;  // prefix[lo] <= x < prefix[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (prefix[mid] <= x) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Address of bf16 element (key, d) of a 64 x 128 tile stored as two
// 128B-swizzled halves of 64 columns.
__device__ __forceinline__ uint32_t dec_elem_addr(uint32_t base, int key, int d) {
  const int half = d >> 6;
  const int byte = (d & 63) * 2;
  return base + half * 8192 + sw128_off(key, byte >> 4) + (byte & 15);
}

// Address of bf16 element (key, d) of a 16-key slice stored as two
// 128B-swizzled halves of 64 columns (16 rows x 128 bytes each).
__device__ __forceinline__ uint32_t slice_elem_addr(uint32_t base, int key, int d) {
  const int half = d >> 6;
  const int byte = (d & 63) * 2;
  return base + half * (kDecSliceKeys * 128) + sw128_off(key, byte >> 4) + (byte & 15);
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int npairs = p.B * p.Hkv;
  const int grid = gridDim.x;
  const int cta = blockIdx.x;
  const int nA = p.has_A ? (p.S_A + kDecChunk - 1) / kDecChunk : 0;
  const int cpe = dec_chunks_per_entry(p.kv_block);
  const int keys_per_entry_chunk = p.kv_block < kDecChunk ? p.kv_block : kDecChunk;

  // ---- per-pair chunk counts and their prefix sum (every CTA computes the same)
  for (int pr = tid; pr < npairs; pr += kDecThreads) sm.prefix[pr + 1] = nA;
  __syncthreads();
  if (p.has_B) {
    const int n_ent = npairs * p.nmax;
    for (int base = 0; base < n_ent; base += 4 * kDecThreads) {
      int jv[4], pv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = base + u * kDecThreads + tid;
        pv[u] = -1;
        jv[u] = -1;
        if (e < n_ent) {
          const int pr = e / p.nmax, n = e % p.nmax;
          pv[u] = pr;
          jv[u] = __ldg(p.idx + (pr / p.Hkv) * p.tsb + (pr % p.Hkv) * p.tsh + n);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (pv[u] < 0) continue;
        if (jv[u] >= 0 && jv[u] < p.n_kb) atomicAdd(&sm.prefix[pv[u] + 1], cpe);
        else if (jv[u] >= p.n_kb && cta == 0) report(p.status, kDevBadIndex);
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    if (lane == 0) sm.prefix[0] = 0;
    for (int base = 0; base < npairs; base += 32) {
      int v = (base + lane < npairs) ? sm.prefix[base + lane + 1] : 0;
      for (int off = 1; off < 32; off <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += t;
      }
      if (base + lane < npairs) sm.prefix[base + lane + 1] = v + carry;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  __syncthreads();
  const int64_t total = sm.prefix[npairs];

  // Pairs with no key at all: write the neutral result (o = 0, lse = -inf).
  for (int pr = cta; pr < npairs; pr += grid) {
    if (sm.prefix[pr + 1] != sm.prefix[pr]) continue;
    const int b = pr / p.Hkv, g = pr % p.Hkv;
    for (int e = tid; e < p.rows * kDecD; e += kDecThreads) {
      const int rr = e / kDecD, d = e % kDecD;
      const int sq = rr / p.G, h = g * p.G + rr % p.G;
      p.o[b * p.osb + sq * p.oss + h * p.osh + d] = __float2bfloat16(0.f);
      if (d == 0) p.lse[(static_cast<int64_t>(b) * p.Hq + h) * p.Sq + sq] = -INFINITY;
    }
  }
  if (total == 0) return;
  // This CTA's chunks: stream-K = the contiguous global range [lo, hi); pair
  // mode = whole pairs cta, cta + grid, ...
  const int64_t lo = p.pair_mode ? 0 : dec_range_lo(cta, total, grid);
  const int64_t hi = p.pair_mode ? total : dec_range_lo(cta + 1, total, grid);
  if (lo >= hi) return;
  const int first_pair = p.pair_mode ? cta : dec_pair_of(sm.prefix, npairs, lo);
  const int pair_step = p.pair_mode ? grid : 1;

  const int grp = warp / kDecGroupWarps, wg = warp % kDecGroupWarps;
  const int gt = tid % kDecGroupThreads;  // thread index inside the group
  const int gq = lane >> 2, cq = lane & 3;
  const float NEG = -INFINITY;
  if (tid == 0) {
    sm.next_pr = first_pair;
    sm.next_x = 0;  // chunks of pair next_pr already handed out (pair-local)
    sm.n_split = 0;
  }
  __syncthreads();

  // running state of the piece in progress (persists across windows)
  uint32_t qa[8][4];
  float m0 = NEG, m1 = NEG, l0 = 0.f, l1 = 0.f;
  float oacc[16][4];
  bool v0 = false, v1 = false;
  int lim0 = -1, lim1 = -1;

  // A pair shared with other CTAs: after this CTA's partial is written, the
  // last CTA to finish the pair merges all partials with the LSE combine.
  auto finish_split = [&](const int pr) {
    __threadfence();
    __syncthreads();
    const int d = tid % kDecD;
    const int rpar = tid / kDecD;
    const int b = pr / p.Hkv, g = pr % p.Hkv;
    const int64_t pbeg = sm.prefix[pr], pend = sm.prefix[pr + 1];
    const int c_first = dec_cta_of(pbeg, total, grid);
    const int c_last = dec_cta_of(pend - 1, total, grid);
    if (tid == 0) {
      const int old = atomicAdd(&p.ws_ticket[pr], 1);
      sm.is_last = (old == dec_nonempty_ctas(c_first, c_last, total, grid) - 1) ? 1 : 0;
      if (sm.is_last) __threadfence();
    }
    __syncthreads();
    if (sm.is_last) {
      for (int rr = rpar; rr < p.rows; rr += 2) {
        float M = -INFINITY;
        for (int cc = c_first; cc <= c_last; ++cc) {
          if (dec_range_lo(cc, total, grid) == dec_range_lo(cc + 1, total, grid)) continue;
          const int fp = dec_pair_of(sm.prefix, npairs, dec_range_lo(cc, total, grid));
          const int sl = (fp == pr) ? 2 * cc : 2 * cc + 1;
          M = fmaxf(M, __ldcg(&p.ws_lse[sl * kDecRows + rr]));
        }
        const float Mn = (M == -INFINITY) ? 0.f : M;
        float W = 0.f, acc = 0.f;
        for (int cc = c_first; cc <= c_last; ++cc) {
          if (dec_range_lo(cc, total, grid) == dec_range_lo(cc + 1, total, grid)) continue;
          const int fp = dec_pair_of(sm.prefix, npairs, dec_range_lo(cc, total, grid));
          const int sl = (fp == pr) ? 2 * cc : 2 * cc + 1;
          const float lv = __ldcg(&p.ws_lse[sl * kDecRows + rr]);
          const float wt = (lv == -INFINITY) ? 0.f : __expf(lv - Mn);
          W += wt;
          acc += wt * __ldcg(&p.ws_part[(static_cast<int64_t>(sl) * kDecRows + rr) * kDecD + d]);
        }
        const int sq = rr / p.G, h = g * p.G + rr % p.G;
        p.o[b * p.osb + sq * p.oss + h * p.osh + d] = __float2bfloat16(W > 0.f ? acc / W : 0.f);
        if (d == 0)
          p.lse[(static_cast<int64_t>(b) * p.Hq + h) * p.Sq + sq] = W > 0.f ? Mn + __logf(W) : -INFINITY;
      }
      if (tid == 0) p.ws_ticket[pr] = 0;
    }
    __syncthreads();
  };

  while (true) {
    // ================= build the next window of chunks =================
    if (tid == 0) {
      int np = 0, nl = 0;
      int pr = sm.next_pr;
      int64_t used = sm.next_x;
      while (pr < npairs && np < kDecMaxPieces && nl < kDecMaxList) {
        const int64_t pbeg = sm.prefix[pr], pend = sm.prefix[pr + 1];
        if (pbeg >= hi) { pr = npairs; break; }
        const int64_t c0 = (lo > pbeg ? lo : pbeg) - pbeg;
        const int64_t c1 = (hi < pend ? hi : pend) - pbeg;
        if (c1 <= c0) { pr += pair_step; used = 0; continue; }
        const int64_t from = c0 + used;
        const int64_t take = min(static_cast<int64_t>(kDecMaxList - nl), c1 - from);
        DecPiece pc;
        pc.pr = pr;
        pc.kbeg = nl;
        pc.kend = nl + static_cast<int>(take);
        pc.flags = (used == 0 ? 1 : 0) | (from + take == c1 ? 2 : 0);
        pc.c_from = static_cast<int>(from);
        sm.piece[np++] = pc;
        nl += static_cast<int>(take);
        if (from + take == c1) { pr += pair_step; used = 0; }
        else used += take;
      }
      sm.n_pieces = np;
      sm.n_list = nl;
      sm.next_pr = pr;
      sm.next_x = used;
    }
    __syncthreads();
    const int n_pieces = sm.n_pieces, n_list = sm.n_list;
    if (n_list == 0) break;
    // chunk metadata of every list position; a piece's valid table entries
    // are compacted first (in table order)
    for (int pi = 0; pi < n_pieces; ++pi) {
      const DecPiece pc = sm.piece[pi];
      const int b = pc.pr / p.Hkv, g = pc.pr % p.Hkv;
      if (p.has_B && warp == 0) {
        const int* row = p.idx + b * p.tsb + g * p.tsh;
        int nv = 0;
        for (int base = 0; base < p.nmax; base += 32) {
          const int n = base + lane;
          const int j = n < p.nmax ? __ldg(row + n) : -1;
          const bool valid = j >= 0 && j < p.n_kb;
          const uint32_t bal = __ballot_sync(0xffffffffu, valid);
          if (valid) sm.entries[nv + __popc(bal & ((1u << lane) - 1u))] = j;
          nv += __popc(bal);
        }
      }
      __syncthreads();
      for (int k = pc.kbeg + tid; k < pc.kend; k += kDecThreads) {
        const int c = pc.c_from + (k - pc.kbeg);
        int src, key0, nk;
        if (c < nA) {
          src = 0;
          key0 = c * kDecChunk;
          nk = min(kDecChunk, p.S_A - key0);
        } else {
          const int e = (c - nA) / cpe, sub = (c - nA) % cpe;
          src = 1;
          key0 = sm.entries[e] * p.kv_block + sub * kDecChunk;
          nk = min(keys_per_entry_chunk, p.S_B - key0);
        }
        nk = max(nk, 0);
        sm.chunk[k] = make_int2(key0, nk | (src << 8) | (pi << 16));
      }
      __syncthreads();
    }

    // ================= consume: two groups, cp.async double buffer =================
    const int n_mine = (n_list - grp + 1) / 2;  // list positions grp, grp + 2, ...
    // Each warp streams its own 16-key slice of its group's chunks through a
    // private double buffer: it waits only for its own copies (no barrier
    // with other warps), so warps progress independently.
    const int kw = wg * kDecSliceKeys;
    auto issue = [&](int j) {
      const int k = grp + 2 * j;
      const int2 ci = sm.chunk[k];
      const int key0 = ci.x, nk = ci.y & 0xff, src = (ci.y >> 8) & 1;
      const int pr = sm.piece[ci.y >> 16].pr;
      const int b = pr / p.Hkv, g = pr % p.Hkv;
      const __nv_bfloat16* krow0 =
          src ? p.kB + b * p.kBsb + g * p.kBsh : p.kA + b * p.kAsb + g * p.kAsh;
      const __nv_bfloat16* vrow0 =
          src ? p.vB + b * p.vBsb + g * p.vBsh : p.vA + b * p.vAsb + g * p.vAsh;
      const int64_t kro = src ? p.kBss : p.kAss, vro = src ? p.vBss : p.vAss;
      const uint32_t kdst = smem_u32(sm.slice[warp][j & 1]);
#pragma unroll
      for (int it = 0; it < kDecSliceKeys * 16 / 32; ++it) {
        const int e = lane + it * 32;
        const int r = e >> 4, ch = e & 15;
        const uint32_t off = (ch >> 3) * (kDecSliceKeys * 128) + sw128_off(r, ch & 7);
        const bool valid = kw + r < nk;
        const int64_t row = valid ? key0 + kw + r : 0;
        const uint32_t bytes = valid ? 16u : 0u;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(kdst + off),
                     "l"(krow0 + row * kro + ch * 8), "r"(bytes)
                     : "memory");
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                         kdst + kDecSliceBytes / 2 + off),
                     "l"(vrow0 + row * vro + ch * 8), "r"(bytes)
                     : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    if (n_mine > 0) issue(0);
    if (n_mine > 1) issue(1);
    int jc = 0;
    for (int pi = 0; pi < n_pieces; ++pi) {
      const DecPiece pc = sm.piece[pi];
      const int b = pc.pr / p.Hkv, g = pc.pr % p.Hkv;
      if (pc.flags & 1) {
        // Q fragments (A operand, 16 rows x 128) and per-row limits for this pair
        const int r0 = gq, r1 = gq + 8;
        v0 = r0 < p.rows;
        v1 = r1 < p.rows;
        lim0 = v0 ? r0 / p.G + (p.S_A - p.Sq) : -1;
        lim1 = v1 ? r1 / p.G + (p.S_A - p.Sq) : -1;
        const __nv_bfloat16* q0 =
            v0 ? p.q + b * p.qsb + (r0 / p.G) * p.qss + (g * p.G + r0 % p.G) * p.qsh : nullptr;
        const __nv_bfloat16* q1 =
            v1 ? p.q + b * p.qsb + (r1 / p.G) * p.qss + (g * p.G + r1 % p.G) * p.qsh : nullptr;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int d = ks * 16 + 2 * cq;
          qa[ks][0] = q0 ? __ldg(reinterpret_cast<const unsigned int*>(q0 + d)) : 0u;
          qa[ks][1] = q1 ? __ldg(reinterpret_cast<const unsigned int*>(q1 + d)) : 0u;
          qa[ks][2] = q0 ? __ldg(reinterpret_cast<const unsigned int*>(q0 + d + 8)) : 0u;
          qa[ks][3] = q1 ? __ldg(reinterpret_cast<const unsigned int*>(q1 + d + 8)) : 0u;
        }
        m0 = m1 = NEG;
        l0 = l1 = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
      }
      for (; jc < n_mine && grp + 2 * jc < pc.kend; ++jc) {
        if (jc + 1 < n_mine) asm volatile("cp.async.wait_group 1;" ::: "memory");
        else asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncwarp();  // this warp's copies are in and visible to all its lanes
        const int2 ci = sm.chunk[grp + 2 * jc];
        const int key0 = ci.x, nkeys = ci.y & 0xff, src = (ci.y >> 8) & 1;
        const uint32_t kbase = smem_u32(sm.slice[warp][jc & 1]);
        const uint32_t vbase = kbase + kDecSliceBytes / 2;
        float s[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
        {
          // ldmatrix x4: matrices (keys kw..+7 | kw+8..+15) x (d lo | d hi of the k-step)
          const int mi = lane >> 3, ri = lane & 7;
          const int key = (mi >> 1) * 8 + ri;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            uint32_t b00, b01, b10, b11;
            const uint32_t addr = slice_elem_addr(kbase, key, ks * 16 + (mi & 1) * 8);
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                         : "=r"(b00), "=r"(b01), "=r"(b10), "=r"(b11)
                         : "r"(addr));
            mma_bf16_16816(s[0], qa[ks], b00, b01);
            mma_bf16_16816(s[1], qa[ks], b10, b11);
          }
        }
        // scale and mask (fast path: a full chunk that needs no causal mask)
        const int lim_min = v1 ? min(lim0, lim1) : lim0;
        const bool full_chunk =
            nkeys >= kDecChunk && (src == 1 || !p.causal_A || key0 + kDecChunk - 1 <= lim_min);
        float mx0 = NEG, mx1 = NEG;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int kc = kw + nt * 8 + 2 * cq + (e & 1);
            bool vis = (e < 2) ? v0 : v1;
            if (!full_chunk) {
              vis = vis && kc < nkeys;
              if (src == 0 && p.causal_A) vis = vis && (key0 + kc) <= ((e < 2) ? lim0 : lim1);
            }
            const float x = vis ? s[nt][e] * p.scale_log2 : NEG;
            s[nt][e] = x;
            if (e < 2) mx0 = fmaxf(mx0, x); else mx1 = fmaxf(mx1, x);
          }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        // lazy running max: raise it only when a row max exceeds it by > 2^8
        float al0 = 1.f, al1 = 1.f;
        if (mx0 > m0 + 8.f) { al0 = ex2_approx(m0 - mx0); m0 = mx0; }
        if (mx1 > m1 + 8.f) { al1 = ex2_approx(m1 - mx1); m1 = mx1; }
        const float mu0 = (m0 == NEG) ? 0.f : m0, mu1 = (m1 == NEG) ? 0.f : m1;
        float ps0 = 0.f, ps1 = 0.f;
        uint32_t pa[4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const float p0 = ex2_approx(s[nt][0] - mu0), p1 = ex2_approx(s[nt][1] - mu0);
          const float p2 = ex2_approx(s[nt][2] - mu1), p3 = ex2_approx(s[nt][3] - mu1);
          ps0 += p0 + p1;
          ps1 += p2 + p3;
          pa[nt * 2 + 0] = pack_bf16x2(p0, p1);
          pa[nt * 2 + 1] = pack_bf16x2(p2, p3);
        }
        l0 = l0 * al0 + ps0;
        l1 = l1 * al1 + ps1;
        if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            oacc[i][0] *= al0; oacc[i][1] *= al0;
            oacc[i][2] *= al1; oacc[i][3] *= al1;
          }
        }
        // PV: A = P (16 x 16 keys of this warp), B = V[16 keys][128]
        {
          const int mi = lane >> 3, ri = lane & 7;
          const int key = (mi & 1) * 8 + ri;
#pragma unroll
          for (int dt2 = 0; dt2 < 8; ++dt2) {
            const int d0 = dt2 * 16 + (mi >> 1) * 8;
            uint32_t x0, x1, x2, x3;
            ldsm_x4_trans(slice_elem_addr(vbase, key, d0), x0, x1, x2, x3);
            mma_bf16_16816(oacc[2 * dt2], pa, x0, x1);
            mma_bf16_16816(oacc[2 * dt2 + 1], pa, x2, x3);
          }
        }
        __syncwarp();  // every lane is done with the buffer: refill it
        if (jc + 2 < n_mine) issue(jc + 2);
      }
      if (!(pc.flags & 2)) continue;  // the pair continues in the next window
      // ---- merge the eight warps' states for this pair
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      // (1) group 1 publishes its state, group 0 folds it into its registers
      if (grp == 1) {
        if (cq == 0) {
          sm.mw[wg][gq] = m0; sm.mw[wg][gq + 8] = m1;
          sm.lw[wg][gq] = l0; sm.lw[wg][gq + 8] = l1;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int d = i * 8 + 2 * cq;
          *reinterpret_cast<float2*>(&sm.ow[wg][gq][d]) = make_float2(oacc[i][0], oacc[i][1]);
          *reinterpret_cast<float2*>(&sm.ow[wg][gq + 8][d]) = make_float2(oacc[i][2], oacc[i][3]);
        }
      }
      __syncthreads();
      if (grp == 0) {
        const float om0 = sm.mw[wg][gq], om1 = sm.mw[wg][gq + 8];
        const float M0 = fmaxf(m0, om0), M1 = fmaxf(m1, om1);
        const float Mu0 = (M0 == NEG) ? 0.f : M0, Mu1 = (M1 == NEG) ? 0.f : M1;
        const float a0 = ex2_approx(m0 - Mu0), b0 = ex2_approx(om0 - Mu0);
        const float a1 = ex2_approx(m1 - Mu1), b1 = ex2_approx(om1 - Mu1);
        l0 = a0 * l0 + b0 * sm.lw[wg][gq];
        l1 = a1 * l1 + b1 * sm.lw[wg][gq + 8];
        m0 = M0;
        m1 = M1;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int d = i * 8 + 2 * cq;
          const float2 x = *reinterpret_cast<const float2*>(&sm.ow[wg][gq][d]);
          const float2 y = *reinterpret_cast<const float2*>(&sm.ow[wg][gq + 8][d]);
          oacc[i][0] = a0 * oacc[i][0] + b0 * x.x;
          oacc[i][1] = a0 * oacc[i][1] + b0 * x.y;
          oacc[i][2] = a1 * oacc[i][2] + b1 * y.x;
          oacc[i][3] = a1 * oacc[i][3] + b1 * y.y;
        }
      }
      __syncthreads();
      // (2) group 0 publishes the folded states
      if (grp == 0) {
        if (cq == 0) {
          sm.mw[wg][gq] = m0; sm.mw[wg][gq + 8] = m1;
          sm.lw[wg][gq] = l0; sm.lw[wg][gq + 8] = l1;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int d = i * 8 + 2 * cq;
          *reinterpret_cast<float2*>(&sm.ow[wg][gq][d]) = make_float2(oacc[i][0], oacc[i][1]);
          *reinterpret_cast<float2*>(&sm.ow[wg][gq + 8][d]) = make_float2(oacc[i][2], oacc[i][3]);
        }
      }
      __syncthreads();
      const int64_t pbeg = sm.prefix[pc.pr], pend = sm.prefix[pc.pr + 1];
      const int64_t c0 = (lo > pbeg ? lo : pbeg) - pbeg;
      const int64_t c1 = (hi < pend ? hi : pend) - pbeg;
      const bool whole = (c0 == 0) && (c1 == pend - pbeg);
      // 256 threads: thread t owns column d = t % 128 of rows r with r % 2 == t / 128
      const int d = tid % kDecD;
      const int rpar = tid / kDecD;
      const int slot = (pc.pr == first_pair) ? 2 * cta : 2 * cta + 1;
      for (int rr = rpar; rr < p.rows; rr += 2) {
        float M = NEG;
        for (int w = 0; w < kDecGroupWarps; ++w) M = fmaxf(M, sm.mw[w][rr]);
        const float Mu = (M == NEG) ? 0.f : M;
        float L = 0.f, acc = 0.f;
        for (int w = 0; w < kDecGroupWarps; ++w) {
          const float wt = ex2_approx(sm.mw[w][rr] - Mu);
          L += wt * sm.lw[w][rr];
          acc += wt * sm.ow[w][rr][d];
        }
        const float ov = L > 0.f ? acc / L : 0.f;
        const float lv = L > 0.f ? (Mu + lg2_approx(L)) * 0.69314718055994531f : NEG;
        const int sq = rr / p.G, h = g * p.G + rr % p.G;
        if (whole) {
          p.o[b * p.osb + sq * p.oss + h * p.osh + d] = __float2bfloat16(ov);
          if (d == 0) p.lse[(static_cast<int64_t>(b) * p.Hq + h) * p.Sq + sq] = lv;
        } else {
          p.ws_part[(static_cast<int64_t>(slot) * kDecRows + rr) * kDecD + d] = ov;
          if (d == 0) p.ws_lse[slot * kDecRows + rr] = lv;
        }
      }
      if (!whole) finish_split(pc.pr);
      __syncthreads();
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();  // the window's list and stages may be reused
  }

}

// ----------------------------------------------------------------------------
// Standalone LSE combine: one warp per (b, s, h) row, 4 columns per lane.
// ----------------------------------------------------------------------------
__global__ void combine_kernel(int n_parts, int B, int Sq, int Hq, const float* __restrict__ o_parts,
                               const float* __restrict__ lse_parts, __nv_bfloat16* o, int64_t osb,
                               int64_t oss, int64_t osh, float* lse) {
  const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t nrows = static_cast<int64_t>(B) * Sq * Hq;
  if (warp_global >= nrows) return;
  const int h = warp_global % Hq;
  const int s = (warp_global / Hq) % Sq;
  const int b = warp_global / (Hq * Sq);
  const int64_t lse_row = (static_cast<int64_t>(b) * Hq + h) * Sq + s;
  const int64_t part_lse_stride = nrows;
  const int64_t part_o_stride = nrows * kDecD;
  float M = -INFINITY;
  for (int pp = 0; pp < n_parts; ++pp) M = fmaxf(M, lse_parts[pp * part_lse_stride + lse_row]);
  const float Mn = (M == -INFINITY) ? 0.f : M;
  float W = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const int64_t orow = ((static_cast<int64_t>(b) * Sq + s) * Hq + h) * kDecD;
  for (int pp = 0; pp < n_parts; ++pp) {
    const float lv = lse_parts[pp * part_lse_stride + lse_row];
    if (lv == -INFINITY) continue;
    const float wt = __expf(lv - Mn);
    W += wt;
    const float4 x = *reinterpret_cast<const float4*>(o_parts + pp * part_o_stride + orow + lane * 4);
    acc.x += wt * x.x; acc.y += wt * x.y; acc.z += wt * x.z; acc.w += wt * x.w;
  }
  const float inv = W > 0.f ? 1.f / W : 0.f;
  __nv_bfloat16* op = o + b * osb + s * oss + h * osh + lane * 4;
  __nv_bfloat162 v01 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  __nv_bfloat162 v23 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  reinterpret_cast<__nv_bfloat162*>(op)[0] = v01;
  reinterpret_cast<__nv_bfloat162*>(op)[1] = v23;
  if (lane == 0) lse[lse_row] = W > 0.f ? Mn + __logf(W) : -INFINITY;
}

}  // namespace sbfa
