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
constexpr int kDecStages = 4;
constexpr int kDecGroupWarps = 4;                        // warps per consumer group
constexpr int kDecGroups = 2;                            // groups take alternate chunks
constexpr int kDecConsumerWarps = kDecGroupWarps * kDecGroups;
// Chunk k uses stage k % kDecStages and group k % kDecGroups.  The stage count
// must be a multiple of the group count so that every stage is always
// consumed by the same group: a group then waits on a stage's phases strictly
// in order and a parity wait can never be satisfied by an older phase.
static_assert(kDecStages % kDecGroups == 0, "each stage must belong to one consumer group");
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;
constexpr int kDecMaxPairs = 4096;
constexpr int kDecMaxEntries = 1024;
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
  const int* idx;
  int64_t tsb, tsh;
  int pair_mode;    // 1: every pair handled whole by one CTA (no workspace)
  int* ws_ticket;   // [B*Hkv]
  float* ws_part;   // [grid*2][rows][D]
  float* ws_lse;    // [grid*2][rows]
  int* status;
};

struct DecStageMeta {
  int src, key0, nkeys, pad;
};

struct DecSmem {
  alignas(1024) uint8_t stage[kDecStages][kDecStageBytes];
  float mw[kDecGroupWarps][kDecRows];
  float lw[kDecGroupWarps][kDecRows];
  float ow[kDecGroupWarps][kDecRows][kDecD];
  int prefix[kDecMaxPairs + 1];
  int entries[kDecMaxEntries];
  DecStageMeta meta[kDecStages];
  uint64_t full[kDecStages];
  uint64_t empty[kDecStages];
  int abort_flag;
  int is_last;
};

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

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__global__ void __launch_bounds__(kDecThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap mapKA,
                  const __grid_constant__ CUtensorMap mapVA,
                  const __grid_constant__ CUtensorMap mapKB,
                  const __grid_constant__ CUtensorMap mapVB, const DecodeParams p) {
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

  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kDecGroupWarps);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  // ---- per-pair chunk counts and their prefix sum (every CTA computes the same)
  // per-pair chunk counts: every thread scans a share of the table entries
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
  const WaitCtx wctx{&sm.abort_flag, p.status};

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
  const int64_t lo = p.pair_mode ? 0 : dec_range_lo(cta, total, grid);
  const int64_t hi = p.pair_mode ? total : dec_range_lo(cta + 1, total, grid);
  if (lo >= hi) return;
  const int first_pair = p.pair_mode ? cta : dec_pair_of(sm.prefix, npairs, lo);
  const int pair_step = p.pair_mode ? grid : 1;

  if (warp == kDecConsumerWarps) {
    // ======================= producer warp =======================
    int st = 0;
    uint32_t ph = 0;
    int issued = 0;
    bool ok = true;
    for (int pr = first_pair; pr < npairs && ok; pr += pair_step) {
      const int64_t pbeg = sm.prefix[pr], pend = sm.prefix[pr + 1];
      if (pbeg >= hi) break;
      if (pend <= lo || pend == pbeg) continue;
      const int b = pr / p.Hkv, g = pr % p.Hkv;
      // compact the valid table entries of this pair
      __syncwarp();
      if (p.has_B) {
        const int* row = p.idx + b * p.tsb + g * p.tsh;
        int nv = 0;
        for (int base = 0; base < p.nmax; base += 32) {
          const int n = base + lane;
          const int j = n < p.nmax ? row[n] : -1;
          const bool valid = j >= 0 && j < p.n_kb;
          const uint32_t bal = __ballot_sync(0xffffffffu, valid);
          if (valid) sm.entries[nv + __popc(bal & ((1u << lane) - 1u))] = j;
          nv += __popc(bal);
        }
      }
      __syncwarp();
      const int64_t c0 = (lo > pbeg ? lo : pbeg) - pbeg;
      const int64_t c1 = (hi < pend ? hi : pend) - pbeg;
      for (int64_t c = c0; c < c1; ++c) {
        if (lane == 0) {
          int src, key0, nk;
          if (c < nA) {
            src = 0;
            key0 = static_cast<int>(c) * kDecChunk;
            nk = min(kDecChunk, p.S_A - key0);
          } else {
            const int e = static_cast<int>(c - nA) / cpe, sub = static_cast<int>(c - nA) % cpe;
            src = 1;
            key0 = sm.entries[e] * p.kv_block + sub * kDecChunk;
            nk = min(keys_per_entry_chunk, p.S_B - key0);
          }
          if (!mbar_wait(&sm.empty[st], ph ^ 1u, wctx)) {
            ok = false;
          } else {
            sm.meta[st] = DecStageMeta{src, key0, nk, 0};
            mbar_arrive_expect_tx(&sm.full[st], kDecStageBytes);
            uint8_t* kdst = sm.stage[st];
            uint8_t* vdst = sm.stage[st] + kDecStageBytes / 2;
            const CUtensorMap* mk = src ? &mapKB : &mapKA;
            const CUtensorMap* mv = src ? &mapVB : &mapVA;
            tma_load_4d(kdst, mk, &sm.full[st], 0, g, key0, b);
            tma_load_4d(kdst + 8192, mk, &sm.full[st], 64, g, key0, b);
            tma_load_4d(vdst, mv, &sm.full[st], 0, g, key0, b);
            tma_load_4d(vdst + 8192, mv, &sm.full[st], 64, g, key0, b);
            ++issued;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (++st == kDecStages) { st = 0; ph ^= 1u; }
      }
    }
    if (!ok && lane == 0) {
      // drain: wait (briefly) for the copies still in flight
      for (int s = 0; s < kDecStages; ++s) mbar_wait_short(&sm.full[s], 0), (void)issued;
    }
    return;
  }

  // ======================= consumer warps =======================
  // Two groups of four warps take alternate chunks; in a chunk warp w of a
  // group owns keys [16w, 16w + 16).  Per warp: S (16 rows x 16 keys) by
  // mma.sync with K fragments from ldmatrix, online softmax with a lazily
  // raised running max, O (16 x 128) += P V with V fragments from
  // ldmatrix.trans.
  const int grp = warp / kDecGroupWarps, wg = warp % kDecGroupWarps;
  const int gq = lane >> 2, cq = lane & 3;
  const float NEG = -INFINITY;
  const int nthr = kDecConsumerWarps * 32;
  int64_t kseq = 0;  // CTA-local index of the next chunk (same order as the producer)
  for (int pr = first_pair; pr < npairs; pr += pair_step) {
    const int64_t pbeg = sm.prefix[pr], pend = sm.prefix[pr + 1];
    if (pbeg >= hi) break;
    if (pend <= lo || pend == pbeg) continue;
    const int b = pr / p.Hkv, g = pr % p.Hkv;
    const int64_t c0 = (lo > pbeg ? lo : pbeg) - pbeg;
    const int64_t c1 = (hi < pend ? hi : pend) - pbeg;
    const bool whole = (c0 == 0) && (c1 == pend - pbeg);

    // Q fragments (A operand, 16 rows x 128) and per-row limits for this pair
    uint32_t qa[8][4];
    const int r0 = gq, r1 = gq + 8;
    const bool v0 = r0 < p.rows, v1 = r1 < p.rows;
    // causal limit of source-A key positions for rows r0, r1
    const int lim0 = v0 ? r0 / p.G + (p.S_A - p.Sq) : -1;
    const int lim1 = v1 ? r1 / p.G + (p.S_A - p.Sq) : -1;
    {
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
    }
    float m0 = NEG, m1 = NEG, l0 = 0.f, l1 = 0.f;
    float oacc[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;

    bool ok = true;
    const int64_t k_first = kseq, k_end = kseq + (c1 - c0);
    kseq = k_end;
    for (int64_t kk = k_first + ((k_first & 1) != grp ? 1 : 0); kk < k_end; kk += 2) {
      const int st = static_cast<int>(kk % kDecStages);
      const uint32_t ph = static_cast<uint32_t>((kk / kDecStages) & 1);
      if (!mbar_wait(&sm.full[st], ph, wctx)) { ok = false; break; }
      const DecStageMeta mt = sm.meta[st];
      const uint32_t kbase = smem_u32(sm.stage[st]);
      const uint32_t vbase = kbase + kDecStageBytes / 2;
      const int kw = wg * 16;
      float s[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
      {
        // ldmatrix x4: matrices (keys kw..+7 | kw+8..+15) x (d lo | d hi of the k-step)
        const int mi = lane >> 3, ri = lane & 7;
        const int key = kw + (mi >> 1) * 8 + ri;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t b00, b01, b10, b11;
          const uint32_t addr = dec_elem_addr(kbase, key, ks * 16 + (mi & 1) * 8);
          asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                       : "=r"(b00), "=r"(b01), "=r"(b10), "=r"(b11)
                       : "r"(addr));
          mma_bf16_16816(s[0], qa[ks], b00, b01);
          mma_bf16_16816(s[1], qa[ks], b10, b11);
        }
      }
      // scale and mask (fast path: a full chunk that needs no causal mask)
      const bool full_chunk = mt.nkeys >= kDecChunk &&
                              (mt.src == 1 || !p.causal_A || mt.key0 + kDecChunk - 1 <= min(lim0, lim1 < 0 ? lim0 : lim1));
      float mx0 = NEG, mx1 = NEG;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kc = kw + nt * 8 + 2 * cq + (e & 1);
          bool vis = (e < 2) ? v0 : v1;
          if (!full_chunk) {
            vis = vis && kc < mt.nkeys;
            if (mt.src == 0 && p.causal_A) vis = vis && (mt.key0 + kc) <= ((e < 2) ? lim0 : lim1);
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
        const int key = kw + (mi & 1) * 8 + ri;
#pragma unroll
        for (int dt2 = 0; dt2 < 8; ++dt2) {
          const int d0 = dt2 * 16 + (mi >> 1) * 8;
          uint32_t x0, x1, x2, x3;
          ldsm_x4_trans(dec_elem_addr(vbase, key, d0), x0, x1, x2, x3);
          mma_bf16_16816(oacc[2 * dt2], pa, x0, x1);
          mma_bf16_16816(oacc[2 * dt2 + 1], pa, x2, x3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[st]);
    }
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
    const bool aborted = named_bar_or(1, nthr, !ok || sm.abort_flag != 0);
    if (grp == 0 && !aborted) {
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
    named_bar_sync(1, nthr);
    // (2) group 0 publishes the folded states
    if (grp == 0 && !aborted) {
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
    named_bar_sync(1, nthr);
    if (!aborted) {
      // 256 threads: thread t owns column d = t % 128 of rows r with r % 2 == t / 128
      const int d = tid % kDecD;
      const int rpar = tid / kDecD;
      const int slot = (pr == first_pair) ? 2 * cta : 2 * cta + 1;
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
      if (!whole) {
        __threadfence();
        named_bar_sync(1, nthr);
        if (tid == 0) {
          const int c_first = dec_cta_of(pbeg, total, grid);
          const int c_last = dec_cta_of(pend - 1, total, grid);
          const int old = atomicAdd(&p.ws_ticket[pr], 1);
          sm.is_last = (old == dec_nonempty_ctas(c_first, c_last, total, grid) - 1) ? 1 : 0;
          if (sm.is_last) __threadfence();
        }
        named_bar_sync(1, nthr);
        if (sm.is_last) {
          const int c_first = dec_cta_of(pbeg, total, grid);
          const int c_last = dec_cta_of(pend - 1, total, grid);
          for (int rr = rpar; rr < p.rows; rr += 2) {
            float M = NEG;
            for (int cc = c_first; cc <= c_last; ++cc) {
              if (dec_range_lo(cc, total, grid) == dec_range_lo(cc + 1, total, grid)) continue;
              const int fp = dec_pair_of(sm.prefix, npairs, dec_range_lo(cc, total, grid));
              const int sl = (fp == pr) ? 2 * cc : 2 * cc + 1;
              M = fmaxf(M, __ldcg(&p.ws_lse[sl * kDecRows + rr]));
            }
            const float Mn = (M == NEG) ? 0.f : M;
            float W = 0.f, acc = 0.f;
            for (int cc = c_first; cc <= c_last; ++cc) {
              if (dec_range_lo(cc, total, grid) == dec_range_lo(cc + 1, total, grid)) continue;
              const int fp = dec_pair_of(sm.prefix, npairs, dec_range_lo(cc, total, grid));
              const int sl = (fp == pr) ? 2 * cc : 2 * cc + 1;
              const float lv = __ldcg(&p.ws_lse[sl * kDecRows + rr]);
              const float wt = (lv == NEG) ? 0.f : __expf(lv - Mn);
              W += wt;
              acc += wt * __ldcg(&p.ws_part[(static_cast<int64_t>(sl) * kDecRows + rr) * kDecD + d]);
            }
            const int sq = rr / p.G, h = g * p.G + rr % p.G;
            p.o[b * p.osb + sq * p.oss + h * p.osh + d] =
                __float2bfloat16(W > 0.f ? acc / W : 0.f);
            if (d == 0)
              p.lse[(static_cast<int64_t>(b) * p.Hq + h) * p.Sq + sq] =
                  W > 0.f ? Mn + __logf(W) : NEG;
          }
          if (tid == 0) p.ws_ticket[pr] = 0;
        }
      }
    }
    named_bar_sync(1, nthr);
    if (aborted) break;
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
