// Split-KV decode kernel: speculative + sparse decode (Incremental_FlashAttention
// README, Usage 2) and short-query block-table attention, fused with the LSE
// combine of the per-CTA pieces.
//
// Work layout: every (batch b, kv-head g) pair owns a fixed run of `pp`
// chunk slots of 64 keys -- the dense source A (k_spec/v_spec) cut into
// chunks and kv_block/64 slots per table entry of source B (k/v), the A
// chunks spread evenly among the B ones (dec_slot): the dense range is the
// same keys of every pair and streams more slowly than the scattered table
// blocks, so a CTA whose range held mostly A chunks used to finish last.  The
// slots of all pairs are laid end to end and CTA c of the persistent grid
// takes the contiguous range [total*c/grid, total*(c+1)/grid): the split is
// known at launch, so no CTA scans the table before streaming.  A table
// entry that is padding (< 0) leaves its slots empty: they cost no load.
//
// Inside a CTA two groups of four warps take alternate chunks; each warp
// owns a 16-key slice of its group's chunks and streams the K and V rows of
// its slices into a private three-stage cp.async ring (16-byte copies, zero
// fill past the end), then runs QK^T and PV on mma.sync m16n8k16 (the M = 16
// tile carries the <= 16 query rows of a pair: Sq positions x G query heads).
// At the end of its part of a pair the CTA merges its warps' running
// (m, l, O) and writes either the final row (the pair lies wholly inside its
// range) or an fp32 partial.  A shared pair is finished by whichever CTA
// takes the last ticket; a CTA takes its tickets (at most two: its first and
// last pair) only once it has streamed its whole range, so no warp stalls on
// a fence mid-stream and no warp ever waits on another CTA; the CTA holding
// the last ticket merges all partials with the LSE combine and resets it.
#pragma once

#include "sbfa_ptx.cuh"

namespace sbfa {

constexpr int kDecChunk = 64;
constexpr int kDecGroupWarps = 4;                        // warps per consumer group
constexpr int kDecGroups = 2;                            // groups take alternate chunks
constexpr int kDecWarps = kDecGroups * kDecGroupWarps;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecWarpStages = 3;                        // cp.async ring depth per warp
constexpr int kDecSliceKeys = 16;                        // keys of a chunk one warp owns
constexpr int kDecSliceBytes = 2 * kDecSliceKeys * 128 * 2;  // K + V slice, bf16
constexpr int kDecMaxPairs = 4096;
constexpr int kDecMaxEntries = 1024;
constexpr int kDecRows = 16;
constexpr int kDecD = 128;
constexpr int kDecSharers = 8;  // sharers of a pair listed ahead of time
constexpr int kDecStashRows = 7;  // rows a warp can park in the merge buffer (see stash)

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

struct DecSmem {
  alignas(1024) uint8_t slice[kDecWarps][kDecWarpStages][kDecSliceBytes];
  float ow[kDecGroupWarps][kDecRows][kDecD];
  float mw[kDecGroupWarps][kDecRows];
  float lw[kDecGroupWarps][kDecRows];
  int2 meta[kDecWarps][kDecWarpStages];  // slice in each stage: {key0, nk | src << 7 | pr << 8}
  uint32_t repeat[kDecWarps][2];         // repeat masks of a warp's even / odd chunk windows
  float stm[kDecWarps][kDecStashRows];   // parked first-piece state: running max, sum
  float stl[kDecWarps][kDecStashRows];
  int last[2];                           // this CTA finishes shared pair 0 / 1
  // CTAs sharing this CTA's first / last pair: their partial slots (-1 for
  // an empty range) when there are at most kDecSharers of them, and count
  int share_slot[2][kDecSharers];
  int share_n[2];
  int share_many[2];
};

static_assert(sizeof(DecSmem) + 1024 <= 232448, "decode shared memory exceeds 227 KB");
static_assert(kDecWarps * kDecStashRows * kDecD <= kDecGroupWarps * kDecRows * kDecD,
              "parked first-piece states must fit the merge buffer");

__device__ __forceinline__ int dec_chunks_per_entry(int kv_block) {
  return kv_block >= kDecChunk ? kv_block / kDecChunk : 1;
}

// Slot c of a pair's pp slots: an A chunk (isA, its index a) or a B chunk
// (its index c - a among the B slots).  A chunk a sits at the slot where
// floor(c * nA / pp) steps up.
__device__ __forceinline__ bool dec_slot(int c, int nA, int pp, int& idx) {
  const int a = static_cast<int>((static_cast<int64_t>(c) * nA) / pp);
  const bool isA = static_cast<int>((static_cast<int64_t>(c + 1) * nA) / pp) > a;
  idx = isA ? a : c - a;
  return isA;
}

__device__ __forceinline__ int64_t dec_range_lo(int c, int64_t total, int grid) {
  return (total * c) / grid;
}

// CTA whose range holds global slot x.
__device__ __forceinline__ int dec_cta_of(int64_t x, int64_t total, int grid) {
  int c = static_cast<int>((x * grid) / total);
  while (c + 1 < grid && dec_range_lo(c + 1, total, grid) <= x) ++c;
  while (c > 0 && dec_range_lo(c, total, grid) > x) --c;
  return c;
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

// DEDUP: a block listed more than once in a table row counts once (the
// repeat scan below); without it the kernel trusts the rows to be sets.
template <bool DEDUP>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int npairs = p.B * p.Hkv;
  const int grid = gridDim.x;
  const int cta = blockIdx.x;
  const float NEG = -INFINITY;
  const int nA = p.has_A ? (p.S_A + kDecChunk - 1) / kDecChunk : 0;
  const int cpe = dec_chunks_per_entry(p.kv_block);
  const int kpc = p.kv_block < kDecChunk ? p.kv_block : kDecChunk;  // keys per B slot
  const int pp = nA + (p.has_B ? p.nmax * cpe : 0);                  // slots per pair

  if (pp == 0) {  // no key at all: every row is (o = 0, lse = -inf)
    for (int pr = cta; pr < npairs; pr += grid) {
      const int b = pr / p.Hkv, g = pr % p.Hkv;
      for (int e = tid; e < p.rows * kDecD; e += kDecThreads) {
        const int rr = e / kDecD, d = e % kDecD;
        const int sq = rr / p.G, h = g * p.G + rr % p.G;
        p.o[b * p.osb + sq * p.oss + h * p.osh + d] = __float2bfloat16(0.f);
        if (d == 0) p.lse[(static_cast<int64_t>(b) * p.Hq + h) * p.Sq + sq] = NEG;
      }
    }
    return;
  }
  const int64_t total = static_cast<int64_t>(npairs) * pp;
  // This CTA's slot sequence: stream-K = the global range [lo, hi); pair
  // mode = whole pairs cta, cta + grid, ...
  int64_t lo = 0, hi = 0, N;
  int n_pieces;
  if (p.pair_mode) {
    n_pieces = cta < npairs ? (npairs - cta + grid - 1) / grid : 0;
    N = static_cast<int64_t>(n_pieces) * pp;
  } else {
    lo = dec_range_lo(cta, total, grid);
    hi = dec_range_lo(cta + 1, total, grid);
    n_pieces = hi > lo ? static_cast<int>((hi - 1) / pp - lo / pp + 1) : 0;
    N = hi - lo;
  }
  if (N == 0) return;
  const int pr_first = static_cast<int>(lo / pp), pr_last = static_cast<int>((hi - 1) / pp);
  // A range that ends one pair and starts the next runs its longer piece
  // first: merging a short leading piece stops all warps early in the stream,
  // while DRAM is busiest, and that stall used to make such CTAs finish last.
  // Sequence position 0 is then slot lo + rot and the range wraps around.
  int64_t rot = 0;
  if (!p.pair_mode && n_pieces == 2) {
    const int64_t first_len = static_cast<int64_t>(pr_first + 1) * pp - lo;
    if (first_len < N - first_len) rot = first_len;
  }
  // global slot of sequence position n
  auto seq_x = [&](int64_t n) -> int64_t {
    if (p.pair_mode) return (cta + (n / pp) * grid) * static_cast<int64_t>(pp) + n % pp;
    const int64_t m = n + rot;
    return lo + (m < N ? m : m - N);
  };

  const int grp = warp / kDecGroupWarps, wg = warp % kDecGroupWarps;
  const int gq = lane >> 2, cq = lane & 3;
  const int n_mine = static_cast<int>((N - grp + 1) / 2);  // positions grp, grp + 2, ...
  const int kw = wg * kDecSliceKeys;

  // Slot metadata of this warp's chunks j in [32 w, 32 w + 32), lane j % 32.
  int mkey = 0, minfo = 0;
  auto load_meta = [&](int win) {
    const int j = win * 32 + lane;
    int key0 = 0, info = 0;
    if (j < n_mine) {
      const int64_t x = seq_x(grp + 2 * static_cast<int64_t>(j));
      const int pr = static_cast<int>(x / pp), c = static_cast<int>(x % pp);
      int nk = 0, src = 0, si;
      if (dec_slot(c, nA, pp, si)) {
        key0 = si * kDecChunk;
        nk = min(kDecChunk, p.S_A - key0);
      } else {
        src = 1;
        const int e = si / cpe, sub = si % cpe;
        const int b = pr / p.Hkv, g = pr % p.Hkv;
        const int jb = __ldg(p.idx + b * p.tsb + g * p.tsh + e);
        if (jb >= 0 && jb < p.n_kb) {
          key0 = jb * p.kv_block + sub * kDecChunk;
          nk = max(min(kpc, p.S_B - key0), 0);
        } else if (jb >= p.n_kb) {
          report(p.status, kDevBadIndex);
        }
      }
      info = nk | (src << 7) | (pr << 8);
    }
    mkey = key0;
    minfo = info;
  };

  // With DEDUP, a table row that lists a block more than once counts it
  // once: the chunks of every repeat after its first entry are skipped at
  // compute time (their copies are still made).  Bit j % 32 of the window's mask in shared memory
  // marks a repeat.  For each pair that the window's table chunks belong to,
  // the warp reads the row's leading entries with one coalesced load per 32
  // entries and every lane compares its own entry against the earlier ones
  // by shuffles.  It runs after the window's first copies are issued, while
  // they fly, and keeps nothing in registers across the streaming loop.
  auto load_dup = [&](int win) {
    const int j = win * 32 + lane;
    int pr = 0, e = 0, jb = -1;
    if (j < n_mine) {
      const int64_t x = seq_x(grp + 2 * static_cast<int64_t>(j));
      const int c = static_cast<int>(x % pp);
      int si;
      if (!dec_slot(c, nA, pp, si)) {
        pr = static_cast<int>(x / pp);
        e = si / cpe;
        jb = __ldg(p.idx + (pr / p.Hkv) * p.tsb + (pr % p.Hkv) * p.tsh + e);
        if (jb >= p.n_kb) jb = -1;
      }
    }
    bool dup = false;
    uint32_t todo = __ballot_sync(0xffffffffu, jb >= 0);
    while (todo) {
      const int pr_l = __shfl_sync(0xffffffffu, pr, __ffs(todo) - 1);
      const bool mine = jb >= 0 && pr == pr_l;
      todo &= ~__ballot_sync(0xffffffffu, mine);
      const int emax = static_cast<int>(__reduce_max_sync(0xffffffffu, mine ? e : 0));
      const int* row = p.idx + (pr_l / p.Hkv) * p.tsb + (pr_l % p.Hkv) * p.tsh;
      for (int c0 = 0; c0 < emax; c0 += 32) {
        const int val = c0 + lane < emax ? __ldg(row + c0 + lane) : -1;
        const int n = min(32, emax - c0);
        for (int sl = 0; sl < n; ++sl) {
          const int xv = __shfl_sync(0xffffffffu, val, sl);
          dup |= mine && c0 + sl < e && xv == jb;
        }
      }
    }
    const uint32_t m = __ballot_sync(0xffffffffu, dup);
    if (lane == 0) sm.repeat[warp][win & 1] = m;
    __syncwarp();
  };

  // Stream chunk j's slice of this warp into ring stage j % kDecWarpStages.
  // One commit group per call (empty past the end), so that "all but the
  // newest kDecWarpStages - 1 groups" is always the group of the oldest stage.
  auto issue = [&](int j) {
    const int stage = j % kDecWarpStages;
    if (j < n_mine) {
      if ((j & 31) == 0 && j > 0) {
        load_meta(j >> 5);
        if (DEDUP) load_dup(j >> 5);
      }
      const int key0 = __shfl_sync(0xffffffffu, mkey, j & 31);
      const int info = __shfl_sync(0xffffffffu, minfo, j & 31);
      if (lane == 0) sm.meta[warp][stage] = make_int2(key0, info);
      const int nk = info & 0x7f, src = (info >> 7) & 1, pr = info >> 8;
      if (nk > kw) {
        const int b = pr / p.Hkv, g = pr % p.Hkv;
        const __nv_bfloat16* krow0 =
            src ? p.kB + b * p.kBsb + g * p.kBsh : p.kA + b * p.kAsb + g * p.kAsh;
        const __nv_bfloat16* vrow0 =
            src ? p.vB + b * p.vBsb + g * p.vBsh : p.vA + b * p.vAsb + g * p.vAsh;
        const int64_t kro = src ? p.kBss : p.kAss, vro = src ? p.vBss : p.vAss;
        // each K and V row is 256 contiguous bytes read by 16 lanes: the L2::256B
        // qualifier lets the first copy bring in the whole row
        const uint32_t kdst = smem_u32(sm.slice[warp][stage]);
#pragma unroll
        for (int it = 0; it < kDecSliceKeys * 16 / 32; ++it) {
          const int e = lane + it * 32;
          const int r = e >> 4, ch = e & 15;
          const uint32_t off = (ch >> 3) * (kDecSliceKeys * 128) + sw128_off(r, ch & 7);
          const bool valid = kw + r < nk;
          const int64_t row = valid ? key0 + kw + r : 0;
          const uint32_t bytes = valid ? 16u : 0u;
          asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16, %2;" ::"r"(kdst + off),
                       "l"(krow0 + row * kro + ch * 8), "r"(bytes)
                       : "memory");
          asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16, %2;" ::"r"(
                           kdst + kDecSliceBytes / 2 + off),
                       "l"(vrow0 + row * vro + ch * 8), "r"(bytes)
                       : "memory");
        }
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  // pair of piece pi
  auto piece_pair = [&](int pi) {
    if (p.pair_mode) return cta + pi * grid;
    if (rot) return pi == 0 ? pr_last : pr_first;
    return static_cast<int>(lo / pp) + pi;
  };
  // Rows r0 = gq and r1 = gq + 8 of the M = 16 tile (row = sq * G + head in group)
  // and their causal limits in source A (bottom-right aligned).
  const int r0 = gq, r1 = gq + 8;
  const bool v0 = r0 < p.rows, v1 = r1 < p.rows;
  const int lim0 = v0 ? r0 / p.G + (p.S_A - p.Sq) : -1;
  const int lim1 = v1 ? r1 / p.G + (p.S_A - p.Sq) : -1;
  // Q fragments (A operand, 16 rows x 128) of pair pr.  Loaded one piece
  // ahead, while the previous piece merges, so no warp waits for them.
  uint32_t qa[8][4];
  auto load_q = [&](int pr) {
    const int b = pr / p.Hkv, g = pr % p.Hkv;
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
  };

  // Pull the query rows of pair pr into L2 ahead of their load_q: at a piece
  // boundary the next piece's Q would otherwise cost a DRAM round trip with
  // the whole CTA waiting.  Lane l takes 128-byte line l of the <= 16 rows.
  auto prefetch_q = [&](int pr) {
    const int rr = lane >> 1;
    if (rr < p.rows) {
      const int b = pr / p.Hkv, g = pr % p.Hkv;
      const __nv_bfloat16* a =
          p.q + b * p.qsb + (rr / p.G) * p.qss + (g * p.G + rr % p.G) * p.qsh + (lane & 1) * 64;
      asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
    }
  };

  // the table read and the first copies go out before the Q loads: the
  // copies need the table, Q is needed only once they land
  load_meta(0);
#pragma unroll
  for (int s = 0; s < kDecWarpStages; ++s) issue(s);
  load_q(piece_pair(0));
  // the query rows of the CTA's next pieces travel with the first copies
  if (warp >= 1 && warp < 4 && warp < n_pieces) prefetch_q(piece_pair(warp));
  // Touch the partial slots of this CTA's shared pairs early: the CTA that
  // merges a pair at the end reads the other sharers' slots, and a cold
  // address translation there cost several microseconds at the very end.
  if (!p.pair_mode && warp == 4 && lane < 2 * kDecSharers) {
    const int k = lane / kDecSharers;
    const int pr = k == 0 ? pr_first : pr_last;
    const int cc = dec_cta_of(static_cast<int64_t>(pr) * pp, total, grid) + lane % kDecSharers;
    if (cc < grid) {
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p.ws_part + static_cast<int64_t>(2 * cc) * kDecRows * kDecD));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p.ws_lse + 2 * cc * kDecRows));
    }
  }
  if (DEDUP) load_dup(0);

  // While the first copies are in flight: which CTAs share this CTA's first
  // and last pair, and the partial slot each of them writes (the 64-bit
  // divisions stay off the end of the kernel).
  if (!p.pair_mode && warp == kDecWarps - 1 && lane < 2 * kDecSharers) {
    const int k = lane / kDecSharers, s = lane % kDecSharers;
    const int pr = k == 0 ? pr_first : pr_last;
    const int c_first = dec_cta_of(static_cast<int64_t>(pr) * pp, total, grid);
    const int c_last = dec_cta_of(static_cast<int64_t>(pr + 1) * pp - 1, total, grid);
    const int cc = c_first + s;
    int slot = -1;
    if (cc <= c_last) {
      const int64_t clo = dec_range_lo(cc, total, grid);
      if (clo < dec_range_lo(cc + 1, total, grid)) slot = (clo / pp == pr) ? 2 * cc : 2 * cc + 1;
    }
    sm.share_slot[k][s] = slot;
    const unsigned mask = __ballot_sync(0xffffu, slot >= 0);
    if (s == 0) {
      sm.share_n[k] = __popc(mask >> (k * kDecSharers) & 0xffu);
      sm.share_many[k] = c_last - c_first + 1 > kDecSharers;
    }
  }

  // A two-piece range with at most kDecStashRows query rows does not stop
  // its warps between the pieces: each warp parks its state for the first
  // piece in the merge buffer (no barrier) and streams on; the parked states
  // are merged once at the end, before the last piece's merge reuses the
  // buffer.  Larger row counts merge between the pieces.
  const bool stash = !p.pair_mode && n_pieces == 2 && p.rows <= kDecStashRows;
  float* const sto = &sm.ow[0][0][0];  // parked O: [warp][row < kDecStashRows][d]

  // running state of the piece in progress
  float m0 = NEG, m1 = NEG, l0 = 0.f, l1 = 0.f;
  float oacc[16][4];
  int j = 0;

  for (int pi = 0; pi < n_pieces; ++pi) {
    int pr;
    int64_t nb, ne;
    bool whole;
    pr = piece_pair(pi);
    if (p.pair_mode) {
      nb = static_cast<int64_t>(pi) * pp;
      ne = nb + pp;
      whole = true;
    } else {
      const int64_t a = static_cast<int64_t>(pr) * pp, e = a + pp;
      const int64_t sb = a > lo ? a : lo, se = e < hi ? e : hi;  // its slots
      nb = sb - lo - rot;
      if (nb < 0) nb += N;
      ne = nb + (se - sb);
      whole = a >= lo && e <= hi;
    }
    const int b = pr / p.Hkv, g = pr % p.Hkv;
    if (pi + 4 < n_pieces && warp == 0) prefetch_q(piece_pair(pi + 4));
    m0 = m1 = NEG;
    l0 = l1 = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    const int j_end = static_cast<int>((ne - grp + 1) / 2);  // chunks with grp + 2 j < ne
    for (; j < j_end; ++j) {
      asm volatile("cp.async.wait_group %0;" ::"n"(kDecWarpStages - 1) : "memory");
      __syncwarp();  // this warp's copies are in and visible to all its lanes
      const int stage = j % kDecWarpStages;
      const int2 mt = sm.meta[warp][stage];
      const int key0 = mt.x, nkeys = mt.y & 0x7f, src = (mt.y >> 7) & 1;
      const bool repeat = DEDUP && ((sm.repeat[warp][(j >> 5) & 1] >> (j & 31)) & 1u);
      if (nkeys > kw && !repeat) {
        const uint32_t kbase = smem_u32(sm.slice[warp][stage]);
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
      }
      __syncwarp();  // every lane is done with the stage: refill it
      issue(j + kDecWarpStages);
    }

    if (pi + 1 < n_pieces) load_q(piece_pair(pi + 1));  // this piece's Q is dead
    // ---- merge the eight warps' states for this pair
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (stash && pi == 0) {
      // park the first piece (rows < kDecStashRows: only row r0 = gq is live)
      if (v0) {
        if (cq == 0) {
          sm.stm[warp][gq] = m0;
          sm.stl[warp][gq] = l0;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i)
          *reinterpret_cast<float2*>(sto + (warp * kDecStashRows + gq) * kDecD + i * 8 + 2 * cq) =
              make_float2(oacc[i][0], oacc[i][1]);
      }
      continue;
    }
    if (stash) {
      // every warp has parked the first piece: merge its eight states
      __syncthreads();
      const int pr0 = piece_pair(0);
      const int b0 = pr0 / p.Hkv, g0 = pr0 % p.Hkv;
      const int64_t a0 = static_cast<int64_t>(pr0) * pp;
      const bool whole0 = a0 >= lo && a0 + pp <= hi;
      const int slot0 = (pr0 == pr_first) ? 2 * cta : 2 * cta + 1;
      const int d = tid % kDecD;
      for (int rr = tid / kDecD; rr < p.rows; rr += 2) {
        float M = NEG;
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sm.stm[w][rr]);
        const float Mu = (M == NEG) ? 0.f : M;
        float L = 0.f, acc = 0.f;
        for (int w = 0; w < kDecWarps; ++w) {
          const float wt = ex2_approx(sm.stm[w][rr] - Mu);
          L += wt * sm.stl[w][rr];
          acc += wt * sto[(w * kDecStashRows + rr) * kDecD + d];
        }
        const float ov = L > 0.f ? acc / L : 0.f;
        const float lv = L > 0.f ? (Mu + lg2_approx(L)) * 0.69314718055994531f : NEG;
        const int sq = rr / p.G, h = g0 * p.G + rr % p.G;
        if (whole0) {
          p.o[b0 * p.osb + sq * p.oss + h * p.osh + d] = __float2bfloat16(ov);
          if (d == 0) p.lse[(static_cast<int64_t>(b0) * p.Hq + h) * p.Sq + sq] = lv;
        } else {
          p.ws_part[(static_cast<int64_t>(slot0) * kDecRows + rr) * kDecD + d] = ov;
          if (d == 0) p.ws_lse[slot0 * kDecRows + rr] = lv;
        }
      }
      __syncthreads();  // the parked states are read: the buffer is free below
    }
    // (1) group 1 publishes its state, group 0 folds it into its registers
    if (grp == 1) {
      if (cq == 0) {
        sm.mw[wg][gq] = m0; sm.mw[wg][gq + 8] = m1;
        sm.lw[wg][gq] = l0; sm.lw[wg][gq + 8] = l1;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {  // rows past p.rows are never read back
        const int d = i * 8 + 2 * cq;
        if (v0) *reinterpret_cast<float2*>(&sm.ow[wg][gq][d]) = make_float2(oacc[i][0], oacc[i][1]);
        if (v1) *reinterpret_cast<float2*>(&sm.ow[wg][gq + 8][d]) = make_float2(oacc[i][2], oacc[i][3]);
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
        const float2 x = v0 ? *reinterpret_cast<const float2*>(&sm.ow[wg][gq][d]) : make_float2(0.f, 0.f);
        const float2 y = v1 ? *reinterpret_cast<const float2*>(&sm.ow[wg][gq + 8][d]) : make_float2(0.f, 0.f);
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
      for (int i = 0; i < 16; ++i) {  // rows past p.rows are never read back
        const int d = i * 8 + 2 * cq;
        if (v0) *reinterpret_cast<float2*>(&sm.ow[wg][gq][d]) = make_float2(oacc[i][0], oacc[i][1]);
        if (v1) *reinterpret_cast<float2*>(&sm.ow[wg][gq + 8][d]) = make_float2(oacc[i][2], oacc[i][3]);
      }
    }
    __syncthreads();
    {
      // 256 threads: thread t owns column d = t % 128 of rows r with r % 2 == t / 128
      const int d = tid % kDecD;
      const int rpar = tid / kDecD;
      const int slot = (pr == pr_first) ? 2 * cta : 2 * cta + 1;
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
    }
    __syncthreads();  // merge buffers free
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  if (p.pair_mode) return;

  // ---- shared pairs: the CTA that took the last ticket merges all partials
  const bool split0 = lo > static_cast<int64_t>(pr_first) * pp ||
                      hi < static_cast<int64_t>(pr_first + 1) * pp;
  const bool split1 = n_pieces > 1 && hi < static_cast<int64_t>(pr_last + 1) * pp;
  auto ctas_sharing = [&](int k, int pr) {
    if (!sm.share_many[k]) return sm.share_n[k];
    const int c_first = dec_cta_of(static_cast<int64_t>(pr) * pp, total, grid);
    const int c_last = dec_cta_of(static_cast<int64_t>(pr + 1) * pp - 1, total, grid);
    int n = 0;
    for (int c = c_first; c <= c_last; ++c)
      n += dec_range_lo(c, total, grid) < dec_range_lo(c + 1, total, grid) ? 1 : 0;
    return n;
  };
  if (tid == 0) {
    // One ticket per shared pair.  The fence releases this CTA's partials
    // (the barrier before it orders every thread's writes ahead of it); the
    // two adds are relaxed, so they travel together; the last taker's
    // second fence acquires the other sharers' partials.
    fence_acq_rel_gpu();
    const int ticket0 = split0 ? atom_add_relaxed_gpu(p.ws_ticket + pr_first, 1) : 0;
    const int ticket1 = split1 ? atom_add_relaxed_gpu(p.ws_ticket + pr_last, 1) : 0;
    sm.last[0] = split0 && ticket0 == ctas_sharing(0, pr_first) - 1;
    sm.last[1] = split1 && ticket1 == ctas_sharing(1, pr_last) - 1;
    if (sm.last[0] || sm.last[1]) fence_acq_rel_gpu();
  }
  __syncthreads();
  // when this CTA finishes both of its shared pairs, warps 0-3 merge the
  // first and warps 4-7 the second, side by side
  const bool both = sm.last[0] && sm.last[1];
  for (int k = 0; k < 2; ++k) {
    if (!sm.last[k]) continue;
    if (both && (warp >> 2) != k) continue;
    const int pr = k == 0 ? pr_first : pr_last;
    const int b = pr / p.Hkv, g = pr % p.Hkv;
    const bool many = sm.share_many[k];
    int c_first = 0, c_last = kDecSharers - 1;
    if (many) {
      c_first = dec_cta_of(static_cast<int64_t>(pr) * pp, total, grid);
      c_last = dec_cta_of(static_cast<int64_t>(pr + 1) * pp - 1, total, grid);
    }
    const int d4 = (tid & 31) * 4;
    // one warp per row, four columns per lane; partials fetched four CTAs at a time
    const int w0 = both ? (warp & 3) : warp, ws = both ? 4 : kDecWarps;
    for (int rr = w0; rr < p.rows; rr += ws) {
      float M = NEG, W = 0.f;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int c0 = c_first; c0 <= c_last; c0 += 4) {
        float lv[4];
        float4 ov[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int cc = c0 + u;
          lv[u] = NEG;
          ov[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          int sl = -1;
          if (cc <= c_last) {
            if (!many) {
              sl = sm.share_slot[k][cc - c_first];
            } else {
              const int64_t clo = dec_range_lo(cc, total, grid);
              if (clo < dec_range_lo(cc + 1, total, grid)) sl = (clo / pp == pr) ? 2 * cc : 2 * cc + 1;
            }
          }
          if (sl >= 0) {
            lv[u] = __ldcg(p.ws_lse + sl * kDecRows + rr);
            ov[u] = __ldcg(reinterpret_cast<const float4*>(
                p.ws_part + (static_cast<int64_t>(sl) * kDecRows + rr) * kDecD + d4));
          }
        }
        float Mn = M;
#pragma unroll
        for (int u = 0; u < 4; ++u) Mn = fmaxf(Mn, lv[u]);
        if (Mn == NEG) continue;
        const float a = (M == NEG) ? 0.f : __expf(M - Mn);
        W *= a;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] *= a;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float wt = (lv[u] == NEG) ? 0.f : __expf(lv[u] - Mn);
          W += wt;
          acc[0] += wt * ov[u].x;
          acc[1] += wt * ov[u].y;
          acc[2] += wt * ov[u].z;
          acc[3] += wt * ov[u].w;
        }
        M = Mn;
      }
      const float inv = W > 0.f ? 1.f / W : 0.f;
      const int sq = rr / p.G, h = g * p.G + rr % p.G;
      __nv_bfloat16* op = p.o + b * p.osb + sq * p.oss + h * p.osh + d4;
#pragma unroll
      for (int e = 0; e < 4; ++e) op[e] = __float2bfloat16(acc[e] * inv);
      if (lane == 0)
        p.lse[(static_cast<int64_t>(b) * p.Hq + h) * p.Sq + sq] = W > 0.f ? M + __logf(W) : NEG;
    }
    if (tid == (both ? 128 * k : 0)) p.ws_ticket[pr] = 0;
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
