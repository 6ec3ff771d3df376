// Block-sparse FlashAttention forward on the 5th-generation tensor cores.
//
// One persistent CTA per SM, warp-specialised (384 threads):
//   warp 0      TMA producer for Q and K tiles; builds each work unit's
//               key-tile schedule in shared memory; gathers K rows of
//               vertical columns
//   warp 1      tcgen05 MMA issuer (one lane); owns the TMEM allocation
//   warp 2      producer for V tiles; gathers V rows of vertical columns
//   warp 3      idle
//   warps 4-7   softmax warpgroup of Q tile 0 (one thread per query row)
//   warps 8-11  softmax warpgroup of Q tile 1
//
// Work unit: four 64-row "segments" (head, query rows) that share one kv head:
// with GQA they are heads of one group at the same q-block (K/V tiles are
// loaded once for all of them); without GQA they are four consecutive
// q-blocks of one head.  Segments 0,1 form M = 128 tile 0 and segments 2,3
// tile 1.  Each segment has a set of 64-key blocks (from the block table, the
// causal range, the gate or the vertical/slash lists); the unit walks the
// 128-key tiles that hold a block of any segment, in ascending order, and for
// each tile t with an active segment runs
//   S_t = Q_t K^T        tcgen05.mma M128 N128 K16 x 8, fp32 in TMEM
//   softmax rows; P_t (bf16) written back over S_t in TMEM
//   O_t += P_t V         tcgen05.mma with A from TMEM, M128 N128 K16 x 8
// The two 64-key halves of a tile are tracked separately: a half that no
// segment of a tile keeps contributes no PV instructions, and a half that no
// segment of the unit keeps loads no V.  Rows of an inactive segment or half
// get P = 0.  The online softmax keeps a lazily raised running max (O is
// rescaled only when a row max grows by more than 2^8), which leaves o and
// lse exact.  MMAs of one thread execute in issue order, so the commit that
// signals S_t(e) also proves that PV_t(e-1) has read P_t(e-1) and written O_t.
//
// Gated mode (Block Sparse Flash Attention, Figure 2) runs each unit in two
// phases.  Phase A, the gate, walks every causal key tile once and computes
// S^T = K Q^T for both Q tiles in one M128 N256 MMA (keys on the TMEM lanes,
// the 256 query rows on the columns; two such buffers fill all of TMEM, so
// the next tile's product overlaps the reading of this one).  Each softmax
// warp reads the 32 keys on its lanes and the 128 rows of its Q tile, takes
// the maximum of each 32-key x 64-row piece, and compares it with the
// segment's threshold: a 64 x 64 block's maximum is >= T exactly when the
// maximum of one of its two 32-key pieces is, so each warp ORs its keep bit
// into the unit's keep bitmap on its own (the diagonal block is always kept).
// Phase B is block-table attention over the keep bitmaps: a pruned block
// loads no V and runs no PV, and its keys are never exponentiated.
//
// TMEM (512 columns): tile t uses [256t, 256t+128) for S (fp32) / P (bf16
// pairs, first 64 columns) and [256t+128, 256t+256) for O; the gate's two
// S^T buffers are [0, 256) and [256, 512).
#pragma once

#include "sbfa_ptx.cuh"

namespace sbfa {

enum PrefillMode : int { kModeTable = 0, kModeDense = 1, kModeGated = 2, kModeVS = 3 };

constexpr int kPfThreads = 384;
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr int kMaxKT = 8192;               // 64-key blocks: Sk <= 524288
constexpr int kBmWords = kMaxKT / 32;
constexpr int kMaxCols = 1024;             // union of vertical columns per unit
constexpr int kTileBytes = 64 * 128 * 2;   // 64 keys x 128 dims bf16
constexpr int kKVTileBytes = 128 * 128 * 2;  // 128 keys: [d-chunk][128 rows][128 B]
constexpr int kQTileBytes = 128 * 128 * 2;
constexpr int kPTileBytes = 128 * 64 * 2;

struct PrefillParams {
  int mode;
  int B, Sq, Sk, Hq, Hkv, G;
  int hp, subs_per_unit, n_sub, n_hgrp, n_subgrp, n_units, n_kt;
  int causal, causal_off;
  // unit order: 0 = by q-block group, heaviest first, across heads; 1 = head
  // by head, heaviest group first within a head, so that the CTAs running at
  // the same time gather from the same head's K/V and share it in L2 (the
  // vertical/slash lists of long sequences; for full causal rows the
  // across-head order balances better)
  int head_major;
  float scale, scale_log2;
  void* o;
  int64_t osb, oss, osh;
  int o_f32;
  float* lse;
  int64_t lse_sb, lse_sh;  // lse element strides of batch (sequence) and head
  // varlen: sequences packed along the row axis by cumulative lengths
  // (nullptr: batched layout); the batch index is then the sequence index,
  // Sq / Sk are the longest lengths and o / lse are indexed by packed row
  const int* cu_q;
  const int* cu_k;
  // table mode
  const int* idx;
  int64_t tsb, tsh, tsqb;
  int nmax, q_block, kv_block, n_kb;
  // table blocks of 16 or 32 keys: log2(kv_block), else 0; the listed blocks
  // are then also kept per segment at that granularity (pf_fb) for masking
  int fine_shift;
  // dense mode: causal sliding window of this many keys (0: none); row r
  // sees keys r + causal_off - window < key <= r + causal_off
  int window;
  // gated mode
  const float* T;
  int nqb;
  float* smax_out;
  uint8_t* keep_out;
  // vertical-slash mode
  const int* vs_bc;
  const int* vs_bo;
  int nnz_s;
  const int* vs_cc;
  const int* vs_ci;
  int nnz_v;
  int vs_nqb;
  // q/k/v for column gathers
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  int64_t ksb, kss, ksh, vsb, vss, vsh;
  int* status;
  unsigned long long wait_ns;  // bounded-wait limit
  unsigned long long* prof;  // 32 counters, self-profiling build only
};

struct PfSched {
  uint32_t bm[4][kBmWords];  // per segment: 64-key blocks to visit (gated: gate candidates)
  // vertical-slash mode: the unit's column list; gated mode: the same words
  // hold the keep bitmaps the gate writes ([4][kBmWords], see pf_kb); table
  // mode with 16- or 32-key blocks: the listed blocks per segment (pf_fb)
  int col[kMaxCols];
  uint8_t colmask[kMaxCols];
  int n_words, n_cols;
  int b, g;
  int tb;                  // batch coordinate of the TMA maps (0 when varlen)
  int q_base, q_len;       // the unit's query rows: packed offset and length
  int k_base, k_len, coff;  // its keys; causal offset k_len - q_len
  int seg_valid[4], seg_head[4], seg_row0[4], seg_qb[4];
  float seg_T[4];
};
static_assert(kMaxCols >= 4 * kBmWords, "keep bitmaps share the column list's storage");

__device__ __forceinline__ uint32_t* pf_kb(PfSched& sc) {
  return reinterpret_cast<uint32_t*>(sc.col);
}
__device__ __forceinline__ uint32_t* pf_fb(PfSched& sc) {
  return reinterpret_cast<uint32_t*>(sc.col);
}
__device__ __forceinline__ const uint32_t* pf_fb(const PfSched& sc) {
  return reinterpret_cast<const uint32_t*>(sc.col);
}

// Pairing slot of the gate's exact block maximum: the two warps that hold
// the two 32-key pieces of a 64-key half meet here (no waiting: the second
// to arrive combines and writes).
struct PfPair {
  float v[2][2];  // [warp of the pair][segment of the tile]
  int cnt;
};

struct PfSmem {
  alignas(1024) uint8_t q[2 * kQTileBytes];  // [64-dim chunk][tile][128 rows][128 B]
  alignas(1024) uint8_t k[kKStages][kKVTileBytes];
  alignas(1024) uint8_t v[kVStages][kKVTileBytes];
  PfSched sched[2];
  PfPair pair[2][2][4];  // gate: [tile][key half][ring of items]
  int pv_flag[2];
  uint32_t tmem_base;
  int abort_flag;
  uint64_t sched_full[2], sched_empty[2];
  uint64_t q_full[2], q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  // o_free[t] completes one phase per unit in which tile t ran a PV (its
  // epilogue has read O), and only then: a tile with no block in a unit
  // signals nothing, so the phases cannot run ahead of the MMA warp's waits.
  uint64_t s_full[2], p_full[2], pv_done[2], o_free[2];
  // split P hand-over (gated): p_full[t] then covers half 0 of tile t's P,
  // p_full1[t] half 1 (one barrier per half, so that each completes one
  // phase per key tile and the softmax cannot run one two phases ahead of
  // the MMA warp's wait); pvh0[t]: the PV of half 0 has completed
  uint64_t p_full1[2], pvh0[2];
  uint64_t ga_full[2], ga_free[2];  // gate: S^T buffers written / read
  uint64_t kb_done;                 // gate: the unit's keep bitmaps are complete
  uint64_t mma_drain;  // one final commit: every MMA of the CTA has completed
};

static_assert(sizeof(PfSmem) + 1024 <= 232448, "prefill shared memory exceeds 227 KB");

// Visit the 128-key tiles that hold a 64-key block of any segment (ascending)
// in the bitmaps `bits` ([4][kBmWords]), then the vertical-column chunks of
// 128.  fn(kt, is_col, mem) where bit (2s + h) of mem says segment s takes
// part in half h; stops when fn returns false.
template <bool COLS, class F>
__device__ __forceinline__ bool pf_for_each(const PfSched& sc, const uint32_t* bits, F&& fn) {
  for (int w = 0; w < sc.n_words; ++w) {
    uint32_t wb[4];
    uint32_t any = 0;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      wb[s] = bits[s * kBmWords + w];
      any |= (wb[s] | (wb[s] >> 1)) & 0x55555555u;
    }
    while (any) {
      const int bit = __ffs(any) - 1;  // even: half 0 of tile (32w + bit) / 2
      any &= any - 1u;
      int mem = 0;
#pragma unroll
      for (int s = 0; s < 4; ++s) mem |= ((wb[s] >> bit) & 3) << (2 * s);
      if (!fn((w * 32 + bit) >> 1, false, mem)) return false;
    }
  }
  if (!COLS) return true;
  const int nch = (sc.n_cols + 127) >> 7;
  for (int c = 0; c < nch; ++c) {
    int mem = 0;
    for (int h = 0; h < 2; ++h) {
      const int e0 = c * 128 + h * 64, e1 = min(sc.n_cols, e0 + 64);
      int m = 0;
      for (int e = e0; e < e1; ++e) m |= sc.colmask[e];
#pragma unroll
      for (int s = 0; s < 4; ++s) mem |= ((m >> s) & 1) << (2 * s + h);
    }
    if (!fn(c, true, mem)) return false;
  }
  return true;
}

__device__ __forceinline__ void pf_set_range(uint32_t* bm, int t0, int t1) {
  for (int t = t0; t < t1; ++t) atomicOr(&bm[t >> 5], 1u << (t & 31));
}

// Build the schedule of unit u (whole warp 0).
__device__ void pf_build_sched(const PrefillParams& p, int u, PfSched& sc, int lane) {
  const int per_sg = p.B * p.Hkv * p.n_hgrp;
  const int sg = p.head_major ? p.n_subgrp - 1 - u % p.n_subgrp
                              : p.n_subgrp - 1 - u / per_sg;  // heaviest (latest rows) first
  const int rest = p.head_major ? u / p.n_subgrp : u % per_sg;
  const int hgrp = rest % p.n_hgrp;
  const int bg = rest / p.n_hgrp;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  const int n_words = (p.n_kt + 31) >> 5;
  int q_base = 0, q_len = p.Sq, k_base = 0, k_len = p.Sk;
  if (p.cu_q) {
    q_base = __ldg(p.cu_q + b);
    q_len = __ldg(p.cu_q + b + 1) - q_base;
    k_base = __ldg(p.cu_k + b);
    k_len = __ldg(p.cu_k + b + 1) - k_base;
  }
  const int coff = k_len - q_len;
  const int n_sub = (q_len + 63) / 64;
  const int n_kt = (k_len + 63) / 64;
  const int n_kb = p.mode == kModeTable ? (k_len + p.kv_block - 1) / p.kv_block : 0;
  for (int e = lane; e < 4 * kBmWords; e += 32) (&sc.bm[0][0])[e] = 0u;
  if (p.mode == kModeGated || p.fine_shift)
    for (int e = lane; e < 4 * kBmWords; e += 32) pf_kb(sc)[e] = 0u;
  if (lane == 0) {
    sc.n_words = n_words;
    sc.n_cols = 0;
    sc.b = b;
    sc.g = g;
    sc.tb = p.cu_q ? 0 : b;
    sc.q_base = q_base;
    sc.q_len = q_len;
    sc.k_base = k_base;
    sc.k_len = k_len;
    sc.coff = coff;
  }
  __syncwarp();
  for (int s = 0; s < 4; ++s) {
    const int hs = s % p.hp, ss = s / p.hp;
    const int head = g * p.G + hgrp * p.hp + hs;
    const int sub = sg * p.subs_per_unit + ss;
    const int valid = sub < n_sub;
    const int row0 = sub * 64;
    if (lane == 0) {
      sc.seg_valid[s] = valid;
      sc.seg_head[s] = head;
      sc.seg_row0[s] = row0;
      sc.seg_qb[s] = sub;
      sc.seg_T[s] = (p.mode == kModeGated && valid) ? p.T[head * p.nqb + sub] : 0.f;
    }
    if (!valid) continue;
    // causal limit: last tile any row of the segment may see
    int kt_end = n_kt;
    if (p.causal) {
      const int last_row = min(row0 + 63, q_len - 1);
      const int max_key = last_row + coff;
      kt_end = max_key < 0 ? 0 : min(n_kt, max_key / 64 + 1);
    }
    uint32_t* bm = sc.bm[s];
    if (p.mode == kModeDense || p.mode == kModeGated) {
      // sliding window: the first tile a row of the segment may see
      int kt_begin = 0;
      if (p.window > 0) kt_begin = max(0, row0 + coff - p.window + 1) / 64;
      for (int w = lane; w * 32 < kt_end; w += 32) {
        const int t0 = max(w * 32, kt_begin), t1 = min(kt_end, w * 32 + 32);
        bm[w] = t1 <= t0 ? 0u
                         : ((t1 - t0 == 32) ? 0xffffffffu : ((1u << (t1 - t0)) - 1u)) << (t0 - w * 32);
      }
    } else if (p.mode == kModeTable && p.fine_shift) {
      // 16- or 32-key blocks: one fine bit per listed block, one coarse bit
      // per 64-key tile that holds one
      const int qb = row0 / p.q_block;
      const int* row = p.idx + b * p.tsb + g * p.tsh + qb * p.tsqb;
      uint32_t* fb = pf_fb(sc) + s * kBmWords;
      for (int n = lane; n < p.nmax; n += 32) {
        const int j = row[n];
        if (j < 0) continue;
        if (j >= n_kb) { report(p.status, kDevBadIndex); continue; }
        const int t = (j << p.fine_shift) >> 6;
        if (t >= kt_end) continue;
        atomicOr(&fb[j >> 5], 1u << (j & 31));
        atomicOr(&bm[t >> 5], 1u << (t & 31));
      }
    } else if (p.mode == kModeTable) {
      const int qb = row0 / p.q_block;
      const int* row = p.idx + b * p.tsb + g * p.tsh + qb * p.tsqb;
      const int tpb = p.kv_block / 64;
      for (int n = lane; n < p.nmax; n += 32) {
        const int j = row[n];
        if (j < 0) continue;
        if (j >= n_kb) { report(p.status, kDevBadIndex); continue; }
        pf_set_range(bm, j * tpb, min(kt_end, j * tpb + tpb));
      }
    } else {  // vertical-slash: listed blocks
      const int64_t base = (static_cast<int64_t>(b) * p.Hq + head) * p.vs_nqb + sub;
      const int cnt = min(p.vs_bc[base], p.nnz_s);
      const int* offs = p.vs_bo + base * p.nnz_s;
      for (int n = lane; n < cnt; n += 32) {
        const int off = offs[n];
        if (off < 0 || off >= k_len || (off & 63)) { report(p.status, kDevBadIndex); continue; }
        const int t = off >> 6;
        if (t < kt_end) atomicOr(&bm[t >> 5], 1u << (t & 31));
      }
    }
  }
  __syncwarp();
  if (p.mode == kModeVS && lane == 0) {
    // merge the four ascending column lists (union, with segment membership)
    int cur[4], cnt[4];
    const int* lst[4];
    for (int s = 0; s < 4; ++s) {
      cur[s] = 0;
      cnt[s] = 0;
      lst[s] = nullptr;
      if (!sc.seg_valid[s]) continue;
      const int64_t base =
          (static_cast<int64_t>(b) * p.Hq + sc.seg_head[s]) * p.vs_nqb + sc.seg_qb[s];
      cnt[s] = min(p.vs_cc[base], p.nnz_v);
      lst[s] = p.vs_ci + base * p.nnz_v;
    }
    int n = 0;
    while (true) {
      int best = 0x7fffffff;
      for (int s = 0; s < 4; ++s)
        if (cur[s] < cnt[s]) best = min(best, lst[s][cur[s]]);
      if (best == 0x7fffffff) break;
      int mem = 0;
      for (int s = 0; s < 4; ++s)
        if (cur[s] < cnt[s] && lst[s][cur[s]] == best) { mem |= 1 << s; ++cur[s]; }
      if (best < 0 || best >= k_len) { report(p.status, kDevBadIndex); continue; }
      if (n == kMaxCols) { report(p.status, kDevOverflow); break; }
      sc.col[n] = best;
      sc.colmask[n] = static_cast<uint8_t>(mem);
      ++n;
    }
    sc.n_cols = n;
  }
  __syncwarp();
}

// Gather 64 K or V rows (vertical columns e0 .. e0+63 of the union list)
// into half `half` of a 128-key tile; rows past the list end are zero.
// Whole warp; completes the copies and the proxy fence before returning.
__device__ __forceinline__ void pf_gather_rows(const PfSched& sc, int e0, int half,
                                               const __nv_bfloat16* base, int64_t sb, int64_t ss,
                                               int64_t sh, uint8_t* dst, int lane) {
  const uint32_t d0 = smem_u32(dst) + half * 8192;
  for (int e = lane; e < 64 * 16; e += 32) {
    const int r = e >> 4, ch = e & 15;  // row, 16-byte chunk of the 256-byte row
    const uint32_t saddr = d0 + (ch >> 3) * 16384 + sw128_off(r, ch & 7);
    const int idx = e0 + r;
    if (idx < sc.n_cols) {
      const __nv_bfloat16* src = base + sc.tb * sb +
                                 static_cast<int64_t>(sc.k_base + sc.col[idx]) * ss + sc.g * sh +
                                 ch * 8;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(src) : "memory");
    } else {
      asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(saddr), "r"(0) : "memory");
    }
  }
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  fence_proxy_async_smem();
  __syncwarp();
}

// Halves of a 128-key tile that tile t (segments 2t, 2t+1) takes part in.
__device__ __forceinline__ int pf_tile_halves(int mem, int t) {
  const int m = (mem >> (4 * t)) & 15;
  return (m | (m >> 2)) & 3;
}

// Byte offset of 64-dim chunk c of Q tile t (rows of both tiles are laid
// out back to back within a chunk, so that the gate's N = 256 operand is one
// K-major matrix).
__device__ __forceinline__ uint32_t pf_q_off(int c, int t) {
  return static_cast<uint32_t>(c * 2 * kQTileBytes / 2 + t * (kQTileBytes / 2));
}

// EXT: the mask extensions, a sliding window (dense mode) or 16- / 32-key
// table blocks (table mode); the other instantiations compile without them.
// VL: sequences packed by cumulative lengths (per-unit bases and lengths are
// read from the schedule; otherwise they are the launch's constants).
template <int MODE, bool EXT, bool VL>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap mapQ,
                   const __grid_constant__ CUtensorMap mapK,
                   const __grid_constant__ CUtensorMap mapV, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  PfSmem& sm = *reinterpret_cast<PfSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  constexpr bool gated = MODE == kModeGated;
  constexpr bool has_cols = MODE == kModeVS;
  // P handed to the MMA warp half by half (half 0's P V then runs while
  // half 1 is computed): faster where kept blocks are isolated (gated phase
  // B: 32K 11.9 -> 10.9 ms), slower for full rows, where the extra hand-over
  // costs more than the overlap gains (dense 16K 2.55 -> 2.73 ms)
  constexpr bool split_p = gated;
  unsigned long long pacc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const long long t_start = clock64();

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.sched_full[i], 1);
      mbar_init(&sm.sched_empty[i], 1 + 1 + 256);
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], 128);
      mbar_init(&sm.pv_done[i], 1);
      mbar_init(&sm.p_full1[i], 128);
      mbar_init(&sm.pvh0[i], 1);
      mbar_init(&sm.o_free[i], 128);
      mbar_init(&sm.ga_full[i], 1);
      mbar_init(&sm.ga_free[i], 8);  // one arrival per softmax warp
    }
    mbar_init(&sm.q_empty, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], 1);
    }
    mbar_init(&sm.kb_done, 8);
    mbar_init(&sm.mma_drain, 1);
    for (int i = 0; i < 16; ++i) (&sm.pair[0][0][0])[i].cnt = 0;
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  // V stages start finite (zero); afterwards they only ever hold loaded rows
  for (int i = tid; i < kVStages * kKVTileBytes / 16; i += kPfThreads)
    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(smem_u32(sm.v[0]) + 16 * i),
                 "r"(0)
                 : "memory");
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtx wctx{&sm.abort_flag, p.status, p.wait_ns};

  if (warp == 0) {
    // ============================ Q/K producer ============================
    if (lane == 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
    }
    int ks = 0;
    uint32_t kph = 0;
    // Armed phases, for the drain before exit: bit s of k_armed says stage s
    // was ever filled, bit s of k_par holds the parity of its last fill; q_last
    // is the last unit whose Q tiles were requested.  A stage is refilled only
    // after its previous fill was consumed, so at most the last phase of each
    // barrier can still be pending.
    uint32_t k_armed = 0, k_par = 0;
    int q_last = -1;
    bool ok = true;
    int n = 0;
    for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++n) {
      const int ub = n & 1;
      PfSched& sc = sm.sched[ub];
      if (lane == 0) ok = mbar_wait(&sm.sched_empty[ub], ((n >> 1) & 1) ^ 1u, wctx);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      pf_build_sched(p, u, sc, lane);
      if (lane == 0) {
        mbar_arrive(&sm.sched_full[ub]);
        ok = mbar_wait_t(&sm.q_empty, (n & 1) ^ 1u, wctx, pacc[1]);
        if (ok) {
          q_last = n;
          for (int t = 0; t < 2; ++t) {
            const int nv = sc.seg_valid[2 * t] + sc.seg_valid[2 * t + 1];
            mbar_arrive_expect_tx(&sm.q_full[t], nv * 2 * 8192);
            for (int h = 0; h < 2; ++h) {
              const int s = 2 * t + h;
              if (!sc.seg_valid[s]) continue;
              for (int c = 0; c < 2; ++c)
                tma_load_4d(sm.q + pf_q_off(c, t) + h * 8192, &mapQ, &sm.q_full[t], c * 64,
                            sc.seg_head[s], (VL ? sc.q_base : 0) + sc.seg_row0[s], VL ? 0 : sc.b);
            }
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      auto body = [&](int kt, bool is_col, int mem) -> bool {
        bool good = true;
        if (lane == 0) good = mbar_wait_t(&sm.k_empty[ks], kph ^ 1u, wctx, pacc[0]);
        good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
        if (!good) return false;
        const int halves = (mem | (mem >> 2) | (mem >> 4) | (mem >> 6)) & 3;
        k_armed |= 1u << ks;
        k_par = (k_par & ~(1u << ks)) | (kph << ks);
        if (!has_cols || !is_col) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&sm.k_full[ks], __popc(halves) * 2 * 8192);
            for (int h = 0; h < 2; ++h) {
              if (!((halves >> h) & 1)) continue;
              for (int c = 0; c < 2; ++c)
                tma_load_4d(sm.k[ks] + c * 16384 + h * 8192, &mapK, &sm.k_full[ks], c * 64, sc.g,
                            (VL ? sc.k_base : 0) + kt * 128 + h * 64, VL ? 0 : sc.b);
            }
          }
        } else {
          for (int h = 0; h < 2; ++h)
            if ((halves >> h) & 1)
              pf_gather_rows(sc, kt * 128 + h * 64, h, p.k, p.ksb, p.kss, p.ksh, sm.k[ks], lane);
          if (lane == 0) mbar_arrive(&sm.k_full[ks]);
        }
        if (++ks == kKStages) { ks = 0; kph ^= 1u; }
        return true;
      };
      if (gated) {
        // phase A (the gate) over the candidates, then phase B over what it kept
        ok = pf_for_each<false>(sc, &sc.bm[0][0], body);
        if (ok && lane == 0) ok = mbar_wait(&sm.kb_done, n & 1, wctx);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (ok) ok = pf_for_each<false>(sc, pf_kb(sc), body);
      } else {
        ok = pf_for_each<has_cols>(sc, &sc.bm[0][0], body);
      }
    }
    // no copy may still be landing in shared memory when the CTA exits
    if (lane == 0) {
      for (int i = 0; i < kKStages; ++i)
        if ((k_armed >> i) & 1) mbar_wait_short(&sm.k_full[i], (k_par >> i) & 1);
      if (q_last >= 0)
        for (int t = 0; t < 2; ++t) mbar_wait_short(&sm.q_full[t], q_last & 1);
    }
  } else if (warp == 2) {
    // ============================= V producer =============================
    int vs = 0;
    uint32_t vph = 0;
    uint32_t v_armed = 0, v_par = 0;  // as k_armed / k_par above
    bool ok = true;
    int n = 0;
    for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++n) {
      const int ub = n & 1;
      PfSched& sc = sm.sched[ub];
      if (lane == 0) {
        ok = mbar_wait(&sm.sched_full[ub], (n >> 1) & 1, wctx);
        if (gated && ok) ok = mbar_wait(&sm.kb_done, n & 1, wctx);
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      auto body = [&](int kt, bool is_col, int mem) -> bool {
        bool good = true;
        const int need = (mem | (mem >> 2) | (mem >> 4) | (mem >> 6)) & 3;
        if (!need) return true;
        if (lane == 0) good = mbar_wait_t(&sm.v_empty[vs], vph ^ 1u, wctx, pacc[0]);
        good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
        if (!good) return false;
        v_armed |= 1u << vs;
        v_par = (v_par & ~(1u << vs)) | (vph << vs);
        if (!has_cols || !is_col) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&sm.v_full[vs], __popc(need) * 2 * 8192);
            for (int h = 0; h < 2; ++h) {
              if (!((need >> h) & 1)) continue;
              for (int c = 0; c < 2; ++c)
                tma_load_4d(sm.v[vs] + c * 16384 + h * 8192, &mapV, &sm.v_full[vs], c * 64, sc.g,
                            (VL ? sc.k_base : 0) + kt * 128 + h * 64, VL ? 0 : sc.b);
            }
          }
        } else {
          for (int h = 0; h < 2; ++h)
            if ((need >> h) & 1)
              pf_gather_rows(sc, kt * 128 + h * 64, h, p.v, p.vsb, p.vss, p.vsh, sm.v[vs], lane);
          if (lane == 0) mbar_arrive(&sm.v_full[vs]);
        }
        if (++vs == kVStages) { vs = 0; vph ^= 1u; }
        return true;
      };
      ok = pf_for_each<has_cols>(sc, gated ? pf_kb(sc) : &sc.bm[0][0], body);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.sched_empty[ub]);
    }
    if (lane == 0)
      for (int i = 0; i < kVStages; ++i)
        if ((v_armed >> i) & 1) mbar_wait_short(&sm.v_full[i], (v_par >> i) & 1);
  } else if (warp == 1) {
    // ============================= MMA issuer =============================
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16(128, 128, 0);
      const uint32_t idesc_pv = idesc_bf16(128, 128, 1);
      const uint32_t idesc_ga = idesc_bf16(128, 256, 0);
      // base descriptors; K-step, tile and stage offsets are added to the
      // start address field (bits 0-13, 16-byte units), which cannot overflow
      // inside the shared window
      const uint64_t qdesc0 = sdesc_sw128(smem_u32(sm.q), 16, 1024);
      const uint64_t kdesc0 = sdesc_sw128(smem_u32(sm.k[0]), 16, 1024);
      const uint64_t vdesc0 = sdesc_sw128(smem_u32(sm.v[0]), 16384, 1024);
      int ks = 0, vs = 0;
      uint32_t kph = 0, vph = 0;
      uint32_t pph = 0;   // bit t: p_full[t] phase
      uint32_t ofph = 0;  // bit t: parity of the next o_free[t] phase to wait for
      uint32_t owe = 0;   // bit t: a unit with PV on tile t has not been waited for
      // before writing tile t's O (or, in the gate, all of TMEM): wait for
      // the epilogue of the last unit that accumulated into it
      auto free_o = [&](int t) -> bool {
        if (!((owe >> t) & 1u)) return true;
        if (!mbar_wait_t(&sm.o_free[t], (ofph >> t) & 1u, wctx, pacc[4])) return false;
        ofph ^= 1u << t;
        owe &= ~(1u << t);
        return true;
      };
      int ai = 0;         // gate items issued so far (S^T buffer ai & 1)
      bool ok = true;
      int n = 0;
      // start-address offsets of K-step kk: Q (chunk stride 2 tiles) and K
      auto q_step = [](int kk) { return static_cast<uint32_t>(((kk >> 2) * 2 * kQTileBytes / 2 + (kk & 3) * 32) >> 4); };
      auto k_step = [](int kk) { return static_cast<uint32_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4); };
      for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++n) {
        const int ub = n & 1;
        PfSched& sc = sm.sched[ub];
        ok = mbar_wait(&sm.sched_full[ub], (n >> 1) & 1, wctx);
        if (!ok) break;
        ok = mbar_wait_t(&sm.q_full[0], n & 1, wctx, pacc[5]) &&
             mbar_wait_t(&sm.q_full[1], n & 1, wctx, pacc[5]);
        if (!ok) break;
        int pv_started = 0;    // bit t
        if (gated) {
          // The gate's S^T buffers cover all of TMEM, O included: the previous
          // unit's epilogue must have read O first.
          ok = free_o(0) && free_o(1);
          if (!ok) break;
          tc_fence_after();
          auto gate = [&](int kt, bool, int) -> bool {
            if (!mbar_wait_t(&sm.k_full[ks], kph, wctx, pacc[0])) return false;
            const int b = ai & 1;
            if (!mbar_wait_t(&sm.ga_free[b], ((ai >> 1) & 1) ^ 1u, wctx, pacc[2])) return false;
            tc_fence_after();
            const uint64_t kd = kdesc0 + static_cast<uint64_t>((ks * kKVTileBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ss(tmem + b * 256, kd + k_step(kk), qdesc0 + q_step(kk), idesc_ga, kk ? 1u : 0u);
            umma_commit(&sm.ga_full[b]);
            umma_commit(&sm.k_empty[ks]);
            if (++ks == kKStages) { ks = 0; kph ^= 1u; }
            ++ai;
            return true;
          };
          ok = pf_for_each<false>(sc, &sc.bm[0][0], gate);
          // phase B reuses the S^T buffers: both must have been read
          for (int i = 1; i <= 2 && ok && ai - i >= 0; ++i)
            ok = mbar_wait_t(&sm.ga_free[(ai - i) & 1], ((ai - i) >> 1) & 1, wctx, pacc[2]);
          if (ok) ok = mbar_wait(&sm.kb_done, n & 1, wctx);
          if (!ok) break;
          tc_fence_after();
        }
        // Issue order (two-tile ping-pong): QK(e,t0), PV(e-1,t1), QK(e,t1),
        // PV(e,t0).  Each softmax warpgroup then computes while the tensor core
        // runs the other tile's work.  The V stage of item e is released after
        // PV(e,t1), which is issued while handling item e+1.
        struct Pending {
          int valid, act1, f0, v_waited, f1;  // f1: split mode only
        } pend = {0, 0, 0, 0, 0};
        auto issue_pv = [&](int t, int flag) -> bool {
          if (!((pv_started >> t) & 1)) {
            if (!free_o(t)) return false;
            tc_fence_after();
          }
          const uint64_t vd = vdesc0 + static_cast<uint64_t>((vs * kKVTileBytes) >> 4);
          uint32_t acc = (pv_started >> t) & 1;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            if (!((flag >> (kk >> 2)) & 1)) continue;
            umma_ts(tmem + t * 256 + 128, tmem + t * 256 + kk * 8, vd + ((kk * 2048) >> 4),
                    idesc_pv, acc);
            acc = 1;
          }
          pv_started |= 1 << t;
          umma_commit(&sm.pv_done[t]);
          return true;
        };
        // Split mode: tile t's PV half by half as the softmax hands over P (flag:
        // the halves any segment keeps, from the schedule), half 0's PV
        // committed to pvh0 before half 1 is waited for.  The V stage must be in.
        auto pv_split = [&](int t, int flag, int& v_waited) -> bool {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (!mbar_wait_t(h == 0 ? &sm.p_full[t] : &sm.p_full1[t], (pph >> t) & 1u, wctx,
                             pacc[2]))
              return false;
            if ((flag >> h) & 1) {
              if (!v_waited) {
                if (!mbar_wait_t(&sm.v_full[vs], vph, wctx, pacc[3])) return false;
                v_waited = 1;
              }
              tc_fence_after();
              if (!((pv_started >> t) & 1) && !free_o(t)) return false;
              tc_fence_after();
              const uint64_t vd = vdesc0 + static_cast<uint64_t>((vs * kKVTileBytes) >> 4);
              uint32_t acc = (pv_started >> t) & 1;
#pragma unroll
              for (int kk = 4 * h; kk < 4 * h + 4; ++kk) {
                umma_ts(tmem + t * 256 + 128, tmem + t * 256 + kk * 8, vd + ((kk * 2048) >> 4),
                        idesc_pv, acc);
                acc = 1;
              }
              pv_started |= 1 << t;
            }
            umma_commit(h == 0 ? &sm.pvh0[t] : &sm.pv_done[t]);
          }
          pph ^= 1u << t;
          return true;
        };
        auto finish_prev = [&]() -> bool {
          if (split_p) {
            if (pend.act1 && !pv_split(1, pend.f1, pend.v_waited)) return false;
            if (pend.f0 | pend.f1) {
              umma_commit(&sm.v_empty[vs]);
              if (++vs == kVStages) { vs = 0; vph ^= 1u; }
            }
            pend.valid = 0;
            return true;
          }
          int f1 = 0;
          if (pend.act1) {
            if (!mbar_wait_t(&sm.p_full[1], (pph >> 1) & 1u, wctx, pacc[2])) return false;
            pph ^= 2u;
            f1 = sm.pv_flag[1];
          }
          if (pend.f0 | f1) {
            if (f1) {
              if (!pend.v_waited) {
                if (!mbar_wait_t(&sm.v_full[vs], vph, wctx, pacc[3])) return false;
                tc_fence_after();
              }
              if (!issue_pv(1, f1)) return false;
            }
            umma_commit(&sm.v_empty[vs]);
            if (++vs == kVStages) { vs = 0; vph ^= 1u; }
          }
          pend.valid = 0;
          return true;
        };
        auto issue_qk = [&](int t, uint64_t kd) {
          const uint64_t qd = qdesc0 + static_cast<uint64_t>(pf_q_off(0, t) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tmem + t * 256, qd + q_step(kk), kd + k_step(kk), idesc_qk, kk ? 1u : 0u);
          umma_commit(&sm.s_full[t]);
        };
        auto body = [&](int kt, bool is_col, int mem) -> bool {
          const int act = (pf_tile_halves(mem, 0) ? 1 : 0) | (pf_tile_halves(mem, 1) ? 2 : 0);
          if (!mbar_wait_t(&sm.k_full[ks], kph, wctx, pacc[0])) return false;
          pacc[7] += 1;
          tc_fence_after();
          const uint64_t kd = kdesc0 + static_cast<uint64_t>((ks * kKVTileBytes) >> 4);
          if (act & 1) issue_qk(0, kd);
          if (pend.valid && !finish_prev()) return false;
          if (act & 2) issue_qk(1, kd);
          umma_commit(&sm.k_empty[ks]);
          if (++ks == kKStages) { ks = 0; kph ^= 1u; }
          int f0 = 0, v_waited = 0;
          if (split_p) {
            f0 = pf_tile_halves(mem, 0);
            if ((act & 1) && !pv_split(0, f0, v_waited)) return false;
            pend = {1, (act >> 1) & 1, f0, v_waited, pf_tile_halves(mem, 1)};
            return true;
          }
          if (act & 1) {
            if (!mbar_wait_t(&sm.p_full[0], pph & 1u, wctx, pacc[2])) return false;
            pph ^= 1u;
            f0 = sm.pv_flag[0];
            if (f0) {
              if (!mbar_wait_t(&sm.v_full[vs], vph, wctx, pacc[3])) return false;
              tc_fence_after();
              v_waited = 1;
              if (!issue_pv(0, f0)) return false;
            }
          }
          pend = {1, (act >> 1) & 1, f0, v_waited, 0};
          return true;
        };
        ok = pf_for_each<has_cols>(sc, gated ? pf_kb(sc) : &sc.bm[0][0], body);
        if (ok && pend.valid) ok = finish_prev();
        owe |= static_cast<uint32_t>(pv_started);
        umma_commit(&sm.q_empty);
        mbar_arrive(&sm.sched_empty[ub]);
      }
      // every issued tcgen05 op must finish before TMEM is freed: a commit
      // to a barrier nothing else uses completes its single phase only then
      umma_commit(&sm.mma_drain);
      mbar_wait_short(&sm.mma_drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ============================ softmax warpgroups ============================
    const int t = (warp - 4) >> 2;        // tile
    const int r = tid - 128 - 128 * t;    // row in tile == TMEM lane
    const int quarter = (warp & 3);
    const int hseg = r >> 6;              // 0/1: segment within tile
    const int seg = 2 * t + hseg;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t lane_addr = lane_base + t * 256;
    const float NEG = -INFINITY;
    uint32_t sph = 0;
    uint32_t pv_total = 0;  // PVs issued for this tile so far (pv_done phases)
    int ai = 0;             // gate items read so far
    bool ok = true;
    int n = 0;
    for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++n) {
      const int ub = n & 1;
      PfSched& sc = sm.sched[ub];
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.sched_full[ub], (n >> 1) & 1, wctx));
      if (!ok) break;
      if (gated) {
        // ---- phase A: the gate.  This warp holds keys 32*quarter .. +31 of
        // each tile (lanes) and the 128 rows of Q tile t (columns).
        const int key_l = quarter * 32 + lane;
        const int h = quarter >> 1;
        auto gate = [&](int kt, bool, int mem) -> bool {
          const int b = ai & 1;
          if (!__all_sync(0xffffffffu, mbar_wait_t(&sm.ga_full[b], (ai >> 1) & 1, wctx, pacc[0])))
            return false;
          tc_fence_after();
          const int key = kt * 128 + key_l;
          const int j = 2 * kt + h;  // 64-key block of this warp's keys
          float wm[2];
#pragma unroll
          for (int ss = 0; ss < 2; ++ss) {
            const int s = 2 * t + ss;
            const int row0 = sc.seg_row0[s];
            // visible query rows row0 + c of this key: c in [lo, hi)
            int lo = 0, hi = min(64, p.Sq - row0);
            if (p.causal) lo = max(0, key - row0 - p.causal_off);
            if (!((mem >> (2 * s + h)) & 1) || key >= p.Sk) hi = 0;
            float x[64];
            tmem_ld64(lane_base + b * 256 + t * 128 + ss * 64, x);
            float m4[4] = {NEG, NEG, NEG, NEG};
            if (lo == 0 && hi == 64) {
#pragma unroll
              for (int c = 0; c < 64; c += 2) m4[(c >> 1) & 3] = max3(m4[(c >> 1) & 3], x[c], x[c + 1]);
            } else {
#pragma unroll
              for (int c = 0; c < 64; ++c)
                m4[c & 3] = fmaxf(m4[c & 3], (c >= lo && c < hi) ? x[c] : NEG);
            }
            wm[ss] = warp_max_f32(fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&sm.ga_free[b]);
            uint32_t* kb = pf_kb(sc);
#pragma unroll
            for (int ss = 0; ss < 2; ++ss) {
              const int s = 2 * t + ss;
              if (!((mem >> (2 * s + h)) & 1)) continue;
              // BSFA Figure 2b: keep iff diagonal or s_max >= T
              if (j == sc.seg_qb[s] || wm[ss] * p.scale >= sc.seg_T[s])
                atomicOr(&kb[s * kBmWords + (j >> 5)], 1u << (j & 31));
            }
            if (p.smax_out) {
              // exact block maximum: the two warps of this key half pair up
              PfPair& ps = sm.pair[t][h][ai & 3];
              ps.v[quarter & 1][0] = wm[0];
              ps.v[quarter & 1][1] = wm[1];
              __threadfence_block();
              if (atomicAdd(&ps.cnt, 1) == 1) {
                __threadfence_block();
#pragma unroll
                for (int ss = 0; ss < 2; ++ss) {
                  const int s = 2 * t + ss;
                  if (!((mem >> (2 * s + h)) & 1)) continue;
                  const float bm = fmaxf(wm[ss], ps.v[(quarter & 1) ^ 1][ss]);
                  p.smax_out[((static_cast<int64_t>(sc.b) * p.Hq + sc.seg_head[s]) * p.nqb +
                              sc.seg_qb[s]) * p.nqb + j] = bm * p.scale;
                }
                ps.cnt = 0;
              }
            }
          }
          ++ai;
          return true;
        };
        ok = pf_for_each<false>(sc, &sc.bm[0][0], gate);
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.kb_done);
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.kb_done, n & 1, wctx));
        if (!ok) break;
        if (p.keep_out && sc.seg_valid[seg]) {
          const uint32_t* kb = pf_kb(sc) + seg * kBmWords;
          const int qb = sc.seg_qb[seg];
          uint8_t* dst = p.keep_out + ((static_cast<int64_t>(sc.b) * p.Hq + sc.seg_head[seg]) * p.nqb +
                                       qb) * p.nqb;
          for (int jj = (r & 63); jj <= qb; jj += 64) dst[jj] = (kb[jj >> 5] >> (jj & 31)) & 1u;
        }
      }
      // ---- attention over the unit's blocks (gated: the blocks the gate kept)
      const int my_valid = sc.seg_valid[seg];
      const int my_row = sc.seg_row0[seg] + (r & 63);
      const bool row_ok = my_valid && my_row < (VL ? sc.q_len : p.Sq);
      const int u_coff = VL ? sc.coff : p.causal_off;  // this unit's causal offset
      float m_used = NEG, l = 0.f;
      int npv = 0;
      auto body = [&](int kt, bool is_col, int mem) -> bool {
        const int tmask = pf_tile_halves(mem, t);
        if (!tmask) return true;
        const int segm = row_ok ? (mem >> (2 * seg)) & 3 : 0;
        // tcgen05.ld below is warp-collective: the warp leaves together
        if (!__all_sync(0xffffffffu, mbar_wait_t(&sm.s_full[t], sph, wctx, pacc[0]))) return false;
        sph ^= 1u;
        tc_fence_after();
        pacc[5] += 1;
        // ---- pass 1: masks and per-half row maxima (one 64-column half at a time)
        auto mask_half = [&](float* sh, int h) {
          if (has_cols && is_col) {
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const int e = kt * 128 + 64 * h + c;
              bool vis = ((segm >> h) & 1) && e < sc.n_cols && ((sc.colmask[e] >> seg) & 1);
              if (vis && p.causal) vis = sc.col[e] <= my_row + u_coff;
              sh[c] = vis ? sh[c] : NEG;
            }
          } else {
            const int key0 = kt * 128 + 64 * h;
            int lim = ((segm >> h) & 1) ? 64 : 0;
            lim = min(lim, (VL ? sc.k_len : p.Sk) - key0);
            if (p.causal) lim = min(lim, my_row + u_coff - key0 + 1);
            if (!EXT) {
              if (lim < 64) {
#pragma unroll
                for (int c = 0; c < 64; ++c) sh[c] = (c < lim) ? sh[c] : NEG;
              }
            } else {
              // first visible key of a sliding window
              const int lo = p.window > 0 ? my_row + u_coff - p.window + 1 - key0 : 0;
              // 16- or 32-key table blocks: which of the half's blocks are listed
              uint32_t fm = 0xffffffffu;
              bool part = false;
              if (p.fine_shift) {
                const int j0 = key0 >> p.fine_shift;  // first fine block of the half
                const uint32_t all = (1u << (64 >> p.fine_shift)) - 1u;
                fm = pf_fb(sc)[seg * kBmWords + (j0 >> 5)] >> (j0 & 31);
                part = (fm & all) != all;
              }
              if (lim < 64 || lo > 0 || part) {
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                  const bool listed = !p.fine_shift || ((fm >> (c >> p.fine_shift)) & 1u);
                  sh[c] = (c < lim && c >= lo && listed) ? sh[c] : NEG;
                }
              }
            }
          }
        };
        // ---- one pass per 64-key half: mask, row max, P = exp2(s - m) into
        // TMEM as bf16 pairs over the first 64 columns of S (half 0 -> columns
        // 0..31, half 1 -> 32..63; half 1 is read from columns 64..127, which
        // P never overwrites).  The running max m is raised (lazily: only past
        // 2^8) from each half's max as it comes; if half 1 raises it, half 0's
        // P, already in TMEM, is scaled to the new m (rare after a row's first
        // tiles).  O and l of earlier tiles take the product of the factors.
        // With split_p each half is handed over as soon as it is written, and
        // O goes to the new scale before that half's P V is added.
        const int my_keep = segm;
        const int flag = tmask;
        float alpha = 1.f, psum = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
          const bool mine = (my_keep >> h) & 1;
          // tcgen05.ld is warp-collective: load when any lane of the warp keeps
          // this half (rows differ in validity inside a ragged block)
          if (__any_sync(0xffffffffu, mine)) {
            float sh[64];
            tmem_ld64(lane_addr + 64 * h, sh);
            mask_half(sh, h);
            float a_h = 1.f;
            if (mine) {
              float m4[4] = {NEG, NEG, NEG, NEG};
#pragma unroll
              for (int c = 0; c < 64; c += 2) m4[(c >> 1) & 3] = max3(m4[(c >> 1) & 3], sh[c], sh[c + 1]);
              const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
              if (mx != NEG) {
                const float mrow = mx * p.scale_log2;
                if (mrow > m_used + 8.f) {
                  a_h = ex2_approx(m_used - mrow);  // 0 while m_used = -inf
                  m_used = mrow;
                }
              }
            }
            if (split_p) {
              // half 0 was handed over already: O (earlier tiles, or for half 1
              // also half 0's P V, once it has completed) goes to the new scale
              // before this half's P V is added
              if ((npv > 0 || h == 1) && __any_sync(0xffffffffu, a_h != 1.f)) {
                if (h == 1) {
                  pacc[4] += 1;
                  if (!__all_sync(0xffffffffu,
                                  mbar_wait_t(&sm.pvh0[t], pv_total & 1, wctx, pacc[1])))
                    return false;
                  tc_fence_after();
                }
                float ob[32];
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                  tmem_ld32(lane_addr + 128 + c * 32, ob);
#pragma unroll
                  for (int i = 0; i < 32; i += 2) mul2(ob[i], ob[i + 1], a_h);
                  tmem_st32(lane_addr + 128 + c * 32, ob);
                }
              }
              l *= a_h;
            } else if (h == 1 && __any_sync(0xffffffffu, a_h != 1.f)) {
              pacc[4] += 1;
              tmem_wait_st();
              float pf[32];
              tmem_ld32(lane_addr, pf);
              uint32_t* pu = reinterpret_cast<uint32_t*>(pf);
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                const float lo = __uint_as_float(pu[c] << 16) * a_h;
                const float hi = __uint_as_float(pu[c] & 0xffff0000u) * a_h;
                pu[c] = pack_bf16x2(lo, hi);
              }
              tmem_st32_nowait(lane_addr, pf);
              psum *= a_h;
            }
            alpha *= a_h;
            const float mu = (m_used == NEG) ? 0.f : m_used;
            const float base = mine ? mu : INFINITY;  // exp2(-inf) = 0 for lanes without it
            float ps4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              float x0, x1;
              fma2(x0, x1, sh[c], sh[c + 1], p.scale_log2, -base);
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              const int a = ((c >> 1) & 1) * 2;
              add2(ps4[a], ps4[a + 1], p0, p1);
              pk[c >> 1] = pack_bf16x2(p0, p1);
            }
            if (split_p) l += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
            else psum += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) pk[c] = 0u;
          }
          if (split_p) {
            tmem_st32(lane_addr + 32 * h, reinterpret_cast<const float*>(pk));
            tc_fence_before();
            mbar_arrive(h == 0 ? &sm.p_full[t] : &sm.p_full1[t]);
          } else if (h == 0) {
            tmem_st32_nowait(lane_addr, reinterpret_cast<const float*>(pk));
          } else {
            tmem_st32(lane_addr + 32, reinterpret_cast<const float*>(pk));
          }
        }
        if (split_p) {  // l already took each half's factor and sum
          ++npv;
          ++pv_total;
          return true;
        }
        // the commit behind s_full also covers the previous PV: O is stable here
        if (npv > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          pacc[6] += 1;
          float ob[32];
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            tmem_ld32(lane_addr + 128 + c * 32, ob);
#pragma unroll
            for (int i = 0; i < 32; i += 2) mul2(ob[i], ob[i + 1], alpha);
            tmem_st32(lane_addr + 128 + c * 32, ob);
          }
        }
        l = l * alpha + psum;
        tc_fence_before();
        if (r == 0) sm.pv_flag[t] = flag;
        mbar_arrive(&sm.p_full[t]);
        ++npv;
        ++pv_total;
        pacc[7] += 1;
        return true;
      };
      ok = pf_for_each<has_cols>(sc, gated ? pf_kb(sc) : &sc.bm[0][0], body);
      if (!ok) break;
      // ---- epilogue: o = O / l, lse = ln(sum)
      const bool store = row_ok;
      const int head = sc.seg_head[seg];
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      if (npv > 0) {
        const bool okd = __all_sync(0xffffffffu,
                                    mbar_wait_t(&sm.pv_done[t], (pv_total - 1) & 1, wctx, pacc[1]));
        if (!okd) { ok = false; break; }
        tc_fence_after();
        float ob[32];
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(lane_addr + 128 + c * 32, ob);
          if (store) {
            const int64_t off = sc.b * p.osb + static_cast<int64_t>((VL ? sc.q_base : 0) + my_row) *
                                p.oss + head * p.osh + c * 32;
#pragma unroll
            for (int i = 0; i < 32; i += 2) mul2(ob[i], ob[i + 1], inv_l);
            if (p.o_f32) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + off);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(ob[4 * i], ob[4 * i + 1], ob[4 * i + 2], ob[4 * i + 3]);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + off);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(pack_bf16x2(ob[8 * i], ob[8 * i + 1]),
                                    pack_bf16x2(ob[8 * i + 2], ob[8 * i + 3]),
                                    pack_bf16x2(ob[8 * i + 4], ob[8 * i + 5]),
                                    pack_bf16x2(ob[8 * i + 6], ob[8 * i + 7]));
            }
          }
        }
      } else if (store) {
        const int64_t off = sc.b * p.osb + static_cast<int64_t>((VL ? sc.q_base : 0) + my_row) *
                            p.oss + head * p.osh;
        for (int c = 0; c < 128; c += 4) {
          if (p.o_f32)
            *reinterpret_cast<float4*>(static_cast<float*>(p.o) + off + c) = make_float4(0, 0, 0, 0);
          else
            *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.o) + off + c) = make_uint2(0, 0);
        }
      }
      if (store)
        p.lse[sc.b * p.lse_sb + head * p.lse_sh + (VL ? sc.q_base : 0) + my_row] =
            l > 0.f ? (m_used + lg2_approx(l)) * 0.69314718055994531f : NEG;
      if (npv > 0) {  // O was read: the MMA warp may write it again
        tc_fence_before();
        mbar_arrive(&sm.o_free[t]);
      }
      mbar_arrive(&sm.sched_empty[ub]);
    }
  }
  // warp 3 idles (reserved)
#if SBFA_PROF_ON
  if (p.prof) {
    int base = -1;
    if (tid == 0) base = 0;            // Q/K producer
    else if (tid == 64) base = 8;      // V producer
    else if (tid == 32) base = 16;     // MMA issuer
    else if (tid == 128) base = 24;    // softmax tile 0
    if (base >= 0) {
      for (int i = 0; i < 8; ++i) atomicAdd(p.prof + base + i, pacc[i]);
      if (base == 24) atomicAdd(p.prof + 32, static_cast<unsigned long long>(clock64() - t_start));
    }
  }
#else
  (void)t_start;
  (void)pacc;
#endif
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace sbfa
