// NSA selected attention over varlen-packed sequences (Flash-Sparse-Attention
// Quickstart: per-token top-k key blocks of 64, cu_seqlens packing), computed
// block-major as in FSA's loop-order swap: instead of each query token
// walking its own top-k blocks (one query row per kv-head: no tensor-core
// tile), every selected key block gathers the query rows that chose it.
//
//   1. count, scan and fill build the inverted index: for each (kv-head g,
//      block) the list of (token, slot) pairs that selected it (a counting
//      sort).  When the key space fits in shared memory each CTA histograms
//      a token range there and touches each global counter once per key
//      (nsa_count_hist_kernel / nsa_fill_hist_kernel); otherwise warps
//      aggregate equal keys with __match_any_sync (nsa_count_kernel /
//      nsa_fill_kernel).
//   2. nsa_units_kernel flattens the units: one unit = one key block and up
//      to 128 query rows (entries x G query heads) that selected it; the
//      table row of unit u holds its key rows, list entries and kv head.
//   3. nsa_main_kernel<1> (row maxima): every CTA takes its share of the
//      units (chunks of kNsaChunk consecutive units dealt out round-robin,
//      so that the whole grid sweeps the sorted (kv head, sequence, block)
//      order together).  Q rows are gathered four at a time by TMA
//      (tile::gather4 over a (token x head) row map) into a 128B-swizzled
//      tile, K comes by TMA, S = Q K^T runs on tcgen05 into TMEM, and each
//      row's largest visible score over the block (log2 domain) is merged
//      into M[row] with an integer atomic max on an order-preserving key.
//   4. nsa_main_kernel<2> (accumulation): the same units again.  With M[row]
//      the maximum over all of the row's selected keys, P = exp2(S - M) <= 1
//      needs no rescaling between blocks: O = P V runs on tcgen05 and each
//      row's unnormalised O and sum of P are added into an fp32 accumulator
//      [token, head, 128] and l[token, head] by red.global.add, staged so
//      that every reduction instruction covers whole 128-byte row pieces.
//      The sweep order keeps the accumulator rows of the current (kv head,
//      sequence) in L2, so the adds do not go to DRAM.
//   5. nsa_finalize_kernel: o = acc / l in bf16, lse = ln 2 (M + log2 l).
//
// The sum over a row's blocks is the LSE combine of its per-block results
// with every term scaled by exp2(-M) up front; the additions into the
// accumulator happen in no fixed order, so results can differ between runs
// in the last bits of the fp32 sums (never by more than fp32 rounding).
#pragma once

#include <type_traits>

#include "sbfa_ptx.cuh"

namespace sbfa {

struct NsaParams {
  int nseq, total, Hq, Hkv, G, topk, nbps;  // nbps: 64-key blocks per sequence slot
  int causal;
  float scale_log2;
  const int* cu;       // [nseq + 1]
  const int* sel;      // [total, Hkv, topk]
  const __nv_bfloat16* q;
  int64_t qss, qsh;
  int* count;          // [Hkv * NB]
  int* cursor;         // [Hkv * NB]
  int* offset;         // [Hkv * NB + 1]
  int* unit_prefix;    // [Hkv * NB + 1]
  int* list;           // [entries]
  int4* unit_a;        // [max units] {first key row, first list entry, entries, kv head}
  int2* unit_b;        // [max units] {sequence start, sequence end}
  int max_units;
  int hist_tokens;     // tokens per CTA of the shared-memory histogram kernels
  float* acc;          // [total * Hq, 128] unnormalised O, zeroed before pass 2
  float* l_acc;        // [total * Hq] sum of P, zeroed before pass 2
  uint32_t* m_key;     // [total * Hq] order key of M (log2 domain), zeroed before pass 1
  __nv_bfloat16* o;
  int64_t oss, osh;
  float* lse;          // [Hq, total]
  int* status;
  unsigned long long wait_ns;  // bounded-wait limit
};

__device__ __forceinline__ int nsa_seq_of(const int* cu, int nseq, int t) {
  int lo = 0, hi = nseq;  // cu[lo] <= t < cu[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid;
  }
  return lo;
}

// Count and fill walk the selection in tiles of kNsaTokTile tokens: each
// warp takes one (kv head, slot) column at a time with its lanes on
// consecutive tokens, so that equal key blocks within a warp (block 0, the
// local blocks) take one atomic between them (__match_any_sync).
constexpr int kNsaTokTile = 64;
constexpr int kNsaIdxThreads = 256;

__device__ __forceinline__ int nsa_key(const NsaParams& p, int t, int s, int c, bool report_bad) {
  const int j = __ldg(p.sel + static_cast<int64_t>(t) * p.Hkv * p.topk + c);
  if (j < 0) return -1;
  const int L = __ldg(p.cu + s + 1) - __ldg(p.cu + s);
  if (j >= (L + 63) / 64) {
    if (report_bad) report(p.status, kDevBadIndex);
    return -1;
  }
  return (c / p.topk) * p.nseq * p.nbps + s * p.nbps + j;
}

__global__ void __launch_bounds__(kNsaIdxThreads) nsa_count_kernel(NsaParams p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per_tok = p.Hkv * p.topk;
  const int ta = blockIdx.x * kNsaTokTile + lane, tb = ta + 32;
  const int sa = ta < p.total ? nsa_seq_of(p.cu, p.nseq, ta) : 0;
  const int sb = tb < p.total ? nsa_seq_of(p.cu, p.nseq, tb) : 0;
  for (int c = warp; c < per_tok; c += kNsaIdxThreads / 32) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int t = hf ? tb : ta;
      const int key = t < p.total ? nsa_key(p, t, hf ? sb : sa, c, true) : -1;
      const unsigned m = __match_any_sync(0xffffffffu, key);
      if (key >= 0 && lane == __ffs(m) - 1) atomicAdd(&p.count[key], __popc(m));
    }
  }
}

// Shared-memory histogram variants, used when the (kv head, block) key space
// fits in shared memory: every CTA takes a contiguous token range, counts
// its entries per key in shared memory, and touches each global counter once
// per key it saw.  With thousands of entries per key this removes the
// global-atomic bottleneck of the per-entry kernels above.
constexpr int kNsaHistThreads = 1024;
constexpr int kNsaHistMaxKeys = 16384;  // fill keeps two int arrays: 128 KB

__global__ void __launch_bounds__(kNsaHistThreads) nsa_count_hist_kernel(NsaParams p) {
  extern __shared__ int hist[];
  const int n_keys = p.Hkv * p.nseq * p.nbps;
  const int per_tok = p.Hkv * p.topk;
  for (int i = threadIdx.x; i < n_keys; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int64_t e0 = static_cast<int64_t>(blockIdx.x) * p.hist_tokens * per_tok;
  const int64_t e1 = min(static_cast<int64_t>(blockIdx.x + 1) * p.hist_tokens,
                         static_cast<int64_t>(p.total)) * per_tok;
  for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const int t = static_cast<int>(e / per_tok), c = static_cast<int>(e % per_tok);
    const int key = nsa_key(p, t, nsa_seq_of(p.cu, p.nseq, t), c, true);
    if (key >= 0) atomicAdd(&hist[key], 1);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n_keys; i += blockDim.x)
    if (hist[i]) atomicAdd(&p.count[i], hist[i]);
}

__global__ void __launch_bounds__(kNsaHistThreads) nsa_fill_hist_kernel(NsaParams p) {
  extern __shared__ int smem_i[];
  const int n_keys = p.Hkv * p.nseq * p.nbps;
  int* cnt = smem_i;            // this CTA's entries per key, then its cursor per key
  int* base = smem_i + n_keys;  // first list position of this CTA's run per key
  const int per_tok = p.Hkv * p.topk;
  for (int i = threadIdx.x; i < n_keys; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  const int64_t e0 = static_cast<int64_t>(blockIdx.x) * p.hist_tokens * per_tok;
  const int64_t e1 = min(static_cast<int64_t>(blockIdx.x + 1) * p.hist_tokens,
                         static_cast<int64_t>(p.total)) * per_tok;
  for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const int t = static_cast<int>(e / per_tok), c = static_cast<int>(e % per_tok);
    const int key = nsa_key(p, t, nsa_seq_of(p.cu, p.nseq, t), c, false);
    if (key >= 0) atomicAdd(&cnt[key], 1);
  }
  __syncthreads();
  // reserve one contiguous run per key for this CTA's entries
  for (int i = threadIdx.x; i < n_keys; i += blockDim.x) {
    base[i] = cnt[i] ? p.offset[i] + atomicAdd(&p.cursor[i], cnt[i]) : 0;
    cnt[i] = 0;
  }
  __syncthreads();
  for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const int t = static_cast<int>(e / per_tok), c = static_cast<int>(e % per_tok);
    const int key = nsa_key(p, t, nsa_seq_of(p.cu, p.nseq, t), c, false);
    if (key >= 0) p.list[base[key] + atomicAdd(&cnt[key], 1)] = t * p.topk + c % p.topk;
  }
}

// Single CTA: exclusive prefix sums of counts and of units per (g, block).
__global__ void nsa_scan_kernel(NsaParams p) {
  __shared__ int warp_tot[2][32];
  const int n = p.Hkv * p.nseq * p.nbps;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  const int per_unit = 128 / p.G;
  int carry_e = 0, carry_u = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const int c = i < n ? p.count[i] : 0;
    const int u = (c + per_unit - 1) / per_unit;
    int xe = c, xu = u;
    for (int off = 1; off < 32; off <<= 1) {
      const int ye = __shfl_up_sync(0xffffffffu, xe, off);
      const int yu = __shfl_up_sync(0xffffffffu, xu, off);
      if (lane >= off) { xe += ye; xu += yu; }
    }
    if (lane == 31) { warp_tot[0][warp] = xe; warp_tot[1][warp] = xu; }
    __syncthreads();
    int be = 0, bu = 0, te = 0, tu = 0;
    for (int w = 0; w < nw; ++w) {
      if (w < warp) { be += warp_tot[0][w]; bu += warp_tot[1][w]; }
      te += warp_tot[0][w];
      tu += warp_tot[1][w];
    }
    if (i < n) {
      p.offset[i] = carry_e + be + xe - c;
      p.unit_prefix[i] = carry_u + bu + xu - u;
      p.cursor[i] = 0;
    }
    carry_e += te;
    carry_u += tu;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    p.offset[n] = carry_e;
    p.unit_prefix[n] = carry_u;
  }
}

__global__ void __launch_bounds__(kNsaIdxThreads) nsa_fill_kernel(NsaParams p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per_tok = p.Hkv * p.topk;
  const int ta = blockIdx.x * kNsaTokTile + lane, tb = ta + 32;
  const int sa = ta < p.total ? nsa_seq_of(p.cu, p.nseq, ta) : 0;
  const int sb = tb < p.total ? nsa_seq_of(p.cu, p.nseq, tb) : 0;
  for (int c = warp; c < per_tok; c += kNsaIdxThreads / 32) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int t = hf ? tb : ta;
      const int key = t < p.total ? nsa_key(p, t, hf ? sb : sa, c, false) : -1;
      const unsigned m = __match_any_sync(0xffffffffu, key);
      const int leader = __ffs(m) - 1;
      int base = 0;
      if (key >= 0 && lane == leader) base = atomicAdd(&p.cursor[key], __popc(m));
      base = __shfl_sync(0xffffffffu, base, leader);
      if (key >= 0)
        p.list[p.offset[key] + base + __popc(m & ((1u << lane) - 1u))] = t * p.topk + c % p.topk;
    }
  }
}


// ----------------------------------------------------------------------------
// main kernel (two passes over the same units)
// ----------------------------------------------------------------------------
constexpr int kNsaThreads = 384;
constexpr int kNsaChunk = 4;  // consecutive units a CTA takes at a time

// Pass 1 keeps four units in flight (Q and K only); pass 2 two (Q, K, V, P).
struct NsaSmem1 {
  static constexpr int NS = 4;
  alignas(1024) uint8_t q[NS][kQTileBytes];
  alignas(1024) uint8_t k[NS][kTileBytes];
  uint32_t tmem_base;
  int abort_flag;
  uint64_t k_full[NS], q_full[NS][2];  // q_full[stage][producer warp]
  uint64_t s_full[NS], p_full[NS];     // p_full: the warpgroup has read S
  uint64_t mma_drain;  // one final commit: every MMA of the CTA has completed
};
struct NsaSmem2 {
  static constexpr int NS = 2;
  alignas(1024) uint8_t q[NS][kQTileBytes];
  alignas(1024) uint8_t k[NS][kTileBytes];
  alignas(1024) uint8_t v[NS][kTileBytes];
  alignas(1024) uint8_t p[NS][kPTileBytes];
  // epilogue staging: each softmax warp turns its 32 rows x 32 fp32 columns
  // around here so that every reduction instruction covers 128-byte row pieces
  alignas(16) float stage[8][32][32];
  uint32_t tmem_base;
  int abort_flag;
  uint64_t k_full[NS], v_full[NS], q_full[NS][2];
  uint64_t s_full[NS], p_full[NS], o_full[NS];
  uint64_t mma_drain;
};

struct NsaUnit {
  int key0, e0, ne, g;  // first key row (global), first list entry, entries, kv head
  int base, end;        // the sequence's token range [base, end)
};

// One thread per unit: locate its (kv head, block) by binary search over
// the unit prefix sums and write its table row.
__global__ void nsa_units_kernel(NsaParams p) {
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  const int n = p.Hkv * p.nseq * p.nbps;
  const int n_units = p.unit_prefix[n];
  if (u >= n_units || u >= p.max_units) return;
  int lo = 0, hi = n;  // unit_prefix[lo] <= u < unit_prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.unit_prefix[mid] <= u) lo = mid; else hi = mid;
  }
  while (lo + 1 < n && p.unit_prefix[lo + 1] <= u) ++lo;  // skip blocks with no unit
  const int g = lo / (p.nseq * p.nbps);
  const int gb = lo % (p.nseq * p.nbps);
  const int s = gb / p.nbps, j = gb % p.nbps;
  const int per_unit = 128 / p.G;
  const int chunk = u - p.unit_prefix[lo];
  const int cnt = p.offset[lo + 1] - p.offset[lo];
  const int base = p.cu[s];
  p.unit_a[u] = make_int4(base + j * 64, p.offset[lo] + chunk * per_unit,
                          min(per_unit, cnt - chunk * per_unit), g);
  p.unit_b[u] = make_int2(base, p.cu[s + 1]);
}

__device__ __forceinline__ NsaUnit nsa_unit(const NsaParams& p, int u) {
  const int4 a = __ldg(p.unit_a + u);
  const int2 b = __ldg(p.unit_b + u);
  NsaUnit r;
  r.key0 = a.x; r.e0 = a.y; r.ne = a.z; r.g = a.w;
  r.base = b.x; r.end = b.y;
  return r;
}

// This CTA's n-th unit and its number of units: chunks of kNsaChunk
// consecutive units, dealt out round-robin over the CTAs.
__device__ __forceinline__ int nsa_cta_unit(int n) {
  return (n / kNsaChunk) * kNsaChunk * static_cast<int>(gridDim.x) +
         static_cast<int>(blockIdx.x) * kNsaChunk + n % kNsaChunk;
}
__device__ __forceinline__ int nsa_cta_units(int n_all) {
  const int per_round = kNsaChunk * static_cast<int>(gridDim.x);
  const int rounds = n_all / per_round;
  const int rem = n_all - rounds * per_round;
  return rounds * kNsaChunk +
         min(max(rem - static_cast<int>(blockIdx.x) * kNsaChunk, 0), kNsaChunk);
}

// PASS 1: row maxima of S into m_key.  PASS 2: O = exp2(S - M) V and the
// sums of P added into acc / l_acc.  Unit n of this CTA uses stage n % NS of
// the rings; its barriers complete phase (n / NS) & 1.
template <int PASS>
__global__ void __launch_bounds__(kNsaThreads, 1)
    nsa_main_kernel(const __grid_constant__ CUtensorMap mapQ,
                    const __grid_constant__ CUtensorMap mapK,
                    const __grid_constant__ CUtensorMap mapV, const NsaParams p) {
  using Smem = std::conditional_t<PASS == 1, NsaSmem1, NsaSmem2>;
  constexpr int NS = Smem::NS;
  // TMEM columns of stage st: pass 1 S (64); pass 2 S (64, P never goes
  // there) then O (128) at +128
  constexpr int kStageCols = PASS == 1 ? 64 : 256;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_all = min(__ldg(p.unit_prefix + p.Hkv * p.nseq * p.nbps), p.max_units);
  const int n_mine = nsa_cta_units(n_all);
  if (tid == 0) {
    for (int b = 0; b < NS; ++b) {
      mbar_init(&sm.k_full[b], 1);
      mbar_init(&sm.q_full[b][0], 1);  // each producer warp arms its own half
      mbar_init(&sm.q_full[b][1], 1);
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.p_full[b], 128);
      if constexpr (PASS == 2) {
        mbar_init(&sm.v_full[b], 1);
        mbar_init(&sm.o_full[b], 1);
      }
    }
    mbar_init(&sm.mma_drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtx wctx{&sm.abort_flag, p.status, p.wait_ns};

  if (warp == 0 || warp == 3) {
    // ===================== producers: Q rows by TMA gather4, K/V by TMA =====================
    // Warp `half` fills rows [64 half, 64 half + 64) of the Q tile: lane l
    // gathers rows 64 half + 4 (l % 16) + {0..3}, columns [64 (l / 16), +64).
    // Rows past the unit's entries repeat its first row (their scores are
    // masked and their outputs dropped).  Unit rows and list entries are
    // loaded one and two units ahead.
    const int half = warp == 0 ? 0 : 1;
    auto load_codes = [&](const NsaUnit& un, int& c0, int& c1) {
      // list entries of rows 64 half + lane and 64 half + 32 + lane
      const int r0 = half * 64 + lane, r1 = r0 + 32;
      c0 = (r0 / p.G < un.ne) ? __ldg(p.list + un.e0 + r0 / p.G) : -1;
      c1 = (r1 / p.G < un.ne) ? __ldg(p.list + un.e0 + r1 / p.G) : -1;
    };
    NsaUnit cur{}, nxt{};
    int c0 = -1, c1 = -1, n0 = -1, n1 = -1, first = 0, first_n = 0;
    if (n_mine > 0) {
      cur = nsa_unit(p, nsa_cta_unit(0));
      load_codes(cur, c0, c1);
      first = __ldg(p.list + cur.e0);
    }
    if (n_mine > 1) nxt = nsa_unit(p, nsa_cta_unit(1));
    bool ok = true;
    // last unit whose Q (and, for warp 0, K) / V copies this warp issued into
    // each stage, for the drain before exit; a stage is refilled only after
    // its previous contents were consumed, so only that last phase can pend
    int qk_last[NS], v_last[NS];
#pragma unroll
    for (int b = 0; b < NS; ++b) qk_last[b] = v_last[b] = -1;
    // Stage n % NS was last used by unit n - NS: Q and K are free once
    // QK(n - NS) has completed (s_full), V once PV(n - NS) has (o_full).
    for (int n = 0; n < n_mine && ok; ++n) {
      const int b = n % NS;
      const uint32_t pw = ((n / NS) & 1) ^ 1u;
      if (n + 1 < n_mine) {
        load_codes(nxt, n0, n1);
        first_n = __ldg(p.list + nxt.e0);
      }
      NsaUnit nn{};
      if (n + 2 < n_mine) nn = nsa_unit(p, nsa_cta_unit(n + 2));
      if (lane == 0) ok = mbar_wait(&sm.s_full[b], pw, wctx);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      qk_last[b] = n;
      if (lane == 0) mbar_arrive_expect_tx(&sm.q_full[b][half], 64 * 128 * 2);
      if (half == 0 && lane == 0) {
        mbar_arrive_expect_tx(&sm.k_full[b], kTileBytes);
        tma_load_4d(sm.k[b], &mapK, &sm.k_full[b], 0, cur.g, cur.key0, 0);
        tma_load_4d(sm.k[b] + 8192, &mapK, &sm.k_full[b], 64, cur.g, cur.key0, 0);
      }
      __syncwarp();
      {
        const int quad = lane & 15, colh = lane >> 4;
        const int rl = 4 * quad;  // first of this lane's four rows within the warp's 64
        int y[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int rw = rl + i;
          // the sending lane's value is fixed per call: fetch both, choose here
          const int v0 = __shfl_sync(0xffffffffu, c0, rw & 31);
          const int v1 = __shfl_sync(0xffffffffu, c1, rw & 31);
          const int code = rw < 32 ? v0 : v1;
          const int r = half * 64 + rw;
          const int t = (code >= 0 ? code : first) / p.topk;
          y[i] = t * p.Hq + cur.g * p.G + r % p.G;
        }
        tma_gather4_2d(sm.q[b] + colh * 16384 + (half * 64 + rl) * 128, &mapQ,
                       &sm.q_full[b][half], colh * 64, y[0], y[1], y[2], y[3]);
      }
      if constexpr (PASS == 2) {
        if (half == 0) {
          if (lane == 0) {
            ok = mbar_wait(&sm.o_full[b], pw, wctx);
            if (ok) {
              v_last[b] = n;
              mbar_arrive_expect_tx(&sm.v_full[b], kTileBytes);
              tma_load_4d(sm.v[b], &mapV, &sm.v_full[b], 0, cur.g, cur.key0, 0);
              tma_load_4d(sm.v[b] + 8192, &mapV, &sm.v_full[b], 64, cur.g, cur.key0, 0);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
      }
      cur = nxt; nxt = nn;
      c0 = n0; c1 = n1; first = first_n;
    }
    // no copy may still be landing in shared memory when the CTA exits
    __syncwarp();
    if (lane == 0) {
      for (int b = 0; b < NS; ++b) {
        if (qk_last[b] >= 0) {
          const uint32_t ph = (qk_last[b] / NS) & 1;
          mbar_wait_short(&sm.q_full[b][half], ph);
          if (half == 0) mbar_wait_short(&sm.k_full[b], ph);
        }
        if constexpr (PASS == 2)
          if (half == 0 && v_last[b] >= 0) mbar_wait_short(&sm.v_full[b], (v_last[b] / NS) & 1);
      }
    }
  } else if (warp == 1) {
    // ===================== MMA issuer =====================
    // Pass 2 order: QK(0), QK(1), PV(0), QK(2), PV(1), ... so that the softmax
    // of one unit overlaps the QK of the next; S(n + 1) reuses the columns of
    // S(n - 1), whose P was consumed by PV(n - 1), issued before it.  Pass 1
    // has no PV: QK(n) waits until the warpgroup has read S(n - NS).
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16(128, 64, 0);
      const uint64_t qdesc0 = sdesc_sw128(smem_u32(sm.q[0]), 16, 1024);
      const uint64_t kdesc0 = sdesc_sw128(smem_u32(sm.k[0]), 16, 1024);
      bool ok = true;
      auto issue_qk = [&](int n) -> bool {
        const int b = n % NS;
        const uint32_t ph = (n / NS) & 1;
        if (PASS == 1 && n >= NS && !mbar_wait(&sm.p_full[b], ph ^ 1u, wctx)) return false;
        if (!mbar_wait(&sm.q_full[b][0], ph, wctx) || !mbar_wait(&sm.q_full[b][1], ph, wctx) ||
            !mbar_wait(&sm.k_full[b], ph, wctx))
          return false;
        tc_fence_after();
        const uint64_t qd = qdesc0 + (b * kQTileBytes >> 4);
        const uint64_t kd = kdesc0 + (b * kTileBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off_q = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          const uint32_t off_k = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
          umma_ss(tmem + b * kStageCols, qd + off_q, kd + off_k, idesc_qk, kk ? 1u : 0u);
        }
        umma_commit(&sm.s_full[b]);
        return true;
      };
      if constexpr (PASS == 1) {
        for (int n = 0; n < n_mine && ok; ++n) ok = issue_qk(n);
      } else {
        const uint32_t idesc_pv = idesc_bf16(128, 128, 1);
        const uint64_t vdesc0 = sdesc_sw128(smem_u32(sm.v[0]), 8192, 1024);
        const uint64_t pdesc0 = sdesc_sw128(smem_u32(sm.p[0]), 16, 1024);
        auto issue_pv = [&](int n) -> bool {
          const int b = n % NS;
          const uint32_t ph = (n / NS) & 1;
          if (!mbar_wait(&sm.p_full[b], ph, wctx) || !mbar_wait(&sm.v_full[b], ph, wctx))
            return false;
          tc_fence_after();
          const uint64_t pd = pdesc0 + (b * kPTileBytes >> 4);
          const uint64_t vd = vdesc0 + (b * kTileBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ss(tmem + b * kStageCols + 128, pd + (kk * 32 >> 4), vd + (kk * 2048 >> 4),
                    idesc_pv, kk ? 1u : 0u);
          umma_commit(&sm.o_full[b]);
          return true;
        };
        if (n_mine > 0) ok = issue_qk(0);
        for (int n = 0; n < n_mine && ok; ++n) {
          if (n + 1 < n_mine) ok = issue_qk(n + 1);
          if (ok) ok = issue_pv(n);
        }
      }
      // drain every tcgen05 op before TMEM is released: a commit to a barrier
      // nothing else uses completes its single phase only then
      umma_commit(&sm.mma_drain);
      mbar_wait_short(&sm.mma_drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ===================== softmax / epilogue warpgroups (ping-pong) =====================
    const int wg = (warp - 4) >> 2;  // units n = wg, wg + 2, ...
    const int r = tid - 128 - 128 * wg;
    const int quarter = warp & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float NEG = -INFINITY;
    bool ok = true;
    // row codes (and, in pass 2, the row's M) one unit ahead
    NsaUnit un_next{};
    int code_next = -1;
    uint32_t mkey_next = 0;
    auto row_of = [&](const NsaUnit& un, int code) -> int64_t {
      return static_cast<int64_t>(code / p.topk) * p.Hq + un.g * p.G + r % p.G;
    };
    auto fetch = [&](int n) {
      un_next = nsa_unit(p, nsa_cta_unit(n));
      code_next = r / p.G < un_next.ne ? __ldg(p.list + un_next.e0 + r / p.G) : -1;
      if (PASS == 2 && code_next >= 0) mkey_next = p.m_key[row_of(un_next, code_next)];
    };
    if (wg < n_mine) fetch(wg);
    for (int n = wg; n < n_mine && ok; n += 2) {
      const int st = n % NS;
      const uint32_t ph = (n / NS) & 1;
      const uint32_t lane_addr = lane_base + st * kStageCols;
      const NsaUnit un = un_next;
      const int code = code_next;
      const uint32_t mkey = mkey_next;
      if (n + 2 < n_mine) fetch(n + 2);
      const bool valid = code >= 0;
      int tl = 0, L = 0;
      int64_t row = -1;
      if (valid) {
        row = row_of(un, code);
        tl = code / p.topk - un.base;
        L = un.end - un.base;
      }
      // tcgen05.ld is warp-collective: the warp agrees before leaving
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[st], ph, wctx))) { ok = false; break; }
      tc_fence_after();
      float s[64];
      tmem_ld32(lane_addr, s);
      tmem_ld32(lane_addr + 32, s + 32);
      const int kb = un.key0 - un.base;  // first key of the block, sequence-local
      if (__all_sync(0xffffffffu, valid && kb + 63 < L && (!p.causal || kb + 63 <= tl))) {
        // every key of the block is visible to every row of this warp
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] *= p.scale_log2;
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int key = kb + c;
          const bool vis = valid && key < L && (!p.causal || key <= tl);
          s[c] = vis ? s[c] * p.scale_log2 : NEG;
        }
      }
      if constexpr (PASS == 1) {
        // S is in registers: the MMA warp may overwrite its columns
        tc_fence_before();
        mbar_arrive(&sm.p_full[st]);
        float m4[4] = {NEG, NEG, NEG, NEG};
#pragma unroll
        for (int c = 0; c < 64; c += 2) m4[(c >> 1) & 3] = max3(m4[(c >> 1) & 3], s[c], s[c + 1]);
        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        if (valid && mx > NEG) atomicMax(p.m_key + row, f32_order_key(mx));
      } else {
        // ---- P = exp2(S - M) with M the row's maximum over all its blocks
        const float M = f32_from_order_key(mkey);
        const float mu = (M > NEG && M < INFINITY) ? M : 0.f;  // no visible key: key 0 (NaN)
        float l = 0.f;
        uint32_t pk[32];
        {
          float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const float p0 = ex2_approx(s[c] - mu), p1 = ex2_approx(s[c + 1] - mu);
            const int a = ((c >> 1) & 1) * 2;
            add2(l4[a], l4[a + 1], p0, p1);
            pk[c >> 1] = pack_bf16x2(p0, p1);
          }
          l = (l4[0] + l4[1]) + (l4[2] + l4[3]);
        }
        const uint32_t prow = smem_u32(sm.p[st]);
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + sw128_off(r, cc)),
                       "r"(pk[cc * 4]), "r"(pk[cc * 4 + 1]), "r"(pk[cc * 4 + 2]),
                       "r"(pk[cc * 4 + 3])
                       : "memory");
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sm.p_full[st]);
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.o_full[st], ph, wctx))) { ok = false; break; }
        tc_fence_after();
        // 32 columns at a time: each lane parks its row in the warp's staging
        // tile (16-byte pieces rotated by row to spread the banks), then lane
        // group i / 8 of each reduction covers the 128 contiguous bytes of one row
        float (*stg)[32] = sm.stage[warp - 4];
        float ob[32];
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(lane_addr + 128 + c * 32, ob);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            *reinterpret_cast<float4*>(&stg[lane][4 * (i ^ (lane & 7))]) =
                make_float4(ob[4 * i], ob[4 * i + 1], ob[4 * i + 2], ob[4 * i + 3]);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int rr = 4 * i + (lane >> 3), piece = lane & 7;
            const long long dst_row = __shfl_sync(0xffffffffu, static_cast<long long>(row), rr);
            const float4 x = *reinterpret_cast<const float4*>(&stg[rr][4 * (piece ^ (rr & 7))]);
            if (dst_row >= 0) red_add_v4_f32(p.acc + dst_row * 128 + c * 32 + 4 * piece, x);
          }
          __syncwarp();
        }
        if (valid && l > 0.f) atomicAdd(p.l_acc + row, l);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// One warp per (token, query head), four columns a lane: o = acc / l,
// lse = ln 2 (M + log2 l).
__global__ void nsa_finalize_kernel(NsaParams p) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = i >> 5;
  const int lane = static_cast<int>(i & 31);
  if (row >= static_cast<int64_t>(p.total) * p.Hq) return;
  const int t = static_cast<int>(row / p.Hq), h = static_cast<int>(row % p.Hq);
  const float l = p.l_acc[row];
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const float4 x = *reinterpret_cast<const float4*>(p.acc + row * 128 + lane * 4);
  __nv_bfloat16* op = p.o + static_cast<int64_t>(t) * p.oss + h * p.osh + lane * 4;
  reinterpret_cast<__nv_bfloat162*>(op)[0] = __floats2bfloat162_rn(x.x * inv, x.y * inv);
  reinterpret_cast<__nv_bfloat162*>(op)[1] = __floats2bfloat162_rn(x.z * inv, x.w * inv);
  if (lane == 0)
    p.lse[static_cast<int64_t>(h) * p.total + t] =
        l > 0.f ? (f32_from_order_key(p.m_key[row]) + lg2_approx(l)) * 0.69314718055994531f
                : -INFINITY;
}

}  // namespace sbfa
