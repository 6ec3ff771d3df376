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
//   3. nsa_main_kernel: every CTA takes a contiguous range of units (units
//      of one key block are adjacent, so neighbouring CTAs share K/V tiles
//      in L2).  Q rows are gathered four at a time by TMA (tile::gather4
//      over a (token x head) row map) into a 128B-swizzled tile, K/V come by
//      TMA, S = Q K^T and O = P V run on tcgen05 with fp32 accumulators in
//      TMEM.  Each row's result over that one block is an fp32 partial
//      (o, lse) stored at its (token, head, slot); the epilogue stages each
//      warp's rows in shared memory so that stores write whole 128-byte rows.
//   4. nsa_combine_kernel merges the top-k partials of every (token, head)
//      with the LSE combine.
#pragma once

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
  float* part_o;       // [total * Hq * topk, 128]
  float* part_lse;     // [total * Hq * topk]
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
// main kernel
// ----------------------------------------------------------------------------
constexpr int kNsaThreads = 384;

struct NsaSmem {
  alignas(1024) uint8_t q[2][kQTileBytes];
  alignas(1024) uint8_t k[2][kTileBytes];
  alignas(1024) uint8_t v[2][kTileBytes];
  alignas(1024) uint8_t p[2][kPTileBytes];
  // epilogue staging: each softmax warp turns its 32 rows x 32 fp32 columns
  // around here so that every store instruction writes whole 128-byte rows
  alignas(16) float stage[8][32][32];
  uint32_t tmem_base;
  int abort_flag;
  uint64_t k_full[2], v_full[2], q_full[2][2];  // q_full[buffer][producer warp]
  uint64_t s_full[2], p_full[2], o_full[2];
  uint64_t mma_drain;  // one final commit: every MMA of the CTA has completed
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

__global__ void __launch_bounds__(kNsaThreads, 1)
    nsa_main_kernel(const __grid_constant__ CUtensorMap mapQ,
                    const __grid_constant__ CUtensorMap mapK,
                    const __grid_constant__ CUtensorMap mapV, const NsaParams p) {
  extern __shared__ uint8_t smem_raw[];
  NsaSmem& sm = *reinterpret_cast<NsaSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_all = min(__ldg(p.unit_prefix + p.Hkv * p.nseq * p.nbps), p.max_units);
  // this CTA's units: the contiguous range [u_lo, u_lo + n_mine)
  const int u_lo = static_cast<int>(static_cast<int64_t>(n_all) * blockIdx.x / gridDim.x);
  const int n_mine = static_cast<int>(static_cast<int64_t>(n_all) * (blockIdx.x + 1) / gridDim.x) - u_lo;
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.k_full[b], 1);
      mbar_init(&sm.v_full[b], 1);
      mbar_init(&sm.q_full[b][0], 1);  // each producer warp arms its own half
      mbar_init(&sm.q_full[b][1], 1);
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.p_full[b], 128);
      mbar_init(&sm.o_full[b], 1);
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
      cur = nsa_unit(p, u_lo);
      load_codes(cur, c0, c1);
      first = __ldg(p.list + cur.e0);
    }
    if (n_mine > 1) nxt = nsa_unit(p, u_lo + 1);
    bool ok = true;
    // last unit whose Q (and, for warp 0, K) / V copies this warp issued into
    // each buffer, for the drain before exit; a buffer is refilled only after
    // its previous contents were consumed, so only that last phase can pend
    int qk_last[2] = {-1, -1}, v_last[2] = {-1, -1};
    // Buffers of unit n (index n & 1) were last used by unit n - 2: Q and K
    // are free once QK(n - 2) has completed (s_full), V once PV(n - 2) has
    // (o_full), which comes after QK(n - 1) and so after Q(n - 1) landed.
    for (int n = 0; n < n_mine && ok; ++n) {
      const int b = n & 1;
      const uint32_t pw = ((n >> 1) & 1) ^ 1u;
      if (n + 1 < n_mine) {
        load_codes(nxt, n0, n1);
        first_n = __ldg(p.list + nxt.e0);
      }
      NsaUnit nn{};
      if (n + 2 < n_mine) nn = nsa_unit(p, u_lo + n + 2);
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
      cur = nxt; nxt = nn;
      c0 = n0; c1 = n1; first = first_n;
    }
    // no copy may still be landing in shared memory when the CTA exits
    __syncwarp();
    if (lane == 0) {
      for (int b = 0; b < 2; ++b) {
        if (qk_last[b] >= 0) {
          const uint32_t ph = (qk_last[b] >> 1) & 1;
          mbar_wait_short(&sm.q_full[b][half], ph);
          if (half == 0) mbar_wait_short(&sm.k_full[b], ph);
        }
        if (half == 0 && v_last[b] >= 0) mbar_wait_short(&sm.v_full[b], (v_last[b] >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ===================== MMA issuer =====================
    // Order: QK(0), QK(1), PV(0), QK(2), PV(1), ... so that the softmax of
    // one unit overlaps the QK of the next.
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16(128, 64, 0);
      const uint32_t idesc_pv = idesc_bf16(128, 128, 1);
      const uint64_t qdesc0 = sdesc_sw128(smem_u32(sm.q[0]), 16, 1024);
      const uint64_t kdesc0 = sdesc_sw128(smem_u32(sm.k[0]), 16, 1024);
      const uint64_t vdesc0 = sdesc_sw128(smem_u32(sm.v[0]), 8192, 1024);
      const uint64_t pdesc0 = sdesc_sw128(smem_u32(sm.p[0]), 16, 1024);
      bool ok = true;
      auto issue_qk = [&](int n) -> bool {
        const int b = n & 1;
        const uint32_t ph = (n >> 1) & 1;
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
          umma_ss(tmem + b * 256, qd + off_q, kd + off_k, idesc_qk, kk ? 1u : 0u);
        }
        umma_commit(&sm.s_full[b]);
        return true;
      };
      auto issue_pv = [&](int n) -> bool {
        const int b = n & 1;
        const uint32_t ph = (n >> 1) & 1;
        if (!mbar_wait(&sm.p_full[b], ph, wctx) || !mbar_wait(&sm.v_full[b], ph, wctx))
          return false;
        tc_fence_after();
        const uint64_t pd = pdesc0 + (b * kPTileBytes >> 4);
        const uint64_t vd = vdesc0 + (b * kTileBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ss(tmem + b * 256 + 128, pd + (kk * 32 >> 4), vd + (kk * 2048 >> 4), idesc_pv,
                  kk ? 1u : 0u);
        umma_commit(&sm.o_full[b]);
        return true;
      };
      if (n_mine > 0) ok = issue_qk(0);
      for (int n = 0; n < n_mine && ok; ++n) {
        if (n + 1 < n_mine) ok = issue_qk(n + 1);
        if (ok) ok = issue_pv(n);
      }
      // drain every tcgen05 op before TMEM is released: a commit to a barrier
      // nothing else uses completes its single phase only then
      umma_commit(&sm.mma_drain);
      mbar_wait_short(&sm.mma_drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ===================== softmax / epilogue warpgroups (ping-pong) =====================
    const int b = (warp - 4) >> 2;
    const int r = tid - 128 - 128 * b;
    const int quarter = warp & 3;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + b * 256;
    const float NEG = -INFINITY;
    bool ok = true;
    // this warpgroup's units n = b, b + 2, ...: row codes one unit ahead
    NsaUnit un_next{};
    int code_next = -1;
    if (b < n_mine) {
      un_next = nsa_unit(p, u_lo + b);
      code_next = r / p.G < un_next.ne ? __ldg(p.list + un_next.e0 + r / p.G) : -1;
    }
    for (int n = b; n < n_mine && ok; n += 2) {
      const uint32_t ph = (n >> 1) & 1;
      const NsaUnit un = un_next;
      const int code = code_next;
      if (n + 2 < n_mine) {
        un_next = nsa_unit(p, u_lo + n + 2);
        code_next = r / p.G < un_next.ne ? __ldg(p.list + un_next.e0 + r / p.G) : -1;
      }
      const bool valid = code >= 0;
      int t = 0, slot = 0, tl = 0, L = 0;
      if (valid) {
        t = code / p.topk;
        slot = code % p.topk;
        tl = t - un.base;
        L = un.end - un.base;
      }
      // tcgen05.ld is warp-collective: the warp agrees before leaving
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[b], ph, wctx))) { ok = false; break; }
      tc_fence_after();
      float s[64];
      tmem_ld32(lane_addr, s);
      tmem_ld32(lane_addr + 32, s + 32);
      float mx = NEG;
      const int kb = un.key0 - un.base;  // first key of the block, sequence-local
      if (__all_sync(0xffffffffu, valid && kb + 63 < L && (!p.causal || kb + 63 <= tl))) {
        // every key of the block is visible to every row of this warp
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          s[c] *= p.scale_log2;
          mx = fmaxf(mx, s[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int key = kb + c;
          const bool vis = valid && key < L && (!p.causal || key <= tl);
          s[c] = vis ? s[c] * p.scale_log2 : NEG;
          mx = fmaxf(mx, s[c]);
        }
      }
      const float mu = (mx == NEG) ? 0.f : mx;
      float l = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float p0 = ex2_approx(s[c] - mu), p1 = ex2_approx(s[c + 1] - mu);
        l += p0 + p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      const uint32_t prow = smem_u32(sm.p[b]);
#pragma unroll
      for (int cc = 0; cc < 8; ++cc)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + sw128_off(r, cc)),
                     "r"(pk[cc * 4]), "r"(pk[cc * 4 + 1]), "r"(pk[cc * 4 + 2]), "r"(pk[cc * 4 + 3])
                     : "memory");
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.p_full[b]);
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.o_full[b], ph, wctx))) { ok = false; break; }
      tc_fence_after();
      const int h = un.g * p.G + r % p.G;
      const int64_t prow_idx = (static_cast<int64_t>(t) * p.Hq + h) * p.topk + slot;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      // 32 columns at a time: each lane parks its row in the warp's staging
      // tile (16-byte pieces rotated by row to spread the banks), then lane
      // group i / 8 of each store writes the 128 contiguous bytes of one row
      float (*stg)[32] = sm.stage[warp - 4];
      float ob[32];
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(lane_addr + 128 + c * 32, ob);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<float4*>(&stg[lane][4 * (i ^ (lane & 7))]) =
              make_float4(ob[4 * i] * inv, ob[4 * i + 1] * inv, ob[4 * i + 2] * inv,
                          ob[4 * i + 3] * inv);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + (lane >> 3), piece = lane & 7;
          const long long dst_row = __shfl_sync(0xffffffffu, valid ? prow_idx : -1ll, rr);
          const float4 x = *reinterpret_cast<const float4*>(&stg[rr][4 * (piece ^ (rr & 7))]);
          if (dst_row >= 0)
            *reinterpret_cast<float4*>(p.part_o + dst_row * 128 + c * 32 + 4 * piece) = x;
        }
        __syncwarp();
      }
      if (valid) p.part_lse[prow_idx] = l > 0.f ? (mu + lg2_approx(l)) * 0.69314718055994531f : NEG;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// One warp per (token, query head): LSE combine of its valid slots.
__global__ void nsa_combine_kernel(NsaParams p) {
  const int64_t wg = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wg >= static_cast<int64_t>(p.total) * p.Hq) return;
  const int t = static_cast<int>(wg / p.Hq), h = static_cast<int>(wg % p.Hq);
  const int g = h / p.G;
  const int s = nsa_seq_of(p.cu, p.nseq, t);
  const int L = p.cu[s + 1] - p.cu[s];
  const int nb = (L + 63) / 64;
  const int* sl = p.sel + (static_cast<int64_t>(t) * p.Hkv + g) * p.topk;
  const int64_t row = (static_cast<int64_t>(t) * p.Hq + h) * p.topk;
  if (p.topk <= 32) {
    // lane k holds slot k's lse; the partial rows of the valid slots are
    // then fetched eight at a time, all loads of a batch in flight together
    float lv = -INFINITY;
    if (lane < p.topk) {
      const int j = __ldg(sl + lane);
      if (j >= 0 && j < nb) lv = p.part_lse[row + lane];
    }
    const float M = warp_max_f32(lv);
    const float Mn = (M == -INFINITY) ? 0.f : M;
    const float w = (lv == -INFINITY) ? 0.f : __expf(lv - Mn);
    float W = w;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) W += __shfl_xor_sync(0xffffffffu, W, off);
    unsigned vm = __ballot_sync(0xffffffffu, w > 0.f);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    while (vm) {
      int ks[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        ks[u] = vm ? __ffs(vm) - 1 : -1;
        vm &= vm - 1u;
      }
      float4 xs[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (ks[u] >= 0)
          xs[u] = *reinterpret_cast<const float4*>(p.part_o + (row + ks[u]) * 128 + lane * 4);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (ks[u] < 0) continue;
        const float wu = __shfl_sync(0xffffffffu, w, ks[u]);
        acc.x += wu * xs[u].x; acc.y += wu * xs[u].y; acc.z += wu * xs[u].z; acc.w += wu * xs[u].w;
      }
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    __nv_bfloat16* op = p.o + static_cast<int64_t>(t) * p.oss + h * p.osh + lane * 4;
    reinterpret_cast<__nv_bfloat162*>(op)[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    reinterpret_cast<__nv_bfloat162*>(op)[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    if (lane == 0) p.lse[static_cast<int64_t>(h) * p.total + t] = W > 0.f ? Mn + __logf(W) : -INFINITY;
    return;
  }
  float M = -INFINITY;
  for (int k = 0; k < p.topk; ++k) {
    const int j = __ldg(sl + k);
    if (j < 0 || j >= nb) continue;
    M = fmaxf(M, p.part_lse[row + k]);
  }
  const float Mn = (M == -INFINITY) ? 0.f : M;
  float W = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k = 0; k < p.topk; ++k) {
    const int j = __ldg(sl + k);
    if (j < 0 || j >= nb) continue;
    const float lv = p.part_lse[row + k];
    if (lv == -INFINITY) continue;
    const float w = __expf(lv - Mn);
    W += w;
    const float4 x = *reinterpret_cast<const float4*>(p.part_o + (row + k) * 128 + lane * 4);
    acc.x += w * x.x; acc.y += w * x.y; acc.z += w * x.z; acc.w += w * x.w;
  }
  const float inv = W > 0.f ? 1.f / W : 0.f;
  __nv_bfloat16* op = p.o + static_cast<int64_t>(t) * p.oss + h * p.osh + lane * 4;
  reinterpret_cast<__nv_bfloat162*>(op)[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  reinterpret_cast<__nv_bfloat162*>(op)[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  if (lane == 0) p.lse[static_cast<int64_t>(h) * p.total + t] = W > 0.f ? Mn + __logf(W) : -INFINITY;
}

}  // namespace sbfa
