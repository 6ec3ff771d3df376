// Vertical/slash index conversion (Sglang Sparse Flash Attention,
// convert_vertical_slash_indexes, and the per-head-count variant
// convert_vertical_slash_indexes_mergehead): one CTA per (batch, head,
// q-block).  With per-head counts, head h uses only the first v_cnt[h]
// vertical and s_cnt[h] slash entries of its rows.
//
// Slash offset s is the diagonal key = row + d - s (d = kv_len - q_len); over
// the q-block's rows [m0, m1) it covers keys [m0+d-s, m1-1+d-s].  Each such
// range is at most 64 keys long, so it touches at most two 64-key blocks; the
// CTA marks them in a shared bitmap, then compacts the bitmap into the
// ascending block_offset list.  Vertical columns that are visible and not
// inside a listed block are compacted, in order, into column_index.
#pragma once

#include "sbfa_ptx.cuh"

namespace sbfa {

constexpr int kCvThreads = 128;
constexpr int kCvMaxWords = 8192 / 32;  // kv_len <= 524288 (64-key blocks)

// Exclusive block-wide prefix sum over kCvThreads values; returns the total.
__device__ __forceinline__ int cv_block_scan(int v, int* warp_tot, int& excl) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  int base = 0, total = 0;
  for (int w = 0; w < kCvThreads / 32; ++w) {
    if (w < warp) base += warp_tot[w];
    total += warp_tot[w];
  }
  excl = base + x - v;
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kCvThreads)
    convert_vs_kernel(const int* __restrict__ q_seqlens, const int* __restrict__ kv_seqlens,
                      const int* __restrict__ vertical, int nnz_v, const int* __restrict__ slash,
                      int nnz_s, const int* __restrict__ v_cnt, const int* __restrict__ s_cnt,
                      int H, int nqb, int block_M, int block_N, int causal,
                      int* __restrict__ block_count, int* __restrict__ block_offset,
                      int* __restrict__ column_count, int* __restrict__ column_index,
                      int* status) {
  __shared__ uint32_t bm[kCvMaxWords];
  __shared__ int warp_tot[kCvThreads / 32];
  const int i = blockIdx.x % nqb;
  const int bh = blockIdx.x / nqb;
  const int b = bh / H;
  const int tid = threadIdx.x;
  const int q_len = q_seqlens[b], kv_len = kv_seqlens[b];
  // entries of this head's rows in use (the row strides stay nnz_v / nnz_s)
  const int h = bh % H;
  const int nv = v_cnt ? min(max(v_cnt[h], 0), nnz_v) : nnz_v;
  const int ns = s_cnt ? min(max(s_cnt[h], 0), nnz_s) : nnz_s;
  const int d = kv_len - q_len;
  const int64_t row = static_cast<int64_t>(bh) * nqb + i;
  const int m0 = i * block_M;
  if (m0 >= q_len) {
    if (tid == 0) {
      block_count[row] = 0;
      column_count[row] = 0;
    }
    return;
  }
  const int m1 = min(m0 + block_M, q_len);
  const int nkb = (kv_len + block_N - 1) / block_N;
  const int nwords = (nkb + 31) >> 5;
  for (int w = tid; w < nwords; w += kCvThreads) bm[w] = 0u;
  __syncthreads();
  const int* sl = slash + static_cast<int64_t>(bh) * nnz_s;
  for (int e = tid; e < ns; e += kCvThreads) {
    const int s = sl[e];
    if (s < 0) { report(status, kDevBadIndex); continue; }
    const int lo = max(m0 + d - s, 0);
    const int hi = min(m1 - 1 + d - s, kv_len - 1);
    if (hi < lo) continue;
    for (int j = lo / block_N; j <= hi / block_N; ++j) atomicOr(&bm[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  // ---- compact the bitmap into ascending block offsets
  int* bo = block_offset + row * nnz_s;
  int written = 0;
  for (int w0 = 0; w0 < nwords; w0 += kCvThreads) {
    const int w = w0 + tid;
    const uint32_t bits = w < nwords ? bm[w] : 0u;
    int excl;
    const int tot = cv_block_scan(__popc(bits), warp_tot, excl);
    int pos = written + excl;
    uint32_t x = bits;
    while (x) {
      const int bit = __ffs(x) - 1;
      x &= x - 1u;
      if (pos < nnz_s) bo[pos] = (w * 32 + bit) * block_N;
      ++pos;
    }
    written += tot;
  }
  if (tid == 0) {
    if (written > nnz_s) report(status, kDevOverflow);
    block_count[row] = min(written, nnz_s);
  }
  // ---- vertical columns not covered by a listed block
  const int* vt = vertical + static_cast<int64_t>(bh) * nnz_v;
  int* ci = column_index + row * nnz_v;
  const int vis_end = causal ? min(kv_len, m1 + d) : kv_len;  // columns < vis_end
  int ncol = 0;
  for (int e0 = 0; e0 < nv; e0 += kCvThreads) {
    const int e = e0 + tid;
    int c = -1;
    bool keep = false;
    if (e < nv) {
      c = vt[e];
      keep = c >= 0 && c < vis_end && !((bm[(c / block_N) >> 5] >> ((c / block_N) & 31)) & 1u);
      if (c < 0) report(status, kDevBadIndex);
    }
    int excl;
    const int tot = cv_block_scan(keep ? 1 : 0, warp_tot, excl);
    if (keep) ci[ncol + excl] = c;
    ncol += tot;
  }
  if (tid == 0) column_count[row] = ncol;
}

// ----------------------------------------------------------------------------
// BSFA threshold calibration (Block Sparse Flash Attention, Figure 2a): for
// every (batch, head, q-block i) T = the k-th largest of the off-diagonal
// block maxima {s_max[i][j] : j < i}, counted with multiplicity, or -inf when
// fewer than k candidates exist.  One CTA per row: exact radix selection over
// the candidates' order-preserving 32-bit keys, eight bits per pass.
// ----------------------------------------------------------------------------
constexpr int kCalThreads = 256;

__global__ void __launch_bounds__(kCalThreads) calibrate_kernel(const float* __restrict__ smax,
                                                                int n_qb, int k_top,
                                                                float* __restrict__ T) {
  __shared__ int hist[256];
  __shared__ uint32_t sel_prefix;
  __shared__ int sel_rank;
  const int64_t row = blockIdx.x;             // (b * Hq + h) * n_qb + i
  const int i = static_cast<int>(row % n_qb);
  const float* cand = smax + row * n_qb;      // s_max[b][h][i][0..n_qb)
  if (i < k_top) {                            // fewer than k candidates j < i
    if (threadIdx.x == 0) T[row] = -INFINITY;
    return;
  }
  uint32_t prefix = 0, mask = 0;
  int rank = k_top;                           // 1-based rank from the top
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += kCalThreads) hist[b] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < i; j += kCalThreads) {
      const uint32_t u = f32_order_key(cand[j]);
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int cum = 0, bucket = 0;
      for (int b = 255; b >= 0; --b) {
        if (cum + hist[b] >= rank) { bucket = b; break; }
        cum += hist[b];
      }
      sel_prefix = prefix | (static_cast<uint32_t>(bucket) << shift);
      sel_rank = rank - cum;
    }
    __syncthreads();
    prefix = sel_prefix;
    rank = sel_rank;
    mask |= 255u << shift;
    __syncthreads();
  }
  if (threadIdx.x == 0) T[row] = f32_from_order_key(prefix);
}

}  // namespace sbfa
