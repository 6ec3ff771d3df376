/*
 * sbfa.h -- C ABI of the block-sparse FlashAttention forward for NVIDIA B200
 * (sm_100a).
 *
 * Every entry point is asynchronous on the given CUDA stream, returns an
 * sbfa_status, allocates nothing and keeps no device state between calls.
 * The caller owns every input, output and workspace buffer (device memory
 * unless stated otherwise).  Argument errors are detected on the host and
 * returned before any launch; sbfa_last_error() then gives a message.
 * Problems only the device can see (a table entry outside the key range, a
 * wait that timed out) never trap: the kernel skips the offending work and
 * ORs an SBFA_DEV_* bit into the optional int32 device status word, which
 * the caller zeroes and reads back (see sbfa_check_status).
 *
 * Common conventions
 *   - Tensors use the (batch, seq, head, dim) layout of the
 *     Incremental_FlashAttention README (Usage 1): q (B, Sq, Hq, D),
 *     k and v (B, Sk, Hkv, D), o like q.  An sbfa_t4 gives the base pointer
 *     and element strides of the first three dims; the last dim must be
 *     contiguous.  Strides must be multiples of 8 elements and base pointers
 *     16-byte aligned (TMA rules).  q, k, v and o are bf16.
 *   - lse is fp32 (B, Hq, Sq), contiguous, natural log of the softmax
 *     denominator.  A row that sees no key gets o = 0, lse = -inf (README,
 *     Usage 1: an empty table is a neutral partial).
 *   - D must be 128.  Hq must be a multiple of Hkv; query head h reads kv
 *     head h / (Hq / Hkv).
 *   - scale <= 0 selects 1/sqrt(D).
 *   - causal masks keys with index > row + (Sk - Sq) (bottom-right
 *     alignment).
 */
#ifndef SBFA_H_
#define SBFA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sbfa_stream_t; /* identical to cudaStream_t */

typedef enum {
  SBFA_OK = 0,
  SBFA_ERR_INVALID_ARG = 1, /* bad pointer, shape, stride or alignment */
  SBFA_ERR_UNSUPPORTED = 2, /* valid request this build does not serve (D != 128, ...) */
  SBFA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  SBFA_ERR_DEVICE = 4,      /* the device status word reported a problem */
  SBFA_ERR_TIMEOUT = 5      /* a kernel wait hit its time limit */
} sbfa_status;

/* Bits of the device status word. */
#define SBFA_DEV_BAD_INDEX 0x1 /* table / index entry outside the key range: entry skipped */
#define SBFA_DEV_TIMEOUT 0x2   /* a bounded barrier wait gave up: the CTA stopped early */
#define SBFA_DEV_OVERFLOW 0x4  /* a per-row list exceeded the kernel's capacity: truncated */

/* A (B, S, H, D) view: base pointer and element strides of B, S and H. */
typedef struct {
  void* ptr;
  int64_t sb, ss, sh;
} sbfa_t4;

typedef struct {
  int32_t B, Sq, Sk, Hq, Hkv, D;
  float scale;    /* <= 0: 1/sqrt(D) */
  int32_t causal; /* 0 or 1 */
} sbfa_shape;

/*
 * Sparse block table (Incremental_FlashAttention README, Usage 1,
 * generalised per (batch, kv-head, q-block)).  Row r of query head h in
 * batch b uses idx[b*sb + (h/G)*sh + (r/q_block)*sqb + n], n < nmax.  Each
 * entry j >= 0 names the keys [j*kv_block, (j+1)*kv_block) clipped to Sk;
 * entries < 0 are padding; order does not matter; a row is a set of blocks:
 * sbfa_fwd counts a block listed more than once once, whichever kernel
 * serves the call (see sbfa_speculative_sparse for its own rule).  An entry
 * >= ceil(Sk / kv_block) is skipped and sets SBFA_DEV_BAD_INDEX.
 * sb = sh = sqb = 0 broadcasts one 1-D table (the README's form).
 */
typedef struct {
  const int32_t* idx;
  int64_t sb, sh, sqb;
  int32_t nmax, q_block, kv_block;
} sbfa_table;

/*
 * sbfa_fwd -- block-table attention forward.
 * Source: Incremental_FlashAttention README, "What's in this fork" (sparse
 * block-table forward) and Usage 1.  Each query row attends only to the keys
 * of the blocks its table row lists (with the causal mask if shape->causal).
 * Constraints: kv_block in {16, 32, 64, 128, 256} (README, "What's in this
 * fork": block sizes at hdim 128); Sk <= 524288, and Sk <= 8192 * kv_block
 * for 16- and 32-key blocks; q_block a multiple of 64 (or >= Sq).  Decode
 * shapes (Sq * Hq/Hkv <= 16 and one q-block) that are not causal, or have
 * Sq = 1, run on the split-KV decode kernel; the rest on the tiled kernel.
 * Outputs: o (bf16, like q), lse (fp32 [B, Hq, Sq]).
 * status: optional device int32, SBFA_DEV_* bits are ORed in.
 */
sbfa_status sbfa_fwd(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v,
                     const sbfa_table* table, sbfa_t4 o, float* lse, int32_t* status,
                     sbfa_stream_t stream);

/*
 * sbfa_fwd_dense -- dense attention over all Sk keys (causal if asked).
 * Source: the README's pass over the speculative K/V subset (Usage 2).
 * Same layouts and limits as sbfa_fwd.
 */
sbfa_status sbfa_fwd_dense(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v,
                           sbfa_t4 o, float* lse, int32_t* status, sbfa_stream_t stream);

/*
 * sbfa_fwd_window -- causal sliding-window attention.
 * Source: Flash-Sparse-Attention, Quickstart (window_size = 512: NSA's
 * sliding-window branch, here on its own, returning (o, lse)).  Row r
 * attends the keys r + (Sk - Sq) - window < key <= r + (Sk - Sq)
 * (bottom-right causal; shape->causal is ignored).  window >= 1.  Same
 * layouts and limits as sbfa_fwd_dense; runs on the tiled kernel, whose
 * schedule visits only the key tiles inside each q-block's window.
 */
sbfa_status sbfa_fwd_window(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v,
                            int32_t window, sbfa_t4 o, float* lse, int32_t* status,
                            sbfa_stream_t stream);

/*
 * sbfa_fwd_partials -- one (o, lse) per table entry.
 * Source: README, Usage 3 (per-block partials for a caller-side combine).
 * o_parts: fp32 [nmax, B, Sq, Hq, D] contiguous; lse_parts: fp32
 * [nmax, B, Hq, Sq] contiguous.  Partial n attends the keys of entry n of
 * each row's table (a padding entry gives o = 0, lse = -inf).  The combine
 * of all nmax partials equals sbfa_fwd when a row lists each block once; a
 * repeated entry yields a repeated partial, which the combine would count
 * twice.
 */
sbfa_status sbfa_fwd_partials(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v,
                              const sbfa_table* table, float* o_parts, float* lse_parts,
                              int32_t* status, sbfa_stream_t stream);

/*
 * sbfa_combine -- exact merge of partial results over disjoint key sets.
 * Source: README, "What's in this fork" (FA(A u B) == Combine(FA(A),
 * FA(B))) and Usage 2.  With M = max_p lse_p and w_p = exp(lse_p - M):
 * lse = M + ln sum_p w_p, o = sum_p w_p o_p / sum_p w_p; all partials empty
 * gives (0, -inf).
 * o_parts: fp32 [n_parts, B, Sq, Hq, D] contiguous, lse_parts: fp32
 * [n_parts, B, Hq, Sq] contiguous.  o: bf16 view (D contiguous), lse: fp32
 * [B, Hq, Sq].  D must be 128.
 */
sbfa_status sbfa_combine(int32_t n_parts, int32_t B, int32_t Sq, int32_t Hq, int32_t D,
                         const float* o_parts, const float* lse_parts, sbfa_t4 o, float* lse,
                         sbfa_stream_t stream);

/*
 * sbfa_speculative_sparse -- fused two-pass speculative + sparse decode.
 * Source: README, Usage 2.  One launch computes, per query row, attention
 * over (a) all S_spec keys of (k_spec, v_spec), causal if causal_spec, and
 * (b) the blocks of (k, v) listed in `missed` (no mask), merged by the LSE
 * combine inside the kernel.  The result equals attention over the union.
 * shape->Sk is the length of k/v; shape->causal is ignored.  A paged KV
 * cache is this call with k/v views of one page pool shared by all
 * sequences (batch stride 0), kv_block = the page size, and each table row
 * listing the pool pages of its missed blocks (FlagAttention's paged
 * attention; pages may be shared between sequences).
 * `missed` lists distinct blocks (README, Usage 2: the blocks the
 * speculative pass missed); the fused kernel does not look for repeats, so
 * a block listed twice would be counted twice.
 * Limits: Sq * (Hq/Hkv) <= 16; missed->q_block >= Sq; missed->kv_block in
 * {16, 32, 64, 128, 256}; B*Hkv <= 4096; missed->nmax <= 1024.
 * ws/ws_bytes: device workspace of at least sbfa_decode_workspace_size()
 * bytes, zero-filled before its first use (the kernel leaves its counters at
 * zero when it completes).  Calls sharing one workspace must not overlap.
 */
sbfa_status sbfa_speculative_sparse(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k_spec,
                                    sbfa_t4 v_spec, int32_t S_spec, int32_t causal_spec,
                                    sbfa_t4 k, sbfa_t4 v, const sbfa_table* missed,
                                    void* ws, size_t ws_bytes, sbfa_t4 o, float* lse,
                                    int32_t* status, sbfa_stream_t stream);

/*
 * sbfa_speculative_sparse_noalloc -- sbfa_speculative_sparse without a
 * caller workspace.  The pages have no counterpart: this entry point exists
 * for callers that cannot call cudaMalloc -- for example code that runs
 * inside a caching allocator's own callback (allocating there re-enters the
 * allocator), code whose device memory is a fixed pool owned by another
 * framework, or latency-critical paths that must not risk the implicit
 * device synchronisation a cudaMalloc can cause.
 * Instead of `ws` it uses a fixed scratch array compiled into the library
 * (about 2.6 MB per GPU that loads the library, held until the process
 * exits): per-pair tickets and per-CTA fp32 partials for at most 4096
 * (batch x kv-head) pairs.  Larger B*Hkv is rejected with
 * SBFA_ERR_UNSUPPORTED.  Allocates nothing: each call zeroes the tickets it
 * uses with cudaMemsetAsync on `stream`, then launches the same split-KV
 * kernel.  The first call on a device looks up the scratch array's device
 * address (cudaGetSymbolAddress) with that device current; make that first
 * call before any stream capture.  All calls share the one array, which keeps
 * the last call's contents: calls that overlap on the GPU (other streams,
 * other host threads) race and give wrong results.
 * Arguments, limits and results are otherwise those of
 * sbfa_speculative_sparse.
 */
sbfa_status sbfa_speculative_sparse_noalloc(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k_spec,
                                            sbfa_t4 v_spec, int32_t S_spec, int32_t causal_spec,
                                            sbfa_t4 k, sbfa_t4 v, const sbfa_table* missed,
                                            sbfa_t4 o, float* lse, int32_t* status,
                                            sbfa_stream_t stream);

/* Workspace bytes the split-KV decode kernel needs on the current device. */
size_t sbfa_decode_workspace_size(int32_t B, int32_t Hkv, int32_t Sq, int32_t Hq);

/*
 * sbfa_fwd_gated -- BSFA gated causal prefill.
 * Source: Block Sparse Flash Attention, Abstract and Figure 2.  For head h
 * and q-block i (64 rows) the kernel computes S = scale*Q_i K_j^T for every
 * causal key block j <= i (64 keys), its exact block max s_max(h,i,j), and
 * keeps the block iff j == i (the diagonal always runs) or
 * s_max >= T[h*nQB + i].  Skipped blocks load no V_j and run no P V_j.
 * Requires Sq == Sk, causal, block == 64.  T: fp32 [Hq, nQB], nQB =
 * ceil(Sq/64); -inf keeps every block.
 * smax_out (nullable): fp32 [B, Hq, nQB, nQB], written for j <= i.
 * keep_out (nullable): uint8 [B, Hq, nQB, nQB], 1/0, written for j <= i.
 */
sbfa_status sbfa_fwd_gated(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v,
                           const float* T, int32_t block, sbfa_t4 o, float* lse,
                           float* smax_out, uint8_t* keep_out, int32_t* status,
                           sbfa_stream_t stream);

/*
 * sbfa_convert_vertical_slash -- raw vertical/slash indices to block lists.
 * Source: Sglang Sparse Flash Attention, Description and I/O contract
 * (convert_vertical_slash_indexes).  For batch b, head h and q-block i with
 * rows [m0, m1), m1 = min(m0 + block_M, q_len), d = kv_len - q_len:
 *   - slash offset s covers keys [m0+d-s, m1-1+d-s] clipped to [0, kv_len);
 *     block_offset[b,h,i,:] lists, ascending, the offsets j*block_N of every
 *     key block meeting the union of these ranges; block_count their number;
 *   - column_index[b,h,i,:] lists, ascending, the vertical columns
 *     c < kv_len (and c <= m1-1+d if causal) that lie in no listed block;
 *     column_count their number.
 * Entries past a count are left unwritten.
 * q_seqlens, kv_seqlens: int32 [B] (device).  vertical: int32 [B, H, nnz_v],
 * slash: int32 [B, H, nnz_s], each row ascending and distinct, slash >= 0.
 * Outputs (int32): block_count, column_count [B, H, nQB]; block_offset
 * [B, H, nQB, nnz_s]; column_index [B, H, nQB, nnz_v]; nQB =
 * ceil(context_size / block_M).  Requires block_M == block_N == 64.
 */
sbfa_status sbfa_convert_vertical_slash(const int32_t* q_seqlens, const int32_t* kv_seqlens,
                                        const int32_t* vertical, int32_t nnz_v,
                                        const int32_t* slash, int32_t nnz_s, int32_t B,
                                        int32_t H, int32_t context_size, int32_t block_M,
                                        int32_t block_N, int32_t causal, int32_t* block_count,
                                        int32_t* block_offset, int32_t* column_count,
                                        int32_t* column_index, int32_t* status,
                                        sbfa_stream_t stream);

/*
 * sbfa_fwd_vertical_slash -- sparse attention over converted block lists.
 * Source: Sglang Sparse Flash Attention (sparse_attn_func).  Row r of
 * q-block i of head h attends the keys of blocks [off, off + block_N) for
 * the first block_count entries of block_offset, plus the first
 * column_count keys of column_index, with the causal mask if asked.
 * Index arrays as produced by sbfa_convert_vertical_slash (per query head;
 * with GQA, query head h reads kv head h / (Hq/Hkv)).  Requires block_M ==
 * block_N == 64.
 */
sbfa_status sbfa_fwd_vertical_slash(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v,
                                    const int32_t* block_count, const int32_t* block_offset,
                                    int32_t nnz_s, const int32_t* column_count,
                                    const int32_t* column_index, int32_t nnz_v,
                                    int32_t block_M, int32_t block_N, sbfa_t4 o, float* lse,
                                    int32_t* status, sbfa_stream_t stream);

/*
 * sbfa_convert_vertical_slash_mergehead -- sbfa_convert_vertical_slash with
 * a per-head number of entries.
 * Source: Sglang Sparse Flash Attention, Description and Signature
 * (convert_vertical_slash_indexes_mergehead: per-head variable sparsity
 * counts vertical_indices_count / slash_indices_count).  Reading taken: the
 * counts are int32 [H] (device); head h uses the first vertical_count[h] of
 * its nnz_v vertical entries and the first slash_count[h] of its nnz_s slash
 * entries (counts are clamped to [0, nnz]); rows are laid out with strides
 * nnz_v / nnz_s as in sbfa_convert_vertical_slash, whose definition, outputs
 * and limits apply otherwise.
 */
sbfa_status sbfa_convert_vertical_slash_mergehead(
    const int32_t* q_seqlens, const int32_t* kv_seqlens, const int32_t* vertical, int32_t nnz_v,
    const int32_t* slash, int32_t nnz_s, const int32_t* vertical_count,
    const int32_t* slash_count, int32_t B, int32_t H, int32_t context_size, int32_t block_M,
    int32_t block_N, int32_t causal, int32_t* block_count, int32_t* block_offset,
    int32_t* column_count, int32_t* column_index, int32_t* status, sbfa_stream_t stream);

/*
 * sbfa_fwd_varlen -- block-table attention over sequences packed by
 * cumulative lengths.
 * Sources: Flash-Sparse-Attention, Quickstart (cu_seqlens packing of a
 * variable-length batch); Incremental_FlashAttention README, Usage 1 (the
 * block table).  Sequence s owns query rows [cu_seqlens_q[s],
 * cu_seqlens_q[s+1]) of q and key rows [cu_seqlens_k[s], cu_seqlens_k[s+1])
 * of k and v.  Local query row r of sequence s and head h attends the keys
 * of the blocks listed in table row idx[s*sb + (h/G)*sh + (r/q_block)*sqb +
 * n]; entries are block indices local to the sequence (block j = local keys
 * [j*kv_block, (j+1)*kv_block) clipped to the sequence's key length), with
 * the sbfa_table rules (padding < 0, repeats count once, entries past the
 * sequence's last block are skipped and reported).  causal: the bottom-right
 * mask of each sequence (local key <= r + k_len - q_len).
 * cu_seqlens_q, cu_seqlens_k: int32 [nseq + 1], device, non-decreasing from
 * 0; total_q = cu_seqlens_q[nseq], total_k = cu_seqlens_k[nseq] (passed
 * from the host); max_seqlen_q / max_seqlen_k >= every sequence's length.
 * q: (1, total_q, Hq, 128) view (sb ignored); k, v: (1, total_k, Hkv, 128);
 * o like q; lse: fp32 [Hq, total_q].  kv_block in {64, 128, 256}; q_block a
 * multiple of 64 or >= max_seqlen_q.  No workspace.
 */
sbfa_status sbfa_fwd_varlen(const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            int32_t nseq, int32_t total_q, int32_t total_k,
                            int32_t max_seqlen_q, int32_t max_seqlen_k, int32_t Hq, int32_t Hkv,
                            int32_t D, float scale, int32_t causal, sbfa_t4 q, sbfa_t4 k,
                            sbfa_t4 v, const sbfa_table* table, sbfa_t4 o, float* lse,
                            int32_t* status, sbfa_stream_t stream);

/*
 * sbfa_fwd_window_varlen -- sbfa_fwd_window over sequences packed by
 * cumulative lengths (the window and the causal offset are per sequence).
 * Packing, layouts and lse as in sbfa_fwd_varlen.
 */
sbfa_status sbfa_fwd_window_varlen(const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                   int32_t nseq, int32_t total_q, int32_t total_k,
                                   int32_t max_seqlen_q, int32_t max_seqlen_k, int32_t Hq,
                                   int32_t Hkv, int32_t D, float scale, int32_t window, sbfa_t4 q,
                                   sbfa_t4 k, sbfa_t4 v, sbfa_t4 o, float* lse, int32_t* status,
                                   sbfa_stream_t stream);

/*
 * sbfa_fwd_vertical_slash_varlen -- sbfa_fwd_vertical_slash over sequences
 * packed by cumulative lengths.
 * Source: Sglang Sparse Flash Attention, Signature and I/O contract
 * (sparse_attn_varlen_func: cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
 * max_seqlen_k).  The index arrays are those sbfa_convert_vertical_slash
 * (or its mergehead form) writes with batch = sequence, q_seqlens /
 * kv_seqlens = the sequence lengths and context_size = max_seqlen_q:
 * [nseq, Hq, ceil(max_seqlen_q / 64), nnz]; offsets and columns are local to
 * the sequence.  Packing, layouts, the causal rule and lse as in
 * sbfa_fwd_varlen; block_M = block_N = 64.
 */
sbfa_status sbfa_fwd_vertical_slash_varlen(
    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int32_t nseq, int32_t total_q,
    int32_t total_k, int32_t max_seqlen_q, int32_t max_seqlen_k, int32_t Hq, int32_t Hkv,
    int32_t D, float scale, int32_t causal, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v,
    const int32_t* block_count, const int32_t* block_offset, int32_t nnz_s,
    const int32_t* column_count, const int32_t* column_index, int32_t nnz_v, int32_t block_M,
    int32_t block_N, sbfa_t4 o, float* lse, int32_t* status, sbfa_stream_t stream);

/*
 * sbfa_fwd_varlen_selected -- NSA selected attention over varlen sequences.
 * Source: Flash-Sparse-Attention (FSA), overview and Quickstart (top-k key
 * blocks of 64 per token, cu_seqlens packing, FSA's block-major loop order).
 * Token t (sequence-local index tl) of query head h attends the keys of its
 * selected blocks sel[t, h/G, :] (sequence-local block indices, -1 =
 * padding, distinct), clipped to its sequence and, if causal, to keys <= tl.
 * cu_seqlens: int32 [nseq + 1] (device), 0 = cu[0] < ... < cu[nseq] = total;
 * max_seqlen >= every sequence length.  q: (1, total, Hq, 128) view whose
 * token stride is Hq times its head stride (rows (token, head) are gathered
 * by TMA from that flattened view), k and v: (1, total, Hkv, 128) views (sb
 * ignored); o like q; lse: fp32 [Hq, total].  sel: int32 [total, Hkv, topk]
 * contiguous.  block must be 64; Hq/Hkv must divide 128.  ws: device
 * workspace of sbfa_varlen_selected_workspace_size() bytes (contents need
 * no initialisation).  Runs on `stream`: two memsets, the inverted-index
 * count / scan / fill, the unit table, and two block-major tcgen05 passes
 * over the (key block, query rows) units: the first takes each row's
 * largest score M, the second adds exp2(S - M) V and the sums of
 * exp2(S - M) into an fp32 accumulator per (token, head); a last kernel
 * writes o = accumulator / sum and lse.  The additions happen in no fixed
 * order: results can differ between runs within fp32 rounding.
 */
sbfa_status sbfa_fwd_varlen_selected(const int32_t* cu_seqlens, int32_t nseq, int32_t total,
                                     int32_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t D,
                                     float scale, int32_t causal, sbfa_t4 q, sbfa_t4 k,
                                     sbfa_t4 v, const int32_t* sel, int32_t topk, int32_t block,
                                     void* ws, size_t ws_bytes, sbfa_t4 o, float* lse,
                                     int32_t* status, sbfa_stream_t stream);

/* Workspace bytes for sbfa_fwd_varlen_selected (0 on bad sizes). */
size_t sbfa_varlen_selected_workspace_size(int32_t nseq, int32_t total, int32_t max_seqlen,
                                           int32_t Hq, int32_t Hkv, int32_t topk);

/*
 * sbfa_check_status -- synchronise `stream`, read the device status word
 * and map it to SBFA_OK / SBFA_ERR_DEVICE / SBFA_ERR_TIMEOUT.
 */
sbfa_status sbfa_check_status(const int32_t* status, sbfa_stream_t stream);

/*
 * sbfa_calibrate_thresholds -- BSFA gate thresholds from block maxima.
 * Source: Block Sparse Flash Attention, Figure 2a (calibration: the k-th
 * largest off-diagonal block maximum of each row of blocks).  smax: fp32
 * [B, Hq, n_qb, n_qb], as sbfa_fwd_gated writes to smax_out (only j < i is
 * read; run the calibration pass with T = -inf to see every block).  T out:
 * fp32 [B, Hq, n_qb] with T[b, h, i] = the k-th largest of
 * {smax[b, h, i, j] : j < i}, counted with multiplicity, and -inf when
 * i < k.  The selection is exact (no rounding).  One launch on `stream`.
 */
sbfa_status sbfa_calibrate_thresholds(const float* smax, int32_t B, int32_t Hq, int32_t n_qb,
                                      int32_t k_top, float* T, sbfa_stream_t stream);

/*
 * sbfa_set_wait_limit_ns -- time limit of the bounded waits inside the
 * pipelined kernels (sbfa_fwd's tiled path, sbfa_fwd_dense, sbfa_fwd_partials,
 * sbfa_fwd_gated, sbfa_fwd_vertical_slash, sbfa_fwd_varlen_selected)
 * launched after the call, for the whole process.  No wait in these kernels
 * is unbounded: one that runs past the limit stops its CTA early (every
 * copy and tensor-core operation the CTA issued is drained first, so the
 * context stays usable) and sets SBFA_DEV_TIMEOUT in the status word, and
 * sbfa_check_status then returns SBFA_ERR_TIMEOUT; the outputs of that
 * launch are incomplete.  0 restores the default of 2 s.  Returns the
 * previous limit.  The split-KV decode kernel and the index kernels have no
 * waits and ignore it.
 */
uint64_t sbfa_set_wait_limit_ns(uint64_t ns);

/* Message of the last error on this host thread ("" if none). */
const char* sbfa_last_error(void);

/* Library version string. */
const char* sbfa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SBFA_H_ */
