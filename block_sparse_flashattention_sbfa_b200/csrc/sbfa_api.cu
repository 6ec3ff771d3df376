// Host side of libsbfa: argument validation, TMA descriptor encoding and
// kernel launches behind the C ABI declared in include/sbfa.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "sbfa.h"
#include "kernel_convert.cuh"
#include "kernel_decode.cuh"
#include "kernel_prefill.cuh"
#include "kernel_nsa.cuh"

namespace {

thread_local std::string g_last_error;

sbfa_status fail(sbfa_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

sbfa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SBFA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define SBFA_CUDA(call)                                 \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

// ---------------------------------------------------------------------------
// TMA descriptor encoding through the driver entry point (no libcuda link).
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 4-D map over a (B, S, H, 128) bf16 view: dims {D, H, S, B}; box
// {64, 1, box_rows, 1}; 128-byte swizzle; out-of-range rows read as zero.
sbfa_status encode_bshd(CUtensorMap* map, const sbfa_t4& t, int B, int S, int H, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return fail(SBFA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const int64_t sh = H > 1 ? t.sh : 128;
  const int64_t ss = S > 1 ? t.ss : sh * H;
  const int64_t sb = B > 1 ? t.sb : ss * S;
  cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(S),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(sh * 2), static_cast<cuuint64_t>(ss * 2),
                           static_cast<cuuint64_t>(sb * 2)};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t.ptr, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SBFA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return SBFA_OK;
}

// 2-D map over `rows` rows of 128 bf16 (row stride `row_stride` elements),
// box 64 columns x 1 row: the source of tile::gather4 row gathers.
sbfa_status encode_rows2d(CUtensorMap* map, const void* ptr, int64_t rows, int64_t row_stride) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return fail(SBFA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride * 2)};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SBFA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return SBFA_OK;
}

struct DevInfo {
  int sms = 0;
};

sbfa_status dev_info(DevInfo* di) {
  static DevInfo cache[64];
  int dev = 0;
  SBFA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(SBFA_ERR_UNSUPPORTED, "device index %d", dev);
  if (cache[dev].sms == 0) {
    cudaDeviceProp prop;
    SBFA_CUDA(cudaGetDeviceProperties(&prop, dev));
    if (prop.major != 10)
      return fail(SBFA_ERR_UNSUPPORTED, "needs an sm_100 GPU (found sm_%d%d)", prop.major,
                  prop.minor);
    cache[dev].sms = prop.multiProcessorCount;
  }
  *di = cache[dev];
  return SBFA_OK;
}

// ---------------------------------------------------------------------------
// validation helpers
// ---------------------------------------------------------------------------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sbfa_status check_view(const sbfa_t4& t, const char* name, bool need_tma) {
  if (!t.ptr) return fail(SBFA_ERR_INVALID_ARG, "%s: null pointer", name);
  if (!aligned16(t.ptr)) return fail(SBFA_ERR_INVALID_ARG, "%s: base not 16-byte aligned", name);
  if (t.sb < 0 || t.ss < 0 || t.sh < 0)
    return fail(SBFA_ERR_INVALID_ARG, "%s: negative stride", name);
  if (need_tma && ((t.sb % 8) || (t.ss % 8) || (t.sh % 8)))
    return fail(SBFA_ERR_INVALID_ARG, "%s: strides must be multiples of 8 elements", name);
  return SBFA_OK;
}

sbfa_status check_shape(const sbfa_shape* s) {
  if (!s) return fail(SBFA_ERR_INVALID_ARG, "shape is null");
  if (s->B <= 0 || s->Sq <= 0 || s->Sk <= 0 || s->Hq <= 0 || s->Hkv <= 0)
    return fail(SBFA_ERR_INVALID_ARG, "non-positive size (B=%d Sq=%d Sk=%d Hq=%d Hkv=%d)", s->B,
                s->Sq, s->Sk, s->Hq, s->Hkv);
  if (s->D != 128) return fail(SBFA_ERR_UNSUPPORTED, "head dim %d (only 128)", s->D);
  if (s->Hq % s->Hkv) return fail(SBFA_ERR_INVALID_ARG, "Hq %% Hkv != 0");
  if (s->causal != 0 && s->causal != 1) return fail(SBFA_ERR_INVALID_ARG, "causal must be 0/1");
  if (s->Sk > sbfa::kMaxKT * 64) return fail(SBFA_ERR_UNSUPPORTED, "Sk > %d", sbfa::kMaxKT * 64);
  return SBFA_OK;
}

float eff_scale(const sbfa_shape* s) {
  return s->scale > 0.f ? s->scale : 1.0f / std::sqrt(static_cast<float>(s->D));
}

#define SBFA_TRY(x)                \
  do {                             \
    sbfa_status st_ = (x);         \
    if (st_ != SBFA_OK) return st_; \
  } while (0)

// Device counters of the self-profiling build (null otherwise); set through
// sbfa_set_profile_counters, which only that build exports.
unsigned long long* g_prof_counters = nullptr;

// Limit of the kernels' bounded waits, read at every launch
// (sbfa_set_wait_limit_ns).
std::atomic<unsigned long long> g_wait_ns{sbfa::kWaitLimitNs};

// ---------------------------------------------------------------------------
// prefill launcher (tcgen05 kernel)
// ---------------------------------------------------------------------------
// Varlen launches describe the packing here: cu_q / cu_k are the device
// cumulative lengths (shape B = number of sequences, Sq / Sk = the longest
// lengths), total_q / total_k the packed row counts of q and k/v.
struct Varlen {
  const int* cu_q = nullptr;
  const int* cu_k = nullptr;
  int total_q = 0, total_k = 0;
};

sbfa_status launch_prefill(sbfa::PrefillParams& p, const sbfa_shape* s, const sbfa_t4& q,
                           const sbfa_t4& k, const sbfa_t4& v, cudaStream_t stream,
                           const Varlen& vl = Varlen()) {
  DevInfo di;
  SBFA_TRY(dev_info(&di));
  p.B = s->B;
  p.Sq = s->Sq;
  p.Sk = s->Sk;
  p.Hq = s->Hq;
  p.Hkv = s->Hkv;
  p.G = s->Hq / s->Hkv;
  p.hp = (p.G % 4 == 0) ? 4 : (p.G % 2 == 0 ? 2 : 1);
  p.subs_per_unit = 4 / p.hp;
  p.n_sub = (s->Sq + 63) / 64;
  p.n_hgrp = p.G / p.hp;
  p.n_subgrp = (p.n_sub + p.subs_per_unit - 1) / p.subs_per_unit;
  const int64_t units = static_cast<int64_t>(p.B) * p.Hkv * p.n_hgrp * p.n_subgrp;
  if (units > 0x7fffffff) return fail(SBFA_ERR_UNSUPPORTED, "too many work units");
  p.n_units = static_cast<int>(units);
  p.n_kt = (s->Sk + 63) / 64;
  p.causal = s->causal;
  p.causal_off = s->Sk - s->Sq;
  p.head_major = (p.mode == sbfa::kModeVS || p.mode == sbfa::kModeGated) ? 1 : 0;
  p.scale = eff_scale(s);
  p.scale_log2 = p.scale * 1.4426950408889634f;
  p.k = static_cast<const __nv_bfloat16*>(k.ptr);
  p.v = static_cast<const __nv_bfloat16*>(v.ptr);
  p.ksb = k.sb; p.kss = k.ss; p.ksh = k.sh;
  p.vsb = v.sb; p.vss = v.ss; p.vsh = v.sh;
  CUtensorMap mq, mk, mv;
  p.cu_q = vl.cu_q;
  p.cu_k = vl.cu_k;
  if (vl.cu_q) {
    SBFA_TRY(encode_bshd(&mq, q, 1, vl.total_q, s->Hq, 64));
    SBFA_TRY(encode_bshd(&mk, k, 1, vl.total_k, s->Hkv, 64));
    SBFA_TRY(encode_bshd(&mv, v, 1, vl.total_k, s->Hkv, 64));
    p.lse_sb = 0;
    p.lse_sh = vl.total_q;
  } else {
    SBFA_TRY(encode_bshd(&mq, q, s->B, s->Sq, s->Hq, 64));
    SBFA_TRY(encode_bshd(&mk, k, s->B, s->Sk, s->Hkv, 64));
    SBFA_TRY(encode_bshd(&mv, v, s->B, s->Sk, s->Hkv, 64));
    p.lse_sb = static_cast<int64_t>(s->Hq) * s->Sq;
    p.lse_sh = s->Sq;
  }
  const size_t smem = sizeof(sbfa::PfSmem) + 1024;
  const bool ext = p.window > 0 || p.fine_shift > 0;
  if ((p.window > 0 && p.mode != sbfa::kModeDense) || (p.fine_shift && p.mode != sbfa::kModeTable))
    return fail(SBFA_ERR_INVALID_ARG, "internal: mask extension in the wrong mode");
  static bool attr_set[64][16] = {};
  int dev = 0;
  SBFA_CUDA(cudaGetDevice(&dev));
  const bool vl_on = vl.cu_q != nullptr;
  const void* fn = nullptr;
  // instantiations: table (with or without small blocks, batched or varlen),
  // dense (plain, window, window varlen), gated, vertical/slash (batched or varlen)
#define SBFA_PF(M, E, V) reinterpret_cast<const void*>(sbfa::prefill_kernel<M, E, V>)
  switch (p.mode) {
    case sbfa::kModeTable:
      fn = ext ? (vl_on ? SBFA_PF(sbfa::kModeTable, true, true) : SBFA_PF(sbfa::kModeTable, true, false))
               : (vl_on ? SBFA_PF(sbfa::kModeTable, false, true) : SBFA_PF(sbfa::kModeTable, false, false));
      break;
    case sbfa::kModeDense:
      if (vl_on && !ext) return fail(SBFA_ERR_INVALID_ARG, "internal: dense varlen without a window");
      fn = ext ? (vl_on ? SBFA_PF(sbfa::kModeDense, true, true) : SBFA_PF(sbfa::kModeDense, true, false))
               : SBFA_PF(sbfa::kModeDense, false, false);
      break;
    case sbfa::kModeGated:
      if (vl_on) return fail(SBFA_ERR_INVALID_ARG, "internal: gated varlen");
      fn = SBFA_PF(sbfa::kModeGated, false, false);
      break;
    case sbfa::kModeVS:
      fn = vl_on ? SBFA_PF(sbfa::kModeVS, false, true) : SBFA_PF(sbfa::kModeVS, false, false);
      break;
    default: return fail(SBFA_ERR_INVALID_ARG, "internal: bad prefill mode");
  }
#undef SBFA_PF
  const int slot = p.mode * 4 + (ext ? 2 : 0) + (vl_on ? 1 : 0);
  if (!attr_set[dev][slot]) {
    SBFA_CUDA(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    attr_set[dev][slot] = true;
  }
  p.prof = g_prof_counters;
  p.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  const int grid = std::min(p.n_units, di.sms);
  void* args[] = {&mq, &mk, &mv, &p};
  SBFA_CUDA(cudaLaunchKernel(fn, dim3(grid), dim3(sbfa::kPfThreads), args, smem, stream));
  SBFA_CUDA(cudaGetLastError());
  return SBFA_OK;
}

sbfa_status check_outputs(const sbfa_t4& o, const float* lse) {
  SBFA_TRY(check_view(o, "o", false));
  if (!lse) return fail(SBFA_ERR_INVALID_ARG, "lse: null pointer");
  return SBFA_OK;
}

// ---------------------------------------------------------------------------
// decode launcher (split-KV kernel)
// ---------------------------------------------------------------------------
struct DecodeWs {
  int* ticket;
  float* part;
  float* lse;
};

size_t decode_ws_bytes(int npairs, int grid) {
  const size_t tick = ((static_cast<size_t>(npairs) * 4 + 255) / 256) * 256;
  const size_t part = static_cast<size_t>(grid) * 2 * sbfa::kDecRows * sbfa::kDecD * 4;
  const size_t lse = static_cast<size_t>(grid) * 2 * sbfa::kDecRows * 4;
  return tick + part + lse;
}

sbfa_status launch_decode(sbfa::DecodeParams& p, const sbfa_shape* s, const sbfa_t4& q,
                          const sbfa_t4* kA, const sbfa_t4* vA, int S_A, int causal_A,
                          const sbfa_t4* kB, const sbfa_t4* vB, const sbfa_table* tb, void* ws,
                          size_t ws_bytes, const sbfa_t4& o, float* lse, int32_t* status,
                          cudaStream_t stream, int grid_cap = 0, int ticket_pairs = 0,
                          bool dedup = false) {
  DevInfo di;
  SBFA_TRY(dev_info(&di));
  const int G = s->Hq / s->Hkv;
  const int npairs = s->B * s->Hkv;
  if (npairs > sbfa::kDecMaxPairs)
    return fail(SBFA_ERR_UNSUPPORTED, "B*Hkv = %d > %d", npairs, sbfa::kDecMaxPairs);
  p.B = s->B; p.Sq = s->Sq; p.Hq = s->Hq; p.Hkv = s->Hkv; p.G = G; p.rows = s->Sq * G;
  p.scale_log2 = eff_scale(s) * 1.4426950408889634f;
  p.q = static_cast<const __nv_bfloat16*>(q.ptr); p.qsb = q.sb; p.qss = q.ss; p.qsh = q.sh;
  p.o = static_cast<__nv_bfloat16*>(o.ptr); p.osb = o.sb; p.oss = o.ss; p.osh = o.sh;
  p.lse = lse;
  p.status = status;
  p.has_A = kA != nullptr;
  p.S_A = S_A;
  p.causal_A = causal_A;
  p.has_B = tb != nullptr;
  auto set_src = [](const sbfa_t4* t, const __nv_bfloat16** ptr, int64_t* sb, int64_t* ss,
                    int64_t* sh) {
    *ptr = static_cast<const __nv_bfloat16*>(t->ptr);
    *sb = t->sb;
    *ss = t->ss;
    *sh = t->sh;
  };
  if (kA) {
    set_src(kA, &p.kA, &p.kAsb, &p.kAss, &p.kAsh);
    set_src(vA, &p.vA, &p.vAsb, &p.vAss, &p.vAsh);
  }
  if (tb) {
    set_src(kB, &p.kB, &p.kBsb, &p.kBss, &p.kBsh);
    set_src(vB, &p.vB, &p.vBsb, &p.vBss, &p.vBsh);
    p.S_B = s->Sk;
    p.kv_block = tb->kv_block;
    p.nmax = tb->nmax;
    p.n_kb = (s->Sk + tb->kv_block - 1) / tb->kv_block;
    p.idx = tb->idx;
    p.tsb = tb->sb;
    p.tsh = tb->sh;
  } else {
    p.S_B = 0; p.kv_block = 64; p.nmax = 0; p.n_kb = 0; p.idx = nullptr; p.tsb = p.tsh = 0;
  }
  const int grid = (grid_cap > 0 && grid_cap < di.sms) ? grid_cap : di.sms;
  if (ws) {
    const int tpairs = ticket_pairs > npairs ? ticket_pairs : npairs;
    const size_t need = decode_ws_bytes(tpairs, grid);
    if (ws_bytes < need)
      return fail(SBFA_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", ws_bytes, need);
    if (!aligned16(ws)) return fail(SBFA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
    uint8_t* w = static_cast<uint8_t*>(ws);
    const size_t tick = ((static_cast<size_t>(tpairs) * 4 + 255) / 256) * 256;
    p.ws_ticket = reinterpret_cast<int*>(w);
    p.ws_part = reinterpret_cast<float*>(w + tick);
    p.ws_lse = reinterpret_cast<float*>(w + tick +
                                        static_cast<size_t>(grid) * 2 * sbfa::kDecRows *
                                            sbfa::kDecD * 4);
    p.pair_mode = 0;
  } else {
    p.ws_ticket = nullptr; p.ws_part = nullptr; p.ws_lse = nullptr;
    p.pair_mode = 1;
  }
  const size_t smem = sizeof(sbfa::DecSmem) + 1024;
  static bool attr_set[64] = {false};
  int dev = 0;
  SBFA_CUDA(cudaGetDevice(&dev));
  if (!attr_set[dev]) {
    SBFA_CUDA(cudaFuncSetAttribute(sbfa::decode_kernel<false>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    SBFA_CUDA(cudaFuncSetAttribute(sbfa::decode_kernel<true>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    attr_set[dev] = true;
  }
  if (dedup)
    sbfa::decode_kernel<true><<<grid, sbfa::kDecThreads, smem, stream>>>(p);
  else
    sbfa::decode_kernel<false><<<grid, sbfa::kDecThreads, smem, stream>>>(p);
  SBFA_CUDA(cudaGetLastError());
  return SBFA_OK;
}

bool decode_shape(const sbfa_shape* s) {
  return s->Sq * (s->Hq / s->Hkv) <= sbfa::kDecRows;
}

sbfa_status check_table(const sbfa_table* t, const sbfa_shape* s, bool prefill) {
  if (!t || !t->idx) return fail(SBFA_ERR_INVALID_ARG, "table: null");
  if (t->nmax < 0) return fail(SBFA_ERR_INVALID_ARG, "table: nmax < 0");
  if (t->sb < 0 || t->sh < 0 || t->sqb < 0) return fail(SBFA_ERR_INVALID_ARG, "table: negative stride");
  if (t->q_block <= 0) return fail(SBFA_ERR_INVALID_ARG, "table: q_block <= 0");
  const int kb = t->kv_block;
  if (prefill) {
    if (kb != 16 && kb != 32 && kb != 64 && kb != 128 && kb != 256)
      return fail(SBFA_ERR_UNSUPPORTED, "kv_block %d (16/32/64/128/256)", kb);
    // 16- and 32-key blocks are tracked one bit each per segment
    if (kb < 64 && s->Sk > sbfa::kBmWords * 32 * kb)
      return fail(SBFA_ERR_UNSUPPORTED, "kv_block %d needs Sk <= %d", kb,
                  sbfa::kBmWords * 32 * kb);
    if (t->q_block % 64 && t->q_block < s->Sq)
      return fail(SBFA_ERR_UNSUPPORTED, "q_block %d: must be a multiple of 64 or >= Sq",
                  t->q_block);
  } else {
    if (kb != 16 && kb != 32 && kb != 64 && kb != 128 && kb != 256)
      return fail(SBFA_ERR_UNSUPPORTED, "kv_block %d", kb);
    if (t->nmax > sbfa::kDecMaxEntries)
      return fail(SBFA_ERR_UNSUPPORTED, "nmax %d > %d", t->nmax, sbfa::kDecMaxEntries);
  }
  return SBFA_OK;
}

// Table fields of the tiled kernel's parameters.
void set_table(sbfa::PrefillParams& p, const sbfa_table* t, int nmax_override = -1) {
  p.idx = t->idx;
  p.tsb = t->sb;
  p.tsh = t->sh;
  p.tsqb = t->sqb;
  p.nmax = nmax_override >= 0 ? nmax_override : t->nmax;
  p.q_block = t->q_block;
  p.kv_block = t->kv_block;
  p.fine_shift = t->kv_block == 16 ? 4 : (t->kv_block == 32 ? 5 : 0);
}

// ---------------------------------------------------------------------------
// NSA selected attention workspace
// ---------------------------------------------------------------------------
struct NsaWs {
  size_t count, cursor, offset, unit_prefix, list, unit_a, unit_b, acc, l_acc, m_key, end_zero,
      total;
  int64_t max_units;
};

size_t al256(size_t x) { return (x + 255) / 256 * 256; }

NsaWs nsa_ws_layout(int nseq, int total, int max_seqlen, int Hq, int Hkv, int topk) {
  const size_t nb = static_cast<size_t>(Hkv) * nseq * ((max_seqlen + 63) / 64);
  NsaWs w;
  size_t off = 0;
  w.count = off; off += al256(nb * 4);
  w.cursor = off; off += al256(nb * 4);
  w.offset = off; off += al256((nb + 1) * 4);
  w.unit_prefix = off; off += al256((nb + 1) * 4);
  w.list = off; off += al256(static_cast<size_t>(total) * Hkv * topk * 4);
  // units: at most entries / rows-per-unit, plus one partial unit per block
  const int64_t per_unit = std::max<int64_t>(1, 128 / std::max(1, Hq / Hkv));
  w.max_units = static_cast<int64_t>(total) * Hkv * topk / per_unit + static_cast<int64_t>(nb);
  w.unit_a = off; off += al256(static_cast<size_t>(w.max_units) * 16);
  w.unit_b = off; off += al256(static_cast<size_t>(w.max_units) * 8);
  // accumulator, sums of P and row-maximum keys: one span, zeroed per call
  w.acc = off; off += al256(static_cast<size_t>(total) * Hq * 128 * 4);
  w.l_acc = off; off += al256(static_cast<size_t>(total) * Hq * 4);
  w.m_key = off; off += al256(static_cast<size_t>(total) * Hq * 4);
  w.end_zero = off;
  w.total = off;
  return w;
}

// ---------------------------------------------------------------------------
// Fixed scratch for sbfa_speculative_sparse_noalloc
// ---------------------------------------------------------------------------
// Callers that cannot allocate device memory (code running inside an
// allocator hook or under a memory budget owned by someone else, or a host
// with no allocator of its own to call) use this file-scope array instead of
// a caller-provided workspace.  It holds the split-KV decode kernel's
// per-pair tickets and per-CTA fp32 partials for up to kNoAllocMaxPairs
// (batch x kv-head) pairs and kNoAllocMaxCtas CTAs.  Every GPU that loads
// the library keeps it until the process exits; all calls share it.
constexpr int kNoAllocMaxPairs = 4096;
constexpr int kNoAllocMaxCtas = 160;
constexpr size_t kNoAllocTicketBytes = kNoAllocMaxPairs * 4;
constexpr size_t kNoAllocBytes =
    kNoAllocTicketBytes +
    static_cast<size_t>(kNoAllocMaxCtas) * 2 * sbfa::kDecRows * (sbfa::kDecD + 1) * 4;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

// Device address of g_noalloc_scratch for the current device.  In host code
// the array's name is only a stand-in, so the address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
sbfa_status noalloc_scratch(void** out) {
  static void* addr[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  SBFA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(SBFA_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
    addr[dev] = p;
  }
  *out = addr[dev];
  return SBFA_OK;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* sbfa_last_error(void) { return g_last_error.c_str(); }

const char* sbfa_version(void) { return "sbfa 0.2 (sm_100a)"; }

uint64_t sbfa_set_wait_limit_ns(uint64_t ns) {
  return g_wait_ns.exchange(ns ? ns : sbfa::kWaitLimitNs);
}

#ifdef SBFA_PROFILE
// Self-profiling build only: device array of 33 uint64 counters that the
// prefill kernel adds its per-role wait cycles to (null disables).
void sbfa_set_profile_counters(unsigned long long* counters) { g_prof_counters = counters; }
#endif

sbfa_status sbfa_fwd(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v,
                     const sbfa_table* table, sbfa_t4 o, float* lse, int32_t* status,
                     sbfa_stream_t stream) {
  g_last_error.clear();
  SBFA_TRY(check_shape(shape));
  SBFA_TRY(check_view(q, "q", true));
  SBFA_TRY(check_view(k, "k", true));
  SBFA_TRY(check_view(v, "v", true));
  SBFA_TRY(check_outputs(o, lse));
  // short query blocks go to the split-KV kernel, which masks no table block:
  // only when the call is not causal or has one query position (for which
  // the bottom-right causal limit admits every key)
  const bool dec = decode_shape(shape) && table && table->q_block >= shape->Sq &&
                   (!shape->causal || shape->Sq == 1);
  SBFA_TRY(check_table(table, shape, !dec));
  if (dec) {
    sbfa::DecodeParams p{};
    // a row is a set of blocks, as on the tiled kernel
    return launch_decode(p, shape, q, nullptr, nullptr, 0, 0, &k, &v, table, nullptr, 0, o,
                         lse, status, reinterpret_cast<cudaStream_t>(stream), 0, 0, true);
  }
  sbfa::PrefillParams p{};
  p.mode = sbfa::kModeTable;
  p.o = o.ptr; p.osb = o.sb; p.oss = o.ss; p.osh = o.sh; p.o_f32 = 0;
  p.lse = lse;
  set_table(p, table);
  p.n_kb = (shape->Sk + table->kv_block - 1) / table->kv_block;
  p.status = status;
  return launch_prefill(p, shape, q, k, v, reinterpret_cast<cudaStream_t>(stream));
}

sbfa_status sbfa_fwd_dense(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v, sbfa_t4 o,
                           float* lse, int32_t* status, sbfa_stream_t stream) {
  g_last_error.clear();
  SBFA_TRY(check_shape(shape));
  SBFA_TRY(check_view(q, "q", true));
  SBFA_TRY(check_view(k, "k", true));
  SBFA_TRY(check_view(v, "v", true));
  SBFA_TRY(check_outputs(o, lse));
  if (decode_shape(shape)) {
    sbfa::DecodeParams p{};
    return launch_decode(p, shape, q, &k, &v, shape->Sk, shape->causal, nullptr, nullptr,
                         nullptr, nullptr, 0, o, lse, status,
                         reinterpret_cast<cudaStream_t>(stream));
  }
  sbfa::PrefillParams p{};
  p.mode = sbfa::kModeDense;
  p.o = o.ptr; p.osb = o.sb; p.oss = o.ss; p.osh = o.sh; p.o_f32 = 0;
  p.lse = lse;
  p.status = status;
  return launch_prefill(p, shape, q, k, v, reinterpret_cast<cudaStream_t>(stream));
}

sbfa_status sbfa_fwd_partials(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v,
                              const sbfa_table* table, float* o_parts, float* lse_parts,
                              int32_t* status, sbfa_stream_t stream) {
  g_last_error.clear();
  SBFA_TRY(check_shape(shape));
  SBFA_TRY(check_view(q, "q", true));
  SBFA_TRY(check_view(k, "k", true));
  SBFA_TRY(check_view(v, "v", true));
  SBFA_TRY(check_table(table, shape, true));
  if (!o_parts || !lse_parts) return fail(SBFA_ERR_INVALID_ARG, "partials: null output");
  if (!aligned16(o_parts)) return fail(SBFA_ERR_INVALID_ARG, "o_parts not 16-byte aligned");
  const int64_t per_o = static_cast<int64_t>(shape->B) * shape->Sq * shape->Hq * shape->D;
  const int64_t per_l = static_cast<int64_t>(shape->B) * shape->Hq * shape->Sq;
  for (int n = 0; n < table->nmax; ++n) {
    sbfa::PrefillParams p{};
    p.mode = sbfa::kModeTable;
    p.o = o_parts + n * per_o;
    p.osb = static_cast<int64_t>(shape->Sq) * shape->Hq * shape->D;
    p.oss = static_cast<int64_t>(shape->Hq) * shape->D;
    p.osh = shape->D;
    p.o_f32 = 1;
    p.lse = lse_parts + n * per_l;
    set_table(p, table, 1);
    p.idx = table->idx + n;
    p.n_kb = (shape->Sk + table->kv_block - 1) / table->kv_block;
    p.status = status;
    SBFA_TRY(launch_prefill(p, shape, q, k, v, reinterpret_cast<cudaStream_t>(stream)));
  }
  return SBFA_OK;
}

sbfa_status sbfa_combine(int32_t n_parts, int32_t B, int32_t Sq, int32_t Hq, int32_t D,
                         const float* o_parts, const float* lse_parts, sbfa_t4 o, float* lse,
                         sbfa_stream_t stream) {
  g_last_error.clear();
  if (n_parts < 0 || B <= 0 || Sq <= 0 || Hq <= 0) return fail(SBFA_ERR_INVALID_ARG, "bad sizes");
  if (D != 128) return fail(SBFA_ERR_UNSUPPORTED, "head dim %d (only 128)", D);
  if ((n_parts > 0 && (!o_parts || !lse_parts)) || !lse || !o.ptr)
    return fail(SBFA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(o_parts)) return fail(SBFA_ERR_INVALID_ARG, "o_parts not 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(o.ptr) & 7u) || (o.sb % 4) || (o.ss % 4) || (o.sh % 4))
    return fail(SBFA_ERR_INVALID_ARG, "o: needs 8-byte aligned rows");
  const int64_t rows = static_cast<int64_t>(B) * Sq * Hq;
  const int threads = 256;
  const int64_t blocks = (rows * 32 + threads - 1) / threads;
  sbfa::combine_kernel<<<static_cast<unsigned>(blocks), threads, 0,
                         reinterpret_cast<cudaStream_t>(stream)>>>(
      n_parts, B, Sq, Hq, o_parts, lse_parts, static_cast<__nv_bfloat16*>(o.ptr), o.sb, o.ss,
      o.sh, lse);
  SBFA_CUDA(cudaGetLastError());
  return SBFA_OK;
}

size_t sbfa_decode_workspace_size(int32_t B, int32_t Hkv, int32_t Sq, int32_t Hq) {
  (void)Sq;
  (void)Hq;
  DevInfo di;
  if (dev_info(&di) != SBFA_OK) return 0;
  return decode_ws_bytes(B * Hkv, di.sms);
}

sbfa_status sbfa_speculative_sparse(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k_spec,
                                    sbfa_t4 v_spec, int32_t S_spec, int32_t causal_spec,
                                    sbfa_t4 k, sbfa_t4 v, const sbfa_table* missed, void* ws,
                                    size_t ws_bytes, sbfa_t4 o, float* lse, int32_t* status,
                                    sbfa_stream_t stream) {
  g_last_error.clear();
  SBFA_TRY(check_shape(shape));
  SBFA_TRY(check_view(q, "q", false));
  SBFA_TRY(check_view(k_spec, "k_spec", true));
  SBFA_TRY(check_view(v_spec, "v_spec", true));
  SBFA_TRY(check_view(k, "k", true));
  SBFA_TRY(check_view(v, "v", true));
  SBFA_TRY(check_outputs(o, lse));
  if (S_spec <= 0) return fail(SBFA_ERR_INVALID_ARG, "S_spec <= 0");
  if (causal_spec != 0 && causal_spec != 1) return fail(SBFA_ERR_INVALID_ARG, "causal_spec");
  if (!decode_shape(shape))
    return fail(SBFA_ERR_UNSUPPORTED, "Sq * Hq/Hkv = %d > %d", shape->Sq * (shape->Hq / shape->Hkv),
                sbfa::kDecRows);
  SBFA_TRY(check_table(missed, shape, false));
  if (missed->q_block < shape->Sq) return fail(SBFA_ERR_UNSUPPORTED, "missed->q_block < Sq");
  if (!ws) return fail(SBFA_ERR_INVALID_ARG, "workspace is null");
  sbfa::DecodeParams p{};
  return launch_decode(p, shape, q, &k_spec, &v_spec, S_spec, causal_spec, &k, &v, missed, ws,
                       ws_bytes, o, lse, status, reinterpret_cast<cudaStream_t>(stream));
}

sbfa_status sbfa_speculative_sparse_noalloc(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k_spec,
                                            sbfa_t4 v_spec, int32_t S_spec, int32_t causal_spec,
                                            sbfa_t4 k, sbfa_t4 v, const sbfa_table* missed,
                                            sbfa_t4 o, float* lse, int32_t* status,
                                            sbfa_stream_t stream) {
  g_last_error.clear();
  SBFA_TRY(check_shape(shape));
  SBFA_TRY(check_view(q, "q", false));
  SBFA_TRY(check_view(k_spec, "k_spec", true));
  SBFA_TRY(check_view(v_spec, "v_spec", true));
  SBFA_TRY(check_view(k, "k", true));
  SBFA_TRY(check_view(v, "v", true));
  SBFA_TRY(check_outputs(o, lse));
  if (S_spec <= 0) return fail(SBFA_ERR_INVALID_ARG, "S_spec <= 0");
  if (causal_spec != 0 && causal_spec != 1) return fail(SBFA_ERR_INVALID_ARG, "causal_spec");
  if (!decode_shape(shape))
    return fail(SBFA_ERR_UNSUPPORTED, "Sq * Hq/Hkv = %d > %d", shape->Sq * (shape->Hq / shape->Hkv),
                sbfa::kDecRows);
  SBFA_TRY(check_table(missed, shape, false));
  if (missed->q_block < shape->Sq) return fail(SBFA_ERR_UNSUPPORTED, "missed->q_block < Sq");
  const int npairs = shape->B * shape->Hkv;
  if (npairs > kNoAllocMaxPairs)
    return fail(SBFA_ERR_UNSUPPORTED,
                "B*Hkv = %d exceeds the fixed scratch limit of %d pairs (use "
                "sbfa_speculative_sparse with a workspace)", npairs, kNoAllocMaxPairs);
  void* scratch = nullptr;
  SBFA_TRY(noalloc_scratch(&scratch));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the tickets must start at zero (a previous call may have stopped early)
  SBFA_CUDA(cudaMemsetAsync(scratch, 0, static_cast<size_t>(npairs) * 4, st));
  // lay the partials out after the full ticket area, as decode_ws_bytes does
  // for npairs = kNoAllocMaxPairs
  sbfa::DecodeParams p{};
  return launch_decode(p, shape, q, &k_spec, &v_spec, S_spec, causal_spec, &k, &v, missed,
                       scratch, kNoAllocBytes, o, lse, status, st, kNoAllocMaxCtas,
                       kNoAllocMaxPairs);
}

sbfa_status sbfa_fwd_gated(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v,
                           const float* T, int32_t block, sbfa_t4 o, float* lse, float* smax_out,
                           uint8_t* keep_out, int32_t* status, sbfa_stream_t stream) {
  g_last_error.clear();
  SBFA_TRY(check_shape(shape));
  SBFA_TRY(check_view(q, "q", true));
  SBFA_TRY(check_view(k, "k", true));
  SBFA_TRY(check_view(v, "v", true));
  SBFA_TRY(check_outputs(o, lse));
  if (!T) return fail(SBFA_ERR_INVALID_ARG, "T is null");
  if (block != 64) return fail(SBFA_ERR_UNSUPPORTED, "gate block %d (only 64)", block);
  if (shape->Sq != shape->Sk || !shape->causal)
    return fail(SBFA_ERR_UNSUPPORTED, "gated mode needs Sq == Sk and causal");
  sbfa::PrefillParams p{};
  p.mode = sbfa::kModeGated;
  p.o = o.ptr; p.osb = o.sb; p.oss = o.ss; p.osh = o.sh; p.o_f32 = 0;
  p.lse = lse;
  p.T = T;
  p.nqb = (shape->Sq + 63) / 64;
  p.smax_out = smax_out;
  p.keep_out = keep_out;
  p.status = status;
  return launch_prefill(p, shape, q, k, v, reinterpret_cast<cudaStream_t>(stream));
}

sbfa_status sbfa_convert_vertical_slash(const int32_t* q_seqlens, const int32_t* kv_seqlens,
                                        const int32_t* vertical, int32_t nnz_v,
                                        const int32_t* slash, int32_t nnz_s, int32_t B,
                                        int32_t H, int32_t context_size, int32_t block_M,
                                        int32_t block_N, int32_t causal, int32_t* block_count,
                                        int32_t* block_offset, int32_t* column_count,
                                        int32_t* column_index, int32_t* status,
                                        sbfa_stream_t stream) {
  g_last_error.clear();
  if (!q_seqlens || !kv_seqlens || !vertical || !slash || !block_count || !block_offset ||
      !column_count || !column_index)
    return fail(SBFA_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || H <= 0 || context_size <= 0 || nnz_v < 0 || nnz_s < 0)
    return fail(SBFA_ERR_INVALID_ARG, "bad sizes");
  if (block_M != 64 || block_N != 64)
    return fail(SBFA_ERR_UNSUPPORTED, "block_M = block_N = 64 only");
  if (context_size > sbfa::kCvMaxWords * 32 * 64)
    return fail(SBFA_ERR_UNSUPPORTED, "context_size too large");
  const int nqb = (context_size + block_M - 1) / block_M;
  const int64_t grid = static_cast<int64_t>(B) * H * nqb;
  sbfa::convert_vs_kernel<<<static_cast<unsigned>(grid), sbfa::kCvThreads, 0,
                            reinterpret_cast<cudaStream_t>(stream)>>>(
      q_seqlens, kv_seqlens, vertical, nnz_v, slash, nnz_s, nullptr, nullptr, H, nqb, block_M,
      block_N, causal, block_count, block_offset, column_count, column_index, status);
  SBFA_CUDA(cudaGetLastError());
  return SBFA_OK;
}

sbfa_status sbfa_convert_vertical_slash_mergehead(
    const int32_t* q_seqlens, const int32_t* kv_seqlens, const int32_t* vertical, int32_t nnz_v,
    const int32_t* slash, int32_t nnz_s, const int32_t* vertical_count,
    const int32_t* slash_count, int32_t B, int32_t H, int32_t context_size, int32_t block_M,
    int32_t block_N, int32_t causal, int32_t* block_count, int32_t* block_offset,
    int32_t* column_count, int32_t* column_index, int32_t* status, sbfa_stream_t stream) {
  g_last_error.clear();
  if (!q_seqlens || !kv_seqlens || !vertical || !slash || !vertical_count || !slash_count ||
      !block_count || !block_offset || !column_count || !column_index)
    return fail(SBFA_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || H <= 0 || context_size <= 0 || nnz_v < 0 || nnz_s < 0)
    return fail(SBFA_ERR_INVALID_ARG, "bad sizes");
  if (block_M != 64 || block_N != 64)
    return fail(SBFA_ERR_UNSUPPORTED, "block_M = block_N = 64 only");
  if (context_size > sbfa::kCvMaxWords * 32 * 64)
    return fail(SBFA_ERR_UNSUPPORTED, "context_size too large");
  const int nqb = (context_size + block_M - 1) / block_M;
  const int64_t grid = static_cast<int64_t>(B) * H * nqb;
  sbfa::convert_vs_kernel<<<static_cast<unsigned>(grid), sbfa::kCvThreads, 0,
                            reinterpret_cast<cudaStream_t>(stream)>>>(
      q_seqlens, kv_seqlens, vertical, nnz_v, slash, nnz_s, vertical_count, slash_count, H, nqb,
      block_M, block_N, causal, block_count, block_offset, column_count, column_index, status);
  SBFA_CUDA(cudaGetLastError());
  return SBFA_OK;
}

sbfa_status sbfa_fwd_vertical_slash(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v,
                                    const int32_t* block_count, const int32_t* block_offset,
                                    int32_t nnz_s, const int32_t* column_count,
                                    const int32_t* column_index, int32_t nnz_v, int32_t block_M,
                                    int32_t block_N, sbfa_t4 o, float* lse, int32_t* status,
                                    sbfa_stream_t stream) {
  g_last_error.clear();
  SBFA_TRY(check_shape(shape));
  SBFA_TRY(check_view(q, "q", true));
  SBFA_TRY(check_view(k, "k", true));
  SBFA_TRY(check_view(v, "v", true));
  SBFA_TRY(check_outputs(o, lse));
  if (block_M != 64 || block_N != 64)
    return fail(SBFA_ERR_UNSUPPORTED, "block_M = block_N = 64 only");
  if (!block_count || !block_offset || !column_count || !column_index)
    return fail(SBFA_ERR_INVALID_ARG, "null index array");
  if (nnz_s < 0 || nnz_v < 0) return fail(SBFA_ERR_INVALID_ARG, "negative nnz");
  if ((k.ss % 8) || (v.ss % 8)) return fail(SBFA_ERR_INVALID_ARG, "k/v row stride");
  sbfa::PrefillParams p{};
  p.mode = sbfa::kModeVS;
  p.o = o.ptr; p.osb = o.sb; p.oss = o.ss; p.osh = o.sh; p.o_f32 = 0;
  p.lse = lse;
  p.vs_bc = block_count; p.vs_bo = block_offset; p.nnz_s = nnz_s;
  p.vs_cc = column_count; p.vs_ci = column_index; p.nnz_v = nnz_v;
  p.vs_nqb = (shape->Sq + 63) / 64;
  p.status = status;
  return launch_prefill(p, shape, q, k, v, reinterpret_cast<cudaStream_t>(stream));
}

// Shared checks of the cu_seqlens entry points; fills the shape the
// launcher sizes its unit grid with (B = sequences, longest lengths).
static sbfa_status varlen_shape(const int32_t* cu_q, const int32_t* cu_k, int32_t nseq, int32_t total_q,
                         int32_t total_k, int32_t max_q, int32_t max_k, int32_t Hq, int32_t Hkv,
                         int32_t D, float scale, int32_t causal, const sbfa_t4& q,
                         const sbfa_t4& k, const sbfa_t4& v, const sbfa_t4& o, const float* lse,
                         sbfa_shape* sh) {
  if (!cu_q || !cu_k) return fail(SBFA_ERR_INVALID_ARG, "cu_seqlens: null pointer");
  if (nseq <= 0 || total_q <= 0 || total_k <= 0 || max_q <= 0 || max_k <= 0)
    return fail(SBFA_ERR_INVALID_ARG, "non-positive size");
  *sh = sbfa_shape{nseq, max_q, max_k, Hq, Hkv, D, scale, causal};
  SBFA_TRY(check_shape(sh));
  SBFA_TRY(check_view(q, "q", true));
  SBFA_TRY(check_view(k, "k", true));
  SBFA_TRY(check_view(v, "v", true));
  SBFA_TRY(check_outputs(o, lse));
  return SBFA_OK;
}

sbfa_status sbfa_fwd_varlen(const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            int32_t nseq, int32_t total_q, int32_t total_k,
                            int32_t max_seqlen_q, int32_t max_seqlen_k, int32_t Hq, int32_t Hkv,
                            int32_t D, float scale, int32_t causal, sbfa_t4 q, sbfa_t4 k,
                            sbfa_t4 v, const sbfa_table* table, sbfa_t4 o, float* lse,
                            int32_t* status, sbfa_stream_t stream) {
  g_last_error.clear();
  sbfa_shape sh;
  SBFA_TRY(varlen_shape(cu_seqlens_q, cu_seqlens_k, nseq, total_q, total_k, max_seqlen_q,
                        max_seqlen_k, Hq, Hkv, D, scale, causal, q, k, v, o, lse, &sh));
  SBFA_TRY(check_table(table, &sh, true));
  sbfa::PrefillParams p{};
  p.mode = sbfa::kModeTable;
  p.o = o.ptr; p.osb = 0; p.oss = o.ss; p.osh = o.sh; p.o_f32 = 0;
  p.lse = lse;
  set_table(p, table);
  p.status = status;
  Varlen vl;
  vl.cu_q = cu_seqlens_q; vl.cu_k = cu_seqlens_k; vl.total_q = total_q; vl.total_k = total_k;
  return launch_prefill(p, &sh, q, k, v, reinterpret_cast<cudaStream_t>(stream), vl);
}

sbfa_status sbfa_fwd_window(const sbfa_shape* shape, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v,
                            int32_t window, sbfa_t4 o, float* lse, int32_t* status,
                            sbfa_stream_t stream) {
  g_last_error.clear();
  SBFA_TRY(check_shape(shape));
  SBFA_TRY(check_view(q, "q", true));
  SBFA_TRY(check_view(k, "k", true));
  SBFA_TRY(check_view(v, "v", true));
  SBFA_TRY(check_outputs(o, lse));
  if (window <= 0) return fail(SBFA_ERR_INVALID_ARG, "window must be positive");
  sbfa_shape sh = *shape;
  sh.causal = 1;  // the window is causal
  sbfa::PrefillParams p{};
  p.mode = sbfa::kModeDense;
  p.window = window;
  p.o = o.ptr; p.osb = o.sb; p.oss = o.ss; p.osh = o.sh; p.o_f32 = 0;
  p.lse = lse;
  p.status = status;
  return launch_prefill(p, &sh, q, k, v, reinterpret_cast<cudaStream_t>(stream));
}

sbfa_status sbfa_fwd_window_varlen(const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                   int32_t nseq, int32_t total_q, int32_t total_k,
                                   int32_t max_seqlen_q, int32_t max_seqlen_k, int32_t Hq,
                                   int32_t Hkv, int32_t D, float scale, int32_t window, sbfa_t4 q,
                                   sbfa_t4 k, sbfa_t4 v, sbfa_t4 o, float* lse, int32_t* status,
                                   sbfa_stream_t stream) {
  g_last_error.clear();
  sbfa_shape sh;
  SBFA_TRY(varlen_shape(cu_seqlens_q, cu_seqlens_k, nseq, total_q, total_k, max_seqlen_q,
                        max_seqlen_k, Hq, Hkv, D, scale, 1, q, k, v, o, lse, &sh));
  if (window <= 0) return fail(SBFA_ERR_INVALID_ARG, "window must be positive");
  sbfa::PrefillParams p{};
  p.mode = sbfa::kModeDense;
  p.window = window;
  p.o = o.ptr; p.osb = 0; p.oss = o.ss; p.osh = o.sh; p.o_f32 = 0;
  p.lse = lse;
  p.status = status;
  Varlen vl;
  vl.cu_q = cu_seqlens_q; vl.cu_k = cu_seqlens_k; vl.total_q = total_q; vl.total_k = total_k;
  return launch_prefill(p, &sh, q, k, v, reinterpret_cast<cudaStream_t>(stream), vl);
}

sbfa_status sbfa_fwd_vertical_slash_varlen(
    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int32_t nseq, int32_t total_q,
    int32_t total_k, int32_t max_seqlen_q, int32_t max_seqlen_k, int32_t Hq, int32_t Hkv,
    int32_t D, float scale, int32_t causal, sbfa_t4 q, sbfa_t4 k, sbfa_t4 v,
    const int32_t* block_count, const int32_t* block_offset, int32_t nnz_s,
    const int32_t* column_count, const int32_t* column_index, int32_t nnz_v, int32_t block_M,
    int32_t block_N, sbfa_t4 o, float* lse, int32_t* status, sbfa_stream_t stream) {
  g_last_error.clear();
  sbfa_shape sh;
  SBFA_TRY(varlen_shape(cu_seqlens_q, cu_seqlens_k, nseq, total_q, total_k, max_seqlen_q,
                        max_seqlen_k, Hq, Hkv, D, scale, causal, q, k, v, o, lse, &sh));
  if (block_M != 64 || block_N != 64)
    return fail(SBFA_ERR_UNSUPPORTED, "block_M = block_N = 64 only");
  if (!block_count || !block_offset || !column_count || !column_index)
    return fail(SBFA_ERR_INVALID_ARG, "null index array");
  if (nnz_s < 0 || nnz_v < 0) return fail(SBFA_ERR_INVALID_ARG, "negative nnz");
  sbfa::PrefillParams p{};
  p.mode = sbfa::kModeVS;
  p.o = o.ptr; p.osb = 0; p.oss = o.ss; p.osh = o.sh; p.o_f32 = 0;
  p.lse = lse;
  p.vs_bc = block_count; p.vs_bo = block_offset; p.nnz_s = nnz_s;
  p.vs_cc = column_count; p.vs_ci = column_index; p.nnz_v = nnz_v;
  p.vs_nqb = (max_seqlen_q + 63) / 64;
  p.status = status;
  Varlen vl;
  vl.cu_q = cu_seqlens_q; vl.cu_k = cu_seqlens_k; vl.total_q = total_q; vl.total_k = total_k;
  return launch_prefill(p, &sh, q, k, v, reinterpret_cast<cudaStream_t>(stream), vl);
}

size_t sbfa_varlen_selected_workspace_size(int32_t nseq, int32_t total, int32_t max_seqlen,
                                           int32_t Hq, int32_t Hkv, int32_t topk) {
  if (nseq <= 0 || total <= 0 || max_seqlen <= 0 || Hq <= 0 || Hkv <= 0 || topk <= 0) return 0;
  return nsa_ws_layout(nseq, total, max_seqlen, Hq, Hkv, topk).total;
}

sbfa_status sbfa_fwd_varlen_selected(const int32_t* cu_seqlens, int32_t nseq, int32_t total,
                                     int32_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t D,
                                     float scale, int32_t causal, sbfa_t4 q, sbfa_t4 k,
                                     sbfa_t4 v, const int32_t* sel, int32_t topk, int32_t block,
                                     void* ws, size_t ws_bytes, sbfa_t4 o, float* lse,
                                     int32_t* status, sbfa_stream_t stream) {
  g_last_error.clear();
  if (!cu_seqlens || !sel || !ws || !lse) return fail(SBFA_ERR_INVALID_ARG, "null pointer");
  if (nseq <= 0 || total <= 0 || max_seqlen <= 0 || Hq <= 0 || Hkv <= 0 || topk <= 0)
    return fail(SBFA_ERR_INVALID_ARG, "non-positive size");
  if (D != 128) return fail(SBFA_ERR_UNSUPPORTED, "head dim %d (only 128)", D);
  if (block != 64) return fail(SBFA_ERR_UNSUPPORTED, "selection block %d (only 64)", block);
  if (Hq % Hkv || 128 % (Hq / Hkv)) return fail(SBFA_ERR_UNSUPPORTED, "Hq/Hkv must divide 128");
  if (causal != 0 && causal != 1) return fail(SBFA_ERR_INVALID_ARG, "causal must be 0/1");
  if (static_cast<int64_t>(total) * topk >= (1ll << 31))
    return fail(SBFA_ERR_UNSUPPORTED, "total * topk too large");
  SBFA_TRY(check_view(q, "q", true));
  SBFA_TRY(check_view(k, "k", true));
  SBFA_TRY(check_view(v, "v", true));
  SBFA_TRY(check_view(o, "o", false));
  // q rows (token, head) are gathered from the flattened row t * Hq + h
  if (Hq > 1 && q.ss != static_cast<int64_t>(Hq) * q.sh)
    return fail(SBFA_ERR_UNSUPPORTED, "q: token stride must equal Hq * head stride");
  const NsaWs L = nsa_ws_layout(nseq, total, max_seqlen, Hq, Hkv, topk);
  if (ws_bytes < L.total)
    return fail(SBFA_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", ws_bytes, L.total);
  if (!aligned16(ws)) return fail(SBFA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  DevInfo di;
  SBFA_TRY(dev_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  sbfa::NsaParams p{};
  p.nseq = nseq; p.total = total; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv; p.topk = topk;
  p.nbps = (max_seqlen + 63) / 64;
  p.causal = causal;
  p.scale_log2 = (scale > 0.f ? scale : 1.0f / std::sqrt(128.f)) * 1.4426950408889634f;
  p.cu = cu_seqlens; p.sel = sel;
  p.q = static_cast<const __nv_bfloat16*>(q.ptr); p.qss = q.ss; p.qsh = q.sh;
  p.count = reinterpret_cast<int*>(w + L.count);
  p.cursor = reinterpret_cast<int*>(w + L.cursor);
  p.offset = reinterpret_cast<int*>(w + L.offset);
  p.unit_prefix = reinterpret_cast<int*>(w + L.unit_prefix);
  p.list = reinterpret_cast<int*>(w + L.list);
  p.unit_a = reinterpret_cast<int4*>(w + L.unit_a);
  p.unit_b = reinterpret_cast<int2*>(w + L.unit_b);
  if (L.max_units >= (1ll << 31)) return fail(SBFA_ERR_UNSUPPORTED, "too many units");
  p.max_units = static_cast<int>(L.max_units);
  p.acc = reinterpret_cast<float*>(w + L.acc);
  p.l_acc = reinterpret_cast<float*>(w + L.l_acc);
  p.m_key = reinterpret_cast<uint32_t*>(w + L.m_key);
  p.o = static_cast<__nv_bfloat16*>(o.ptr); p.oss = o.ss; p.osh = o.sh;
  p.lse = lse;
  p.status = status;
  p.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  const int64_t nb = static_cast<int64_t>(Hkv) * nseq * p.nbps;
  if (nb > (1 << 26)) return fail(SBFA_ERR_UNSUPPORTED, "too many key blocks");
  CUtensorMap mq, mk, mv;
  SBFA_TRY(encode_rows2d(&mq, q.ptr, static_cast<int64_t>(total) * Hq, Hq > 1 ? q.sh : q.ss));
  SBFA_TRY(encode_bshd(&mk, k, 1, total, Hkv, 64));
  SBFA_TRY(encode_bshd(&mv, v, 1, total, Hkv, 64));
  SBFA_CUDA(cudaMemsetAsync(p.count, 0, nb * 4, st));
  SBFA_CUDA(cudaMemsetAsync(w + L.acc, 0, L.end_zero - L.acc, st));
  // inverted index: shared-memory histograms when the key space fits, else
  // one global atomic per (warp, key)
  const bool hist = nb <= sbfa::kNsaHistMaxKeys;
  const unsigned g1 = static_cast<unsigned>((total + sbfa::kNsaTokTile - 1) / sbfa::kNsaTokTile);
  p.hist_tokens = (total + di.sms - 1) / di.sms;
  const unsigned gh = static_cast<unsigned>((total + p.hist_tokens - 1) / p.hist_tokens);
  const size_t hsm = static_cast<size_t>(nb) * 4;
  static bool hist_attr[64] = {false};
  int hdev = 0;
  SBFA_CUDA(cudaGetDevice(&hdev));
  if (hist && !hist_attr[hdev]) {
    SBFA_CUDA(cudaFuncSetAttribute(sbfa::nsa_count_hist_kernel,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   sbfa::kNsaHistMaxKeys * 4));
    SBFA_CUDA(cudaFuncSetAttribute(sbfa::nsa_fill_hist_kernel,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   sbfa::kNsaHistMaxKeys * 8));
    hist_attr[hdev] = true;
  }
  if (hist) sbfa::nsa_count_hist_kernel<<<gh, sbfa::kNsaHistThreads, hsm, st>>>(p);
  else sbfa::nsa_count_kernel<<<g1, sbfa::kNsaIdxThreads, 0, st>>>(p);
  SBFA_CUDA(cudaGetLastError());
  sbfa::nsa_scan_kernel<<<1, 1024, 0, st>>>(p);
  SBFA_CUDA(cudaGetLastError());
  if (hist) sbfa::nsa_fill_hist_kernel<<<gh, sbfa::kNsaHistThreads, 2 * hsm, st>>>(p);
  else sbfa::nsa_fill_kernel<<<g1, sbfa::kNsaIdxThreads, 0, st>>>(p);
  SBFA_CUDA(cudaGetLastError());
  sbfa::nsa_units_kernel<<<static_cast<unsigned>((L.max_units + 255) / 256), 256, 0, st>>>(p);
  SBFA_CUDA(cudaGetLastError());
  const size_t smem1 = sizeof(sbfa::NsaSmem1) + 1024;
  const size_t smem2 = sizeof(sbfa::NsaSmem2) + 1024;
  static bool attr_set[64] = {false};
  int dev = 0;
  SBFA_CUDA(cudaGetDevice(&dev));
  if (!attr_set[dev]) {
    SBFA_CUDA(cudaFuncSetAttribute(sbfa::nsa_main_kernel<1>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1));
    SBFA_CUDA(cudaFuncSetAttribute(sbfa::nsa_main_kernel<2>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2));
    attr_set[dev] = true;
  }
  // pass 1: row maxima; pass 2: accumulation over the same units
  sbfa::nsa_main_kernel<1><<<di.sms, sbfa::kNsaThreads, smem1, st>>>(mq, mk, mv, p);
  SBFA_CUDA(cudaGetLastError());
  sbfa::nsa_main_kernel<2><<<di.sms, sbfa::kNsaThreads, smem2, st>>>(mq, mk, mv, p);
  SBFA_CUDA(cudaGetLastError());
  const int64_t rows = static_cast<int64_t>(total) * Hq;
  sbfa::nsa_finalize_kernel<<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, st>>>(p);
  SBFA_CUDA(cudaGetLastError());
  return SBFA_OK;
}

sbfa_status sbfa_calibrate_thresholds(const float* smax, int32_t B, int32_t Hq, int32_t n_qb,
                                      int32_t k_top, float* T, sbfa_stream_t stream) {
  g_last_error.clear();
  if (!smax || !T) return fail(SBFA_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || Hq <= 0 || n_qb <= 0) return fail(SBFA_ERR_INVALID_ARG, "non-positive size");
  if (k_top <= 0) return fail(SBFA_ERR_INVALID_ARG, "k must be positive");
  const int64_t rows = static_cast<int64_t>(B) * Hq * n_qb;
  if (rows >= (1ll << 31)) return fail(SBFA_ERR_UNSUPPORTED, "too many rows");
  DevInfo di;
  SBFA_TRY(dev_info(&di));
  sbfa::calibrate_kernel<<<static_cast<unsigned>(rows), sbfa::kCalThreads, 0,
                           reinterpret_cast<cudaStream_t>(stream)>>>(smax, n_qb, k_top, T);
  SBFA_CUDA(cudaGetLastError());
  return SBFA_OK;
}

sbfa_status sbfa_check_status(const int32_t* status, sbfa_stream_t stream) {
  g_last_error.clear();
  SBFA_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  if (!status) return SBFA_OK;
  int32_t h = 0;
  SBFA_CUDA(cudaMemcpy(&h, status, sizeof(h), cudaMemcpyDeviceToHost));
  if (h & SBFA_DEV_TIMEOUT) return fail(SBFA_ERR_TIMEOUT, "device status 0x%x", h);
  if (h) return fail(SBFA_ERR_DEVICE, "device status 0x%x", h);
  return SBFA_OK;
}

}  // extern "C"
