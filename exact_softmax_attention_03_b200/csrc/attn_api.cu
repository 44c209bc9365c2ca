// attn_api.cu — the C ABI declared in include/attn.h: host-side argument
// validation, TMA descriptor encoding, launch configuration and error codes.
// Compiled as a single translation unit with the kernels it launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <type_traits>

#include "../../include/attn.h"
#include "backward_kernels.cuh"
#include "decode_kernels.cuh"
#include "merge_kernel.cuh"
#include "prefill_kernel.cuh"

namespace {

thread_local char g_err[512] = "";
std::atomic<unsigned long long> g_launches{0};

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int ok() {
  g_err[0] = '\0';
  return ATTN_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The device current on this thread must be a compute-capability 10.0 part
// (sm_100a code only). Result cached per device ordinal.
int check_device(int* dev_out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  static std::atomic<int> cache[64];   // 0 unknown, 1 ok, 2 unsupported
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load();
    if (c == 1) { *dev_out = dev; return ATTN_OK; }
    if (c == 2) return fail(ATTN_ERR_UNSUPPORTED, "device %d is not sm_100", dev);
  }
  int major = 0, minor = 0;
  if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
    return fail(ATTN_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
  const bool good = (major == 10 && minor == 0);
  if (dev >= 0 && dev < 64) cache[dev].store(good ? 1 : 2);
  if (!good) return fail(ATTN_ERR_UNSUPPORTED, "device %d is sm_%d%d, need sm_100", dev, major, minor);
  *dev_out = dev;
  return ATTN_OK;
}

// Number of SMs of device `dev`, cached per device ordinal.
int sm_count(int dev, int* out) {
  static std::atomic<int> cache[64];
  if (dev >= 0 && dev < 64 && cache[dev].load() > 0) {
    *out = cache[dev].load();
    return ATTN_OK;
  }
  int n = 0;
  cudaError_t e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess || n <= 0) return fail(ATTN_ERR_CUDA, "SM count: %s", cudaGetErrorString(e));
  if (dev >= 0 && dev < 64) cache[dev].store(n);
  *out = n;
  return ATTN_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 4-D view {d, H, N, B} of a contiguous bf16 [B, N, H, d] tensor; box
// {64, 1, 128, 1} with 128-byte swizzle (one 128-row x 128-byte block).
// 4-D view {d, H, N, B} of a [B, N, H, d] bf16 tensor, boxes of 64 columns x
// box_rows rows with the 128-byte swizzle.
// (box_cols = 32: 64-byte rows with the 64-byte swizzle.)
int make_map(CUtensorMap* map, const void* base, int d, int H, int N, int B, int box_rows = 128,
             int box_cols = 64) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(H), cuuint64_t(N), cuuint64_t(B)};
  cuuint64_t strides[3] = {cuuint64_t(d) * 2, cuuint64_t(H) * d * 2, cuuint64_t(N) * H * d * 2};
  cuuint32_t box[4] = {cuuint32_t(box_cols), 1, cuuint32_t(box_rows), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return ATTN_OK;
}

// Page pool [num_pages, page_size, H, d] as a 5-D tensor {64, d/64, H, page_size,
// num_pages}: one box of {64, d/64, 1, box_rows, 1} brings box_rows rows of one
// page, every 64-column block of each row.
int make_map_pool(CUtensorMap* map, const void* base, int d, int H, int ps, int np, int box_rows) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[5] = {64, cuuint64_t(d / 64), cuuint64_t(H), cuuint64_t(ps), cuuint64_t(np)};
  cuuint64_t strides[4] = {128, cuuint64_t(d) * 2, cuuint64_t(H) * d * 2, cuuint64_t(ps) * H * d * 2};
  cuuint32_t box[5] = {64, cuuint32_t(d / 64), 1, cuuint32_t(box_rows), 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return ATTN_OK;
}

bool finite_pos(float x) { return std::isfinite(x) && x > 0.f; }

constexpr long long kMaxIndex = (1ll << 31) - 1;
// longest cache a decode call takes: its split length, rounded up to whole
// 128-key tiles, must still fit the kernels' 32-bit positions
constexpr long long kMaxKeys = kMaxIndex - 127;

int validate_fwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal) {
  if (!q || !k || !v || !o) return fail(ATTN_ERR_INVALID_ARG, "q, k, v and o must be non-null");
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1)
    return fail(ATTN_ERR_INVALID_ARG, "B, Hq, Hkv, Nq, Nk must be >= 1");
  if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  if (d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not in {64, 128}", d);
  if (!finite_pos(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (causal != 0 && causal != 1) return fail(ATTN_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16))
    return fail(ATTN_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned");
  if (lse && !aligned(lse, 4)) return fail(ATTN_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  // index arithmetic in the kernels uses 32-bit rows and positions
  if (static_cast<long long>(B) * Nq > kMaxIndex || static_cast<long long>(B) * Nk > kMaxIndex ||
      static_cast<long long>(B) * Hq > kMaxIndex)
    return fail(ATTN_ERR_INVALID_ARG, "sizes too large");
  return ATTN_OK;
}

// Packed variable-length input: sequence offsets (device) and packed row counts.
struct Packed {
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
};

// Multiplier and shift of attn::fdiv for the divisor d >= 1 (see FastDiv).
attn::FastDiv make_fastdiv(int d) {
  attn::FastDiv f{0u, 0u};
  if (d <= 1) return f;
  int l = 0;
  while ((1ll << l) < d) ++l;                            // ceil(log2 d)
  const unsigned long long two_p = 1ull << (31 + l);
  f.m = static_cast<uint32_t>((two_p + static_cast<unsigned long long>(d) - 1) / static_cast<unsigned long long>(d));
  f.s = static_cast<uint32_t>(l - 1);
  return f;
}

template <int D, bool F32OUT, bool VARLEN>
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
               int Hkv, int Nq, int Nk, float scale, int causal, int window_left,
               cudaStream_t stream, int dev, const Packed* pk = nullptr) {
  using L = attn::FwdLayout<D, VARLEN>;
  CUtensorMap mq, mk, mv;
  int rc;
  // packed input: one "batch" of total rows; the kernel adds each sequence's offset
  const int rq = pk ? pk->total_q : Nq, rk = pk ? pk->total_k : Nk, nb = pk ? 1 : B;
  if ((rc = make_map(&mq, q, D, Hq, rq, nb)) != ATTN_OK) return rc;
  if ((rc = make_map(&mk, k, D, Hkv, rk, nb)) != ATTN_OK) return rc;
  if ((rc = make_map(&mv, v, D, Hkv, rk, nb)) != ATTN_OK) return rc;
  CUtensorMap mo = mq;                 // O map: used by the bf16-output kernels only
  if (!F32OUT && (rc = (VARLEN ? make_map(&mo, o, D, Hq, rq, 1, 32, 32)
                               : make_map(&mo, o, D, Hq, Nq, B, 32))) != ATTN_OK)
    return rc;

  attn::FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Nq = Nq; p.Nk = Nk;
  if (pk) {
    p.cu_q = pk->cu_q;
    p.cu_k = pk->cu_k;
    p.total_q = pk->total_q;
    p.total_k = pk->total_k;
  }
  p.causal = causal;
  p.window_left = window_left < 0 ? -1 : window_left;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  const int G = Hq / Hkv;
  p.pair_heads = (G % 2 == 0) ? 1 : 0;
  p.n_qblk = (Nq + 127) / 128;
  if (p.pair_heads) {
    p.n_units = p.n_qblk;
    p.n_bh = B * Hkv * (G / 2);
  } else {
    p.n_units = (p.n_qblk + 1) / 2;
    p.n_bh = B * Hq;
  }
  p.nbh_seq = p.n_bh / B;
  p.vl_hg = p.nbh_seq;
  p.hg = p.n_bh;
  if (!pk) {
    // Head groups for the equal-length work list: the largest divisor of n_bh
    // for which two consecutive groups' K/V (the keys one item touches: all of
    // them, or the window plus a row unit) fit in 64 MB of L2. Items run level
    // by level within a group, so every row unit of a head meets its K/V there.
    // Groups are used only when the whole problem's K/V would not stay in
    // L2 next to the Q and O streams (above 96 MB).
    const double span = window_left >= 0 ? std::min<double>(Nk, double(window_left) + 256.0) : Nk;
    const double kv_touch = span * D * 2.0 * 2.0;                 // K and V of one kv head
    const int run = p.pair_heads ? G / 2 : G;                     // consecutive bh sharing a kv head
    if (std::ceil(double(p.n_bh) / run) * kv_touch > 96.0 * (1 << 20)) {
      for (int hg = p.n_bh; hg >= 1; --hg) {
        if (p.n_bh % hg) continue;
        p.hg = hg;
        const double kv_heads = std::ceil(double(hg) / run);
        if (2.0 * kv_heads * kv_touch <= 64.0 * (1 << 20)) break;
      }
    }
  }
  p.per_group = p.n_units * p.hg;
  // bf16 O: staged bulk tensor stores (the kernel keeps the per-row stores as a
  // launch-time alternative, p.bulk_o = 0)
  p.bulk_o = !F32OUT ? 1 : 0;
  if (pk) {
    // Head groups for the packed work list: the largest divisor of the items per
    // (sequence, unit) for which the K/V the concurrently running items touch
    // (estimated from the average sequence) stays within 96 MB of L2.
    const double kv_per_seq_head = double(pk->total_k) / B * D * 2.0 * 2.0;
    const int items_per_kv_head = p.nbh_seq / Hkv;
    for (int hg = p.nbh_seq; hg >= 1; --hg) {
      if (p.nbh_seq % hg) continue;
      const double live = std::min(148.0, double(B) * hg);     // items running at once
      const double kv_heads = std::max(1.0, live / items_per_kv_head);
      p.vl_hg = hg;
      if (kv_heads * kv_per_seq_head <= 96.0 * (1 << 20)) break;
    }
  }
  p.fd_hg = make_fastdiv(p.hg);
  p.fd_vlhg = make_fastdiv(p.vl_hg);
  p.fd_per_b = make_fastdiv(p.nbh_seq);
  p.fd_inner = make_fastdiv(p.pair_heads ? G / 2 : G);
  const long long items = static_cast<long long>(p.n_units) * p.n_bh;
  if (items > kMaxIndex) return fail(ATTN_ERR_INVALID_ARG, "problem too large for one launch");
  if (pk && (B > L::VL_MAX_SEQS || p.n_units > L::VL_MAX_UNITS))
    return fail(ATTN_ERR_INVALID_ARG, "packed input limited to %d sequences and %d row units "
                "(max_seqlen_q %d gives %d)", L::VL_MAX_SEQS, L::VL_MAX_UNITS, Nq, p.n_units);
  p.n_items = static_cast<int>(items);
  int sms = 0;
  if ((rc = sm_count(dev, &sms)) != ATTN_OK) return rc;
  const long long grid = std::min<long long>(items, sms);   // persistent: one CTA per SM

  static std::atomic<unsigned long long> attr_set{0};   // per-device bit
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load() & bit)) {
    // the in-kernel register split needs this many registers per thread at launch
    cudaFuncAttributes fa{};
    cudaError_t e = cudaFuncGetAttributes(&fa, attn::attn_fwd_kernel<D, F32OUT, VARLEN>);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaFuncGetAttributes: %s", cudaGetErrorString(e));
    if (fa.numRegs < attn::kFwdRegsLaunchMin)
      return fail(ATTN_ERR_UNSUPPORTED, "attn_fwd kernel built with %d registers per thread, needs %d",
                  fa.numRegs, attn::kFwdRegsLaunchMin);
    e = cudaFuncSetAttribute(attn::attn_fwd_kernel<D, F32OUT, VARLEN>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM_ALLOC);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    attr_set.fetch_or(bit);
  }
  attn::attn_fwd_kernel<D, F32OUT, VARLEN><<<unsigned(grid), attn::kFwdThreads, L::SMEM_ALLOC, stream>>>(mq, mk, mv, mo, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "attn_fwd launch: %s", cudaGetErrorString(e));
  g_launches.fetch_add(1);
  return ok();
}

int fwd_entry(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
              int Hkv, int Nq, int Nk, int d, float scale, int causal, int window_left,
              cudaStream_t stream, bool f32out, const Packed* pk = nullptr) {
  int rc = validate_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal);
  if (rc != ATTN_OK) return rc;
  int dev = 0;
  if ((rc = check_device(&dev)) != ATTN_OK) return rc;
  if (pk != nullptr) {   // packed sequences: bf16 output only
    return d == 128 ? launch_fwd<128, false, true>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal, window_left, stream, dev, pk)
                    : launch_fwd<64, false, true>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal, window_left, stream, dev, pk);
  }
  if (d == 128) {
    return f32out ? launch_fwd<128, true, false>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal, window_left, stream, dev)
                  : launch_fwd<128, false, false>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal, window_left, stream, dev);
  }
  return f32out ? launch_fwd<64, true, false>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal, window_left, stream, dev)
                : launch_fwd<64, false, false>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal, window_left, stream, dev);
}

// ------------------------------------------------------------------ decode --

constexpr int kNumSMs = 148;

int decode_group_tile(int G) {
  if (G % 4 == 0) return 4;
  if (G % 2 == 0) return 2;
  return 1;
}

// Split count chosen from sizes alone (so the workspace size needs no Hkv):
// assuming work items of four query heads, the smallest split count whose
// items spread over the SMs with at least 95% balance (persistent CTAs take
// items round-robin), each item streaming at least one 128-key tile.
int auto_splits(int B, int Hq, int Lmax) {
  const long long base = std::max(1ll, (static_cast<long long>(B) * Hq + 3) / 4);
  const int cap = static_cast<int>(std::max(1ll, std::min(64ll, (static_cast<long long>(Lmax) + 127) / 128)));
  int best = cap;
  for (int s = 1; s <= cap; ++s) {
    const long long items = base * s;
    const long long rounds = (items + kNumSMs - 1) / kNumSMs;
    if (items >= kNumSMs && double(items) / double(rounds * kNumSMs) >= 0.95) { best = s; break; }
  }
  return best;
}

struct DecodeShape {
  int S;
  int chunk;
  size_t acc_bytes, ml_bytes, total;
  bool too_large;     // the workspace would exceed 2^62 bytes
};

DecodeShape decode_shape(int B, int Hq, int d, int num_splits, int Lmax) {
  // callers pass 1 <= Lmax <= kMaxKeys; 64-bit so that no sum below overflows
  DecodeShape s{};
  const long long L = Lmax;
  long long S = num_splits > 0 ? num_splits : auto_splits(B, Hq, Lmax);
  if (S > L) S = L;
  const long long quantum = 128;                    // keys per K/V tile
  long long chunk = (L + S - 1) / S;
  chunk = (chunk + quantum - 1) / quantum * quantum;
  S = (L + chunk - 1) / chunk;
  s.S = static_cast<int>(S);
  s.chunk = static_cast<int>(chunk);
  // B * Hq * S * (d + 2) floats can pass 2^64 for extreme sizes: count in 128 bits
  const unsigned __int128 rows = static_cast<unsigned __int128>(B) * Hq * S;
  s.too_large = rows * (d + 2) * sizeof(float) > (static_cast<unsigned __int128>(1) << 62);
  if (s.too_large) return s;
  auto round256 = [](size_t x) { return (x + 255) / 256 * 256; };
  s.acc_bytes = round256(static_cast<size_t>(rows) * d * sizeof(float));
  s.ml_bytes = round256(static_cast<size_t>(rows) * 2 * sizeof(float));
  s.total = s.acc_bytes + s.ml_bytes;
  return s;
}

template <int D, int GT, bool PAGED>
int launch_decode_kernels(attn::DecodeParams& p, const void* k_cache, const void* v_cache,
                          cudaStream_t stream, int dev) {
  using L = attn::DecLayout<D>;
  CUtensorMap mk, mv;
  int rc;
  if constexpr (PAGED) {
    const int rows = p.page_size < 128 ? p.page_size : 128;
    if ((rc = make_map_pool(&mk, k_cache, D, p.Hkv, p.page_size, p.num_pages, rows)) != ATTN_OK) return rc;
    if ((rc = make_map_pool(&mv, v_cache, D, p.Hkv, p.page_size, p.num_pages, rows)) != ATTN_OK) return rc;
  } else {
    if ((rc = make_map(&mk, k_cache, D, p.Hkv, p.Lmax, p.B)) != ATTN_OK) return rc;
    if ((rc = make_map(&mv, v_cache, D, p.Hkv, p.Lmax, p.B)) != ATTN_OK) return rc;
  }
  const int G = p.Hq / p.Hkv;
  const long long items = static_cast<long long>(p.B) * p.Hkv * (G / GT) * p.S;
  if (items > kMaxIndex) return fail(ATTN_ERR_INVALID_ARG, "decode problem too large");
  p.n_items = static_cast<int>(items);
  int sms = 0;
  if ((rc = sm_count(dev, &sms)) != ATTN_OK) return rc;
  static std::atomic<unsigned long long> attr_set{0};   // per-device bit
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(attn::decode_split_kernel<D, GT, PAGED>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM_ALLOC);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    attr_set.fetch_or(bit);
  }
  const int grid = static_cast<int>(std::min<long long>(items, sms));
  attn::decode_split_kernel<D, GT, PAGED><<<grid, attn::kDecodeSplitThreads, L::SMEM_ALLOC, stream>>>(mk, mv, p);
  const long long n = static_cast<long long>(p.B) * p.Hq;
  attn::decode_combine_kernel<D><<<unsigned((n + 3) / 4), 128, 0, stream>>>(p);
  return ATTN_OK;
}

// Head dim and group tile are compile-time in the kernels: pick the instance.
template <bool PAGED>
int dispatch_decode(attn::DecodeParams& p, int d, const void* k_cache, const void* v_cache,
                    cudaStream_t stream, int dev) {
  const int GT = decode_group_tile(p.Hq / p.Hkv);
  if (d == 128) {
    if (GT == 4) return launch_decode_kernels<128, 4, PAGED>(p, k_cache, v_cache, stream, dev);
    if (GT == 2) return launch_decode_kernels<128, 2, PAGED>(p, k_cache, v_cache, stream, dev);
    return launch_decode_kernels<128, 1, PAGED>(p, k_cache, v_cache, stream, dev);
  }
  if (GT == 4) return launch_decode_kernels<64, 4, PAGED>(p, k_cache, v_cache, stream, dev);
  if (GT == 2) return launch_decode_kernels<64, 2, PAGED>(p, k_cache, v_cache, stream, dev);
  return launch_decode_kernels<64, 1, PAGED>(p, k_cache, v_cache, stream, dev);
}

// ------------------------------------------------------ no-alloc decode --
// Fixed scratch for attn_decode_noalloc: the library's own device memory, so
// that callers which cannot allocate still get a split-KV decode. Host code
// must not pass this symbol itself to a kernel (on the host it is only a
// stand-in); it passes the device address looked up below.
static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[ATTN_DECODE_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array for device `dev` (the current device),
// looked up once per device and cached.
int noalloc_scratch(int dev, void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  if (dev < 0 || dev >= 64) return fail(ATTN_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_decode_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(ATTN_ERR_CUDA, "cudaGetSymbolAddress(decode scratch): %s", cudaGetErrorString(e));
    addr[dev] = p;
  }
  *out = addr[dev];
  return ATTN_OK;
}

// ---------------------------------------------------------------- backward --

size_t bwd_ws_dq_bytes(int B, int Hq, int Nq, int d) {
  return (static_cast<size_t>(B) * Nq * Hq * d * sizeof(float) + 255) / 256 * 256;
}
size_t bwd_ws_bytes(int B, int Hq, int Nq, int d) {
  return bwd_ws_dq_bytes(B, Hq, Nq, d) +
         (static_cast<size_t>(B) * Hq * Nq * sizeof(float) + 255) / 256 * 256;
}

template <int D>
int launch_bwd(const void* q, const void* k, const void* v, attn::BwdParams& p, cudaStream_t stream,
               int dev) {
  using L = attn::BwdLayout<D>;
  const long long nbh = static_cast<long long>(p.B) * p.Hkv;
  const long long nctas = static_cast<long long>((p.Nk + 127) / 128) * nbh;
  if (nctas > kMaxIndex) return fail(ATTN_ERR_INVALID_ARG, "problem too large for one launch");
  CUtensorMap mq, mk, mv, mdo, mdk, mdv;
  int rc;
  if ((rc = make_map(&mq, q, D, p.Hq, p.Nq, p.B)) != ATTN_OK) return rc;
  if ((rc = make_map(&mk, k, D, p.Hkv, p.Nk, p.B)) != ATTN_OK) return rc;
  if ((rc = make_map(&mv, v, D, p.Hkv, p.Nk, p.B)) != ATTN_OK) return rc;
  if ((rc = make_map(&mdo, p.dout, D, p.Hq, p.Nq, p.B)) != ATTN_OK) return rc;
  // dK, dV leave through 32-row bulk tensor stores
  if ((rc = make_map(&mdk, p.dk, D, p.Hkv, p.Nk, p.B, 32)) != ATTN_OK) return rc;
  if ((rc = make_map(&mdv, p.dv, D, p.Hkv, p.Nk, p.B, 32)) != ATTN_OK) return rc;
  static std::atomic<unsigned long long> attr_set{0};   // per-device bit
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(attn::bwd_main_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM_ALLOC);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    attr_set.fetch_or(bit);
  }
  const long long rows = static_cast<long long>(p.B) * p.Nq * p.Hq;
  attn::bwd_prep_kernel<D><<<unsigned((rows * 32 + 255) / 256), 256, 0, stream>>>(p);
  // chunk of (batch, K/V head) pairs whose Q, dO (bf16) and dQ accumulator
  // (fp32) rows take about 48 MB of L2
  const long long unit = static_cast<long long>(p.Hq / p.Hkv) * p.Nq * D * 8;
  p.bh_chunk = static_cast<int>(std::max(1ll, std::min(nbh, (48ll << 20) / unit)));
  attn::bwd_main_kernel<D><<<unsigned(nctas), attn::kBwdThreads, L::SMEM_ALLOC, stream>>>(mq, mk, mv, mdo, mdk, mdv, p);
  const long long fin = static_cast<long long>(p.B) * p.Hq * ((p.Nq + attn::kFinQ - 1) / attn::kFinQ);
  attn::bwd_finalize_kernel<D><<<unsigned(fin), 256, 0, stream>>>(p);
  return ATTN_OK;
}

}  // namespace

extern "C" {

int attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, void* o,
                        float* lse, const int* seqlens, int B, int Hq, int Hkv, int Lmax, int d,
                        float scale, int window_left, int num_splits, cudaStream_t stream) {
  if (!q || !k_cache || !v_cache || !o)
    return fail(ATTN_ERR_INVALID_ARG, "q, k_cache, v_cache and o must be non-null");
  if (B < 1 || Hq < 1 || Hkv < 1 || Lmax < 1)
    return fail(ATTN_ERR_INVALID_ARG, "B, Hq, Hkv, Lmax must be >= 1");
  if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  if (d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not in {64, 128}", d);
  if (!finite_pos(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (num_splits < 0) return fail(ATTN_ERR_INVALID_ARG, "num_splits must be >= 0");
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16))
    return fail(ATTN_ERR_INVALID_ARG, "q, k_cache, v_cache, o must be 16-byte aligned");
  if (lse && !aligned(lse, 4)) return fail(ATTN_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  if (seqlens && !aligned(seqlens, 4)) return fail(ATTN_ERR_INVALID_ARG, "seqlens must be 4-byte aligned");
  if (static_cast<long long>(B) * Lmax > kMaxIndex || static_cast<long long>(B) * Hq > kMaxIndex ||
      Lmax > kMaxKeys)
    return fail(ATTN_ERR_INVALID_ARG, "sizes too large");
  const DecodeShape sh = decode_shape(B, Hq, d, num_splits, Lmax);
  if (sh.too_large) return fail(ATTN_ERR_INVALID_ARG, "sizes too large");
  if (sh.total > ATTN_DECODE_NOALLOC_SCRATCH_BYTES)
    return fail(ATTN_ERR_WORKSPACE,
                "these sizes need %zu bytes of scratch (%d splits) but the fixed scratch holds %zu; "
                "use attn_decode with a caller workspace or fewer splits",
                sh.total, sh.S, static_cast<size_t>(ATTN_DECODE_NOALLOC_SCRATCH_BYTES));
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != ATTN_OK) return rc;
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(dev, &scratch)) != ATTN_OK) return rc;

  attn::DecodeParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k_cache);
  p.v = static_cast<const uint16_t*>(v_cache);
  p.o = static_cast<uint16_t*>(o);
  p.lse = lse;
  p.seqlens = seqlens;
  p.ws_acc = static_cast<float*>(scratch);
  p.ws_ml = reinterpret_cast<float*>(static_cast<char*>(scratch) + sh.acc_bytes);
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lmax = Lmax;
  p.S = sh.S;
  p.chunk = sh.chunk;
  p.window_left = window_left < 0 ? -1 : window_left;
  p.scale_log2 = scale * 1.4426950408889634f;
  rc = dispatch_decode<false>(p, d, k_cache, v_cache, stream, dev);
  if (rc != ATTN_OK) return rc;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "attn_decode_noalloc launch: %s", cudaGetErrorString(e));
  g_launches.fetch_add(2);
  return ok();
}


int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int Nq, int Nk, int d, float scale, int causal, int window_left,
             cudaStream_t stream) {
  return fwd_entry(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, window_left, stream, false);
}

int attn_fwd_f32o(const void* q, const void* k, const void* v, float* o, float* lse, int B, int Hq,
                  int Hkv, int Nq, int Nk, int d, float scale, int causal, int window_left,
                  cudaStream_t stream) {
  return fwd_entry(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, window_left, stream, true);
}

int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int Hq, int Hkv,
                    int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                    float scale, int causal, int window_left, cudaStream_t stream) {
  if (!cu_seqlens_q || !cu_seqlens_k)
    return fail(ATTN_ERR_INVALID_ARG, "cu_seqlens_q and cu_seqlens_k must be non-null");
  if (!aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4))
    return fail(ATTN_ERR_INVALID_ARG, "cu_seqlens must be 4-byte aligned");
  if (total_q < 1 || total_k < 1)
    return fail(ATTN_ERR_INVALID_ARG, "total_q and total_k must be >= 1");
  if (max_seqlen_q > total_q || max_seqlen_k > total_k)
    return fail(ATTN_ERR_INVALID_ARG, "max_seqlen_q/k cannot exceed total_q/k");
  if (static_cast<long long>(total_q) * Hq > kMaxIndex || static_cast<long long>(total_k) * Hkv > kMaxIndex)
    return fail(ATTN_ERR_INVALID_ARG, "sizes too large");
  const Packed pk{cu_seqlens_q, cu_seqlens_k, total_q, total_k};
  return fwd_entry(q, k, v, o, lse, B, Hq, Hkv, max_seqlen_q, max_seqlen_k, d, scale, causal,
                   window_left, stream, false, &pk);
}

size_t attn_bwd_workspace_bytes(int B, int Hq, int Nq, int d) {
  if (B < 1 || Hq < 1 || Nq < 1 || (d != 64 && d != 128)) return 0;
  // the size limits attn_bwd applies
  if (static_cast<long long>(B) * Nq > kMaxIndex || static_cast<long long>(B) * Hq > kMaxIndex ||
      static_cast<long long>(B) * Nq * Hq > kMaxIndex * 8ll / d)
    return 0;
  return bwd_ws_bytes(B, Hq, Nq, d);
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nk,
             int d, float scale, int causal, int window_left, void* workspace,
             size_t workspace_bytes, cudaStream_t stream) {
  int rc = validate_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal);
  if (rc != ATTN_OK) return rc;
  if (!dout || !lse || !dq || !dk || !dv)
    return fail(ATTN_ERR_INVALID_ARG, "dout, lse, dq, dk and dv must be non-null");
  if (!aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16))
    return fail(ATTN_ERR_INVALID_ARG, "dout, dq, dk, dv must be 16-byte aligned");
  // B * Nq and B * Hq are below 2^31 here, so B * Nq * Hq fits 64 bits
  if (static_cast<long long>(B) * Nq * Hq > kMaxIndex * 8ll / d)
    return fail(ATTN_ERR_INVALID_ARG, "sizes too large");
  const size_t need = bwd_ws_bytes(B, Hq, Nq, d);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(ATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, got %zu", need,
                workspace == nullptr ? size_t(0) : workspace_bytes);
  if (!aligned(workspace, 256)) return fail(ATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  int dev = 0;
  if ((rc = check_device(&dev)) != ATTN_OK) return rc;
  attn::BwdParams p{};
  p.o = static_cast<const uint16_t*>(o);
  p.dout = static_cast<const uint16_t*>(dout);
  p.lse = lse;
  p.dq_acc = static_cast<float*>(workspace);
  p.delta = reinterpret_cast<float*>(static_cast<char*>(workspace) + bwd_ws_dq_bytes(B, Hq, Nq, d));
  p.dq = static_cast<uint16_t*>(dq);
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Nq = Nq; p.Nk = Nk;
  p.causal = causal;
  p.window_left = window_left < 0 ? -1 : window_left;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  rc = d == 128 ? launch_bwd<128>(q, k, v, p, stream, dev) : launch_bwd<64>(q, k, v, p, stream, dev);
  if (rc != ATTN_OK) return rc;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "attn_bwd launch: %s", cudaGetErrorString(e));
  g_launches.fetch_add(3);
  return ok();
}

int attn_merge(const float* o_parts, const float* lse_parts, int R, void* o, float* lse, int B,
               int Nq, int Hq, int d, cudaStream_t stream) {
  if (!o_parts || !lse_parts || !o)
    return fail(ATTN_ERR_INVALID_ARG, "o_parts, lse_parts and o must be non-null");
  if (R < 1 || B < 1 || Nq < 1 || Hq < 1)
    return fail(ATTN_ERR_INVALID_ARG, "R, B, Nq, Hq must be >= 1");
  if (R > 64) return fail(ATTN_ERR_UNSUPPORTED, "at most 64 parts (got %d)", R);
  if (d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not in {64, 128}", d);
  if (!aligned(o_parts, 16) || !aligned(o, 8) || !aligned(lse_parts, 4) || (lse && !aligned(lse, 4)))
    return fail(ATTN_ERR_INVALID_ARG, "o_parts must be 16-byte, o 8-byte, lse 4-byte aligned");
  if (static_cast<long long>(B) * Nq > kMaxIndex || static_cast<long long>(B) * Hq > kMaxIndex)
    return fail(ATTN_ERR_INVALID_ARG, "sizes too large");
  const long long rows = static_cast<long long>(B) * Nq * Hq;     // < 2^62 here
  if (rows > kMaxIndex * 16ll / d || rows > kMaxIndex * 16ll / R)
    return fail(ATTN_ERR_INVALID_ARG, "sizes too large");
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != ATTN_OK) return rc;
  // one warp per (b, head, 32 query rows)
  const long long warps = static_cast<long long>(B) * Hq * ((Nq + 31) / 32);
  const unsigned grid = unsigned((warps * 32 + 255) / 256);
  uint16_t* ob = static_cast<uint16_t*>(o);
  // part count rounded up to a compile-time bound: all loads go out at once
  auto go = [&](auto dtag, auto rtag) {
    constexpr int DD = decltype(dtag)::value, RR = decltype(rtag)::value;
    attn::attn_merge_kernel<DD, RR><<<grid, 256, 0, stream>>>(o_parts, lse_parts, R, ob, lse, B, Nq, Hq);
  };
  using D128 = std::integral_constant<int, 128>;
  using D64 = std::integral_constant<int, 64>;
  auto by_r = [&](auto dtag) {
    if (R <= 2) go(dtag, std::integral_constant<int, 2>{});
    else if (R <= 4) go(dtag, std::integral_constant<int, 4>{});
    else if (R <= 8) go(dtag, std::integral_constant<int, 8>{});
    else if (R <= 16) go(dtag, std::integral_constant<int, 16>{});
    else go(dtag, std::integral_constant<int, 64>{});
  };
  if (d == 128) by_r(D128{});
  else by_r(D64{});
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "attn_merge launch: %s", cudaGetErrorString(e));
  g_launches.fetch_add(1);
  return ok();
}

size_t attn_decode_workspace_bytes(int B, int Hq, int d, int num_splits, int Lmax) {
  if (B < 1 || Hq < 1 || Lmax < 1 || Lmax > kMaxKeys || (d != 64 && d != 128) || num_splits < 0)
    return 0;
  const DecodeShape sh = decode_shape(B, Hq, d, num_splits, Lmax);
  return sh.too_large ? 0 : sh.total;
}

int attn_decode(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                const int* seqlens, int B, int Hq, int Hkv, int Lmax, int d, float scale,
                int window_left, int num_splits, void* workspace, size_t workspace_bytes,
                cudaStream_t stream) {
  if (!q || !k_cache || !v_cache || !o)
    return fail(ATTN_ERR_INVALID_ARG, "q, k_cache, v_cache and o must be non-null");
  if (B < 1 || Hq < 1 || Hkv < 1 || Lmax < 1)
    return fail(ATTN_ERR_INVALID_ARG, "B, Hq, Hkv, Lmax must be >= 1");
  if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  if (d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not in {64, 128}", d);
  if (!finite_pos(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (num_splits < 0) return fail(ATTN_ERR_INVALID_ARG, "num_splits must be >= 0");
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16))
    return fail(ATTN_ERR_INVALID_ARG, "q, k_cache, v_cache, o must be 16-byte aligned");
  if (lse && !aligned(lse, 4)) return fail(ATTN_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  if (seqlens && !aligned(seqlens, 4)) return fail(ATTN_ERR_INVALID_ARG, "seqlens must be 4-byte aligned");
  if (static_cast<long long>(B) * Lmax > kMaxIndex || static_cast<long long>(B) * Hq > kMaxIndex ||
      Lmax > kMaxKeys)
    return fail(ATTN_ERR_INVALID_ARG, "sizes too large");
  const DecodeShape sh = decode_shape(B, Hq, d, num_splits, Lmax);
  if (sh.too_large) return fail(ATTN_ERR_INVALID_ARG, "sizes too large");
  if (workspace == nullptr || workspace_bytes < sh.total)
    return fail(ATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, got %zu", sh.total,
                workspace == nullptr ? size_t(0) : workspace_bytes);
  if (!aligned(workspace, 256)) return fail(ATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != ATTN_OK) return rc;

  attn::DecodeParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k_cache);
  p.v = static_cast<const uint16_t*>(v_cache);
  p.o = static_cast<uint16_t*>(o);
  p.lse = lse;
  p.seqlens = seqlens;
  p.ws_acc = static_cast<float*>(workspace);
  p.ws_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) + sh.acc_bytes);
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lmax = Lmax;
  p.S = sh.S;
  p.chunk = sh.chunk;
  p.window_left = window_left < 0 ? -1 : window_left;
  p.scale_log2 = scale * 1.4426950408889634f;
  rc = dispatch_decode<false>(p, d, k_cache, v_cache, stream, dev);
  if (rc != ATTN_OK) return rc;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "attn_decode launch: %s", cudaGetErrorString(e));
  g_launches.fetch_add(2);
  return ok();
}

int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, void* o, float* lse,
                      const int* block_table, const int* seqlens, int B, int Hq, int Hkv,
                      int num_pages, int page_size, int pages_per_seq, int d, float scale,
                      int window_left, int num_splits, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream) {
  if (!q || !k_pages || !v_pages || !o || !block_table)
    return fail(ATTN_ERR_INVALID_ARG, "q, k_pages, v_pages, o and block_table must be non-null");
  if (B < 1 || Hq < 1 || Hkv < 1 || num_pages < 1 || pages_per_seq < 1)
    return fail(ATTN_ERR_INVALID_ARG, "B, Hq, Hkv, num_pages, pages_per_seq must be >= 1");
  if (!(page_size == 16 || page_size == 32 || page_size == 64 || (page_size >= 128 && page_size % 128 == 0)))
    return fail(ATTN_ERR_INVALID_ARG, "page_size %d must be 16, 32, 64 or a multiple of 128", page_size);
  if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  if (d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not in {64, 128}", d);
  if (!finite_pos(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (num_splits < 0) return fail(ATTN_ERR_INVALID_ARG, "num_splits must be >= 0");
  if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(o, 16))
    return fail(ATTN_ERR_INVALID_ARG, "q, k_pages, v_pages, o must be 16-byte aligned");
  if (!aligned(block_table, 4)) return fail(ATTN_ERR_INVALID_ARG, "block_table must be 4-byte aligned");
  if (lse && !aligned(lse, 4)) return fail(ATTN_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  if (seqlens && !aligned(seqlens, 4)) return fail(ATTN_ERR_INVALID_ARG, "seqlens must be 4-byte aligned");
  const long long Lmax = static_cast<long long>(pages_per_seq) * page_size;
  if (Lmax > kMaxKeys || static_cast<long long>(B) * pages_per_seq > kMaxIndex ||
      static_cast<long long>(B) * Hq > kMaxIndex || static_cast<long long>(num_pages) >= kMaxIndex)
    return fail(ATTN_ERR_INVALID_ARG, "sizes too large");
  const DecodeShape sh = decode_shape(B, Hq, d, num_splits, static_cast<int>(Lmax));
  if (sh.too_large) return fail(ATTN_ERR_INVALID_ARG, "sizes too large");
  if (workspace == nullptr || workspace_bytes < sh.total)
    return fail(ATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, got %zu", sh.total,
                workspace == nullptr ? size_t(0) : workspace_bytes);
  if (!aligned(workspace, 256)) return fail(ATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != ATTN_OK) return rc;

  attn::DecodeParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k_pages);
  p.v = static_cast<const uint16_t*>(v_pages);
  p.o = static_cast<uint16_t*>(o);
  p.lse = lse;
  p.seqlens = seqlens;
  p.ws_acc = static_cast<float*>(workspace);
  p.ws_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) + sh.acc_bytes);
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lmax = static_cast<int>(Lmax);
  p.S = sh.S;
  p.chunk = sh.chunk;
  p.window_left = window_left < 0 ? -1 : window_left;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.block_table = block_table;
  p.page_size = page_size;
  p.pages_per_seq = pages_per_seq;
  p.num_pages = num_pages;
  rc = dispatch_decode<true>(p, d, k_pages, v_pages, stream, dev);
  if (rc != ATTN_OK) return rc;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "attn_decode_paged launch: %s", cudaGetErrorString(e));
  g_launches.fetch_add(2);
  return ok();
}

const char* attn_last_error(void) { return g_err; }

int attn_device_status(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
  int val = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&val, attn::g_attn_status, sizeof(int));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(attn::g_attn_status, &zero, sizeof(int));
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "status word: %s", cudaGetErrorString(e));
  if (val == attn::kStatusBadInput)
    return fail(ATTN_ERR_INVALID_ARG, "a device-side check failed (inconsistent cu_seqlens): "
                                      "the offending sequences were skipped");
  if (val == attn::kStatusBounds)
    return fail(ATTN_ERR_INTERNAL, "a bounds or protocol check of the debug build failed: "
                                   "the access was skipped");
  if (val != 0) return fail(ATTN_ERR_TIMEOUT, "a device-side wait timed out");
  return ok();
}

int attn_debug_checks(void) { return attn::kDebugBounds ? 1 : 0; }

int attn_selftest_wait_timeout(cudaStream_t stream) {
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != ATTN_OK) return rc;
  attn::selftest_wait_kernel<<<1, 32, 0, stream>>>();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "selftest launch: %s", cudaGetErrorString(e));
  g_launches.fetch_add(1);
  return ok();
}

unsigned long long attn_launch_count(void) { return g_launches.load(); }

}  // extern "C"
