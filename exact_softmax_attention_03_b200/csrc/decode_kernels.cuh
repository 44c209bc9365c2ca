// decode_kernels.cuh — single-query decode over a contiguous KV cache.
//
// Cached decode reads every visible K/V row once per step and does O(L d)
// arithmetic ("Chapter 3: MHA Limitations, MQA, GQA, and FlashAttention",
// section 3.1: small-batch decode is bandwidth-bound). The keys of each
// (sequence, kv head) are split into chunks; a persistent CTA streams one
// chunk at a time through shared memory with TMA, keeps online-softmax
// states ("Modern Attention ...", section 3: running max / running
// denominator), and writes an unnormalised partial (acc, m, l). A second
// kernel merges the partials of all chunks with the rescale-to-common-maximum
// rule of "Chapter 3 ...", section 3.5, and writes O and the log-sum-exp.
//
// All G = Hq / Hkv query heads of a K/V group are handled by the CTA that
// streams that group's keys (GT at a time), so each K/V byte is read once per
// group tile ("Chapter 3 ...", section 3.3).
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "sm100_ptx.cuh"

namespace attn {

// 5-D tiled TMA load (paged pool viewed as {64, d/64, Hkv, page rows, pages}).
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "r"(c4), "r"(bar)
      : "memory");
}

struct DecodeParams {
  const uint16_t* q;        // [B, Hq, D] bf16
  const uint16_t* k;        // [B, Lmax, Hkv, D] bf16 (paged: [num_pages, page_size, Hkv, D])
  const uint16_t* v;        // same layout as k
  uint16_t* o;              // [B, Hq, D] bf16
  float* lse;               // [B, Hq] or null
  const int* seqlens;       // [B] or null
  float* ws_acc;            // [B, Hq, S, D] unnormalised partial outputs
  float* ws_ml;             // [B, Hq, S, 2] partial (max, sum), max in log2 units
  int B, Hq, Hkv, Lmax, S, chunk;
  int window_left;
  float scale_log2;         // scale * log2(e)
  int n_items;              // B * Hkv * (G / GT) * S
  // paged cache only: logical key t of sequence b is row t % page_size of page
  // block_table[b * pages_per_seq + t / page_size]
  const int* block_table;   // [B, pages_per_seq] int32
  int page_size, pages_per_seq, num_pages;
};


__device__ __forceinline__ int decode_seqlen(const DecodeParams& p, int b) {
  if (p.seqlens == nullptr) return p.Lmax;
  int L = __ldg(p.seqlens + b);
  return L < 0 ? 0 : (L > p.Lmax ? p.Lmax : L);
}

// ---- split kernel -----------------------------------------------------------
//
// Persistent CTAs (one per SM) walk the work items (sequence, K/V head, group
// tile of GT query heads, key split). Warp 8 streams each split's keys as
// 128-key K and V tiles through a 3-stage TMA ring (128-byte swizzled, the
// same 4-D view of the cache as the prefill kernel uses). Warps 0-7 each own
// 16 keys of every tile:
//   Q.K:  two lanes per key, each over half of the head dim, reading 16-byte
//         chunks of the swizzled K rows (bank-conflict free) and the query
//         rows from shared memory (broadcast), with bf16 x bf16 -> fp32 fused
//         multiply-adds (no unpacking of the bf16 operands);
//   softmax: warp-wide running max per query head, exp2 in the log2 domain;
//   P.V:  lanes split the head dim; P (bf16) goes through shared memory.
// Each warp keeps its own (max, sum, accumulator); at the end of a split the
// eight warps' states are merged and written as one partial.
template <int D>
struct DecLayout {
  static constexpr int BN = 128;                         // keys per stage
  static constexpr int TILE = BN * D * 2;                // one K or V stage tile
  static constexpr int HALF = 128 * 128;                 // one 64-column swizzle block
  static constexpr int STAGES = 3;
  static constexpr int GT_MAX = 4;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = STAGES * TILE;
  static constexpr int OFF_Q = 2 * STAGES * TILE;                    // [GT][D] bf16
  static constexpr int OFF_P = OFF_Q + GT_MAX * D * 2;                // [8 warps][16 keys][GT] u32
  static constexpr int OFF_ML = OFF_P + 8 * 16 * GT_MAX * 4;          // [8][GT][2] f32
  static constexpr int OFF_ACC = OFF_ML + 8 * GT_MAX * 2 * 4;         // [8][GT][D] f32
  static constexpr int OFF_BAR = OFF_ACC + 8 * GT_MAX * D * 4;
  // barriers: full[STAGES], empty[STAGES], consumer sync, drain
  static constexpr int NBAR = 2 * STAGES + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;                 // abort flag
  // [1] stages the producer loaded, [2] stages the consumers used (compared at
  // the end of the CTA in the bounds-checking debug build)
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = BYTES + 1024;
};

constexpr int kDecodeSplitThreads = 288;   // 8 consumer warps + 1 producer warp

struct DecItem {
  int b, hkv, hq0, split;
  int k_first, n_stages;     // first key of the first 128-key tile, tiles to visit
  int lo, hi;                // visible keys [lo, hi)
};

template <int GT>
__device__ __forceinline__ void dec_item(const DecodeParams& p, int item, DecItem& it) {
  const int G = p.Hq / p.Hkv;
  const int ntile = G / GT;
  it.split = item % p.S;
  int rest = item / p.S;
  const int gt = rest % ntile;
  rest /= ntile;
  it.hkv = rest % p.Hkv;
  it.b = rest / p.Hkv;
  it.hq0 = it.hkv * G + gt * GT;
  const int L = decode_seqlen(p, it.b);
  int lo = 0;
  if (p.window_left >= 0) lo = max(0, L - 1 - p.window_left);
  it.lo = lo;
  it.hi = min(L, (it.split + 1) * p.chunk);
  it.k_first = max(it.split * p.chunk, (lo / 128) * 128);
  it.n_stages = it.hi > it.k_first ? (it.hi - it.k_first + 127) / 128 : 0;
}

// acc_lo += a.lo * b.lo and acc_hi += a.hi * b.hi for bf16 pairs a, b.
__device__ __forceinline__ void fma_bf16x2(float& acc_lo, float& acc_hi, uint32_t a, uint32_t b) {
  asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\t"
      "mov.b32 {a0, a1}, %2;\n\tmov.b32 {b0, b1}, %3;\n\t"
      "fma.rn.f32.bf16 %0, a0, b0, %0;\n\tfma.rn.f32.bf16 %1, a1, b1, %1;\n\t}"
      : "+f"(acc_lo), "+f"(acc_hi)
      : "r"(a), "r"(b));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// PAGED: the K/V tensor maps view the page pool as [num_pages, page_size,
// Hkv, D] with boxes of min(page_size, 128) rows; each 128-key tile is one box
// per 64-column half (page_size a multiple of 128) or 128 / page_size boxes
// (page_size 16, 32 or 64), each from the page the block table names. Pages
// wholly past the visible keys are read at page index num_pages, outside the
// map, which the copy engine fills with zeros (same byte count, no stale data).
template <int D, int GT, bool PAGED>
__global__ void __launch_bounds__(kDecodeSplitThreads, 1)
decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const DecodeParams p) {
  using L = DecLayout<D>;
  constexpr int EPL = D / 32;                  // head-dim elements per lane in P.V
  constexpr int NCH = D / 16;                  // 16-byte chunks per lane in Q.K (half of a row)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::OFF_BAR + 8u * uint32_t(i); };
  const int B_FULL = 0, B_EMPTY = L::STAGES, B_SYNC = 2 * L::STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 8);
    }
    mbar_init(bar(B_SYNC), 256);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int n_items = p.n_items;
  if (warp == 8) {
    // ======================= TMA producer ====================================
    // The whole warp walks the stages (waits agree through a warp vote). Lane 0
    // announces each stage's bytes; the copies are issued by lane 0 (contiguous
    // cache) or, for a paged cache, by lane i for box i, in parallel.
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    int st = 0;
    bool alive = true;
    // paged: this lane's box of the next stage has its page read from the block
    // table one stage ahead, so the read overlaps the wait for a free slot
    const int ps = PAGED ? p.page_size : 128;
    const int rows = ps < 128 ? ps : 128;              // keys per box
    const bool box_lane = PAGED && lane * rows < 128;
    int page_next = 0;
    auto fetch_page = [&](const DecItem& w, int s) -> int {
      const int t = w.k_first + 128 * s + lane * rows;
      const long long ti = static_cast<long long>(w.b) * p.pages_per_seq + t / ps;
      return t < w.hi && in_bounds(ti, static_cast<long long>(p.B) * p.pages_per_seq)
                 ? __ldg(p.block_table + ti) : p.num_pages;
    };
    for (int item = blockIdx.x; alive && item < n_items; item += gridDim.x) {
      DecItem w;
      dec_item<GT>(p, item, w);
      if (box_lane && w.n_stages > 0) page_next = fetch_page(w, 0);
      for (int s = 0; s < w.n_stages; ++s, ++st) {
        const int slot = st % L::STAGES;
        const uint32_t ph = uint32_t(st / L::STAGES) & 1u;
        const int page_cur = page_next;
        if (box_lane && s + 1 < w.n_stages) page_next = fetch_page(w, s + 1);
        if (!(alive = __all_sync(0xffffffffu, mbar_wait(bar(B_EMPTY + slot), ph ^ 1u, abort_flag))))
          break;
        if (lane == 0) mbar_arrive_expect_tx(bar(B_FULL + slot), 2 * L::TILE);
        const int key0 = w.k_first + 128 * s;
        if constexpr (!PAGED) {
          if (lane == 0) {
            for (int c = 0; c < D / 64; ++c) {
              tma_load_4d(sb + L::OFF_K + slot * L::TILE + c * L::HALF, &tmK, bar(B_FULL + slot),
                          c * 64, w.hkv, key0, w.b);
              tma_load_4d(sb + L::OFF_V + slot * L::TILE + c * L::HALF, &tmV, bar(B_FULL + slot),
                          c * 64, w.hkv, key0, w.b);
            }
          }
        } else if (box_lane) {
          // one copy per page brings every 64-column block of its rows: the
          // stage image is [row][block][64] (128-byte line = row * D/64 + block)
          const int r0 = lane * rows;
          const int prow = (key0 + r0) % ps;
          const uint32_t off = slot * L::TILE + r0 * (D / 64) * 128;
          tma_load_5d(sb + L::OFF_K + off, &tmK, bar(B_FULL + slot), 0, 0, w.hkv, prow, page_cur);
          tma_load_5d(sb + L::OFF_V + off, &tmV, bar(B_FULL + slot), 0, 0, w.hkv, prow, page_cur);
        }
        __syncwarp();
      }
    }
    // no copy may still be landing at exit: wait for the last phase of each stage
    for (int i = max(0, st - L::STAGES); i < st; ++i)
      mbar_wait(bar(B_FULL + i % L::STAGES), uint32_t(i / L::STAGES) & 1u, nullptr);
    if (lane == 0) reinterpret_cast<volatile int*>(smem + L::OFF_MISC)[1] = st;
    __syncwarp();
  } else {
    // ======================= consumer warps ==================================
    const int key_in_warp = lane >> 1;         // Q.K: key of this lane within the warp's 16
    const int dh = lane & 1;                   // Q.K: which half of the head dim
    const int row = 16 * warp + key_in_warp;   // row of this lane's key in the stage tile
    int st = 0, syncs = 0;
    bool ok = true;
    uint32_t* pbuf = reinterpret_cast<uint32_t*>(smem + L::OFF_P) + warp * 16 * GT;
    float* red_ml = reinterpret_cast<float*>(smem + L::OFF_ML);
    float* red_acc = reinterpret_cast<float*>(smem + L::OFF_ACC);
    auto consumer_sync = [&]() -> bool {
      mbar_arrive(bar(B_SYNC));
      const bool w = mbar_wait(bar(B_SYNC), uint32_t(syncs & 1), abort_flag);
      ++syncs;
      return __all_sync(0xffffffffu, w);
    };
    for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
      DecItem w;
      dec_item<GT>(p, item, w);
      // query rows of this group tile -> shared memory (bf16, 16 bytes per thread)
      for (int i = threadIdx.x; i < GT * D / 8; i += 256) {
        const int g = i / (D / 8), c = i % (D / 8);
        if (!in_bounds((static_cast<long long>(w.b) * p.Hq + w.hq0 + g), static_cast<long long>(p.B) * p.Hq))
          continue;
        *reinterpret_cast<uint4*>(smem + L::OFF_Q + (g * D + 8 * c) * 2) =
            *reinterpret_cast<const uint4*>(p.q + (size_t(w.b) * p.Hq + w.hq0 + g) * D + 8 * c);
      }
      if (!(ok = consumer_sync())) break;

      float m[GT], lsum[GT], acc[GT][EPL];
#pragma unroll
      for (int g = 0; g < GT; ++g) {
        m[g] = -CUDART_INF_F;
        lsum[g] = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
      }
      for (int s = 0; s < w.n_stages; ++s, ++st) {
        const int slot = st % L::STAGES;
        const uint32_t ph = uint32_t(st / L::STAGES) & 1u;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(B_FULL + slot), ph, abort_flag)))) break;
        const uint32_t ks = sb + L::OFF_K + slot * L::TILE;
        const uint32_t vs = sb + L::OFF_V + slot * L::TILE;
        const int key0 = w.k_first + 128 * s;

        // ---- Q.K for this lane's key, its half of the head dim ----------------
        float de[GT], dodd[GT];
#pragma unroll
        for (int g = 0; g < GT; ++g) { de[g] = 0.f; dodd[g] = 0.f; }
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          // rotate the chunk order of the second half so a phase of 8 lanes
          // touches 8 different 16-byte bank groups
          const int ci = dh ? ((i + NCH / 2) % NCH) : i;
          const int c = dh * NCH + ci;                     // chunk of the full row
          uint32_t kaddr;
          if constexpr (PAGED) {
            const int line = row * (D / 64) + c / 8;
            kaddr = ks + line * 128 + (((c % 8) ^ (line & 7)) * 16);
          } else {
            kaddr = ks + (c / 8) * L::HALF + row * 128 + (((c % 8) ^ (row & 7)) * 16);
          }
          const uint4 kv = lds128(kaddr);
#pragma unroll
          for (int g = 0; g < GT; ++g) {
            const uint4 qv = lds128(sb + L::OFF_Q + (g * D + 8 * c) * 2);
            fma_bf16x2(de[g], dodd[g], kv.x, qv.x);
            fma_bf16x2(de[g], dodd[g], kv.y, qv.y);
            fma_bf16x2(de[g], dodd[g], kv.z, qv.z);
            fma_bf16x2(de[g], dodd[g], kv.w, qv.w);
          }
        }
        const int key = key0 + row;
        const bool valid = key >= w.lo && key < w.hi;
        float sc[GT], wmax[GT];
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          float d = de[g] + dodd[g];
          d += __shfl_xor_sync(0xffffffffu, d, 1);
          sc[g] = valid ? d * p.scale_log2 : -CUDART_INF_F;
          wmax[g] = sc[g];
        }
#pragma unroll
        for (int off = 2; off < 32; off <<= 1) {
#pragma unroll
          for (int g = 0; g < GT; ++g) wmax[g] = fmaxf(wmax[g], __shfl_xor_sync(0xffffffffu, wmax[g], off));
        }
        // ---- online softmax over this warp's 16 keys --------------------------
        float alpha[GT];
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          const float mn = fmaxf(m[g], wmax[g]);
          alpha[g] = (m[g] == -CUDART_INF_F) ? 0.f : ex2_approx(m[g] - mn);
          const float mu = (mn == -CUDART_INF_F) ? 0.f : mn;
          const float pr = ex2_approx(sc[g] - mu);          // 0 for masked keys
          const uint32_t pb = pack_bf16x2(pr, pr);           // bf16 P for P.V, both halves
          lsum[g] = fmaf(lsum[g], alpha[g], dh ? 0.f : pr);  // the sum keeps fp32 P
          if (dh == 0) pbuf[key_in_warp * GT + g] = pb;
          m[g] = mn;
        }
        __syncwarp();
        // ---- P.V: lanes split the head dim ------------------------------------
#pragma unroll
        for (int g = 0; g < GT; ++g)
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[g][e] *= alpha[g];
        const int d0 = lane * EPL;                          // first head-dim element
        const int vc = d0 / 8;                              // its 16-byte chunk
        const uint32_t vbase = vs + (vc / 8) * L::HALF + ((d0 * 2) % 16);
#pragma unroll 4
        for (int kk = 0; kk < 16; ++kk) {
          const int r = 16 * warp + kk;
          uint32_t va;
          if constexpr (PAGED) {
            const int line = r * (D / 64) + vc / 8;
            va = vs + line * 128 + (((vc % 8) ^ (line & 7)) * 16) + ((d0 * 2) % 16);
          } else {
            va = vbase + r * 128 + (((vc % 8) ^ (r & 7)) * 16);
          }
          uint32_t v2[EPL / 2];
          if constexpr (EPL == 4) {
            asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v2[0]), "=r"(v2[1]) : "r"(va));
          } else {
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v2[0]) : "r"(va));
          }
#pragma unroll
          for (int g = 0; g < GT; ++g) {
            const uint32_t pp = pbuf[kk * GT + g];
#pragma unroll
            for (int e = 0; e < EPL / 2; ++e) fma_bf16x2(acc[g][2 * e], acc[g][2 * e + 1], v2[e], pp);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_EMPTY + slot));
      }
      if (!ok) break;

      // ---- merge the eight warps' states into one partial -------------------
#pragma unroll
      for (int g = 0; g < GT; ++g) {
        float l = lsum[g];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
        if (lane == 0) {
          red_ml[(warp * GT + g) * 2 + 0] = m[g];
          red_ml[(warp * GT + g) * 2 + 1] = l;
        }
#pragma unroll
        for (int e = 0; e < EPL; ++e) red_acc[(warp * GT + g) * D + lane * EPL + e] = acc[g][e];
      }
      if (!(ok = consumer_sync())) break;
      for (int idx = threadIdx.x; idx < GT * D; idx += 256) {
        const int g = idx / D, dd = idx % D;
        float M = -CUDART_INF_F;
#pragma unroll
        for (int r = 0; r < 8; ++r) M = fmaxf(M, red_ml[(r * GT + g) * 2]);
        float Ls = 0.f, a = 0.f;
        if (M != -CUDART_INF_F) {
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const float wt = ex2_approx(red_ml[(r * GT + g) * 2] - M);
            Ls = fmaf(red_ml[(r * GT + g) * 2 + 1], wt, Ls);
            a = fmaf(red_acc[(r * GT + g) * D + dd], wt, a);
          }
        }
        const size_t prow = (size_t(w.b) * p.Hq + w.hq0 + g) * p.S + w.split;
        const long long n_part = static_cast<long long>(p.B) * p.Hq * p.S;   // partial rows
        if (!in_bounds(static_cast<long long>(prow), n_part)) continue;
        p.ws_acc[prow * D + dd] = a;
        if (dd == 0) {
          p.ws_ml[prow * 2 + 0] = M;
          p.ws_ml[prow * 2 + 1] = Ls;
        }
      }
      if (!(ok = consumer_sync())) break;
    }
    if (threadIdx.x == 0) reinterpret_cast<volatile int*>(smem + L::OFF_MISC)[2] = st;
  }
  __syncthreads();
  if (kDebugBounds && threadIdx.x == 0 && *abort_flag == 0) {
    const volatile int* cnt = reinterpret_cast<const volatile int*>(smem + L::OFF_MISC);
    (void)same_count(cnt[1], cnt[2]);                  // stages loaded = stages used
  }
}

// Combine kernel: one warp per (b, hq). grid = ceil(B * Hq / 4), block = 128.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
  constexpr int EPL = D / 32;                   // elements per lane
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x * 4 + warp;
  if (bh >= p.B * p.Hq) return;
  if (!in_bounds(bh, static_cast<long long>(p.B) * p.Hq)) return;
  const int S = p.S;
  const float* ml = p.ws_ml + size_t(bh) * S * 2;

  float M = -CUDART_INF_F;
  for (int s = lane; s < S; s += 32) M = fmaxf(M, ml[2 * s]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));

  float out[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) out[e] = 0.f;
  float Lsum = 0.f;
  if (M != -CUDART_INF_F) {
    for (int s = 0; s < S; ++s) {
      const float ms = ml[2 * s];
      const float w = ex2_approx(ms - M);       // empty split: exp2(-inf) = 0
      Lsum = fmaf(ml[2 * s + 1], w, Lsum);
      const float* a = p.ws_acc + (size_t(bh) * S + s) * D + lane * EPL;
#pragma unroll
      for (int e = 0; e < EPL; ++e) out[e] = fmaf(a[e], w, out[e]);
    }
  }
  const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
  uint16_t* o = p.o + size_t(bh) * D + lane * EPL;
#pragma unroll
  for (int e = 0; e < EPL; e += 2) {
    *reinterpret_cast<uint32_t*>(o + e) = pack_bf16x2(out[e] * inv, out[e + 1] * inv);
  }
  if (p.lse != nullptr && lane == 0) {
    p.lse[bh] = Lsum > 0.f ? (M + __log2f(Lsum)) * 0.6931471805599453f : -CUDART_INF_F;
  }
}

}  // namespace attn
