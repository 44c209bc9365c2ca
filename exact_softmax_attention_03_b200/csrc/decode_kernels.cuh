// decode_kernels.cuh — single-query decode over a contiguous KV cache.
//
// Cached decode reads every visible K/V row once per step and does O(L d)
// arithmetic ("Chapter 3: MHA Limitations, MQA, GQA, and FlashAttention",
// section 3.1: small-batch decode is bandwidth-bound). The keys of each
// (sequence, kv head) are split into chunks; one CTA streams one chunk with
// 16-byte read-only loads, keeps an online-softmax state per key lane-group
// ("Modern Attention ...", section 3: running max / running denominator), and
// writes an unnormalised partial (acc, m, l). A second kernel merges the
// partials of all chunks with the rescale-to-common-maximum rule of
// "Chapter 3 ...", section 3.5, and writes O and the log-sum-exp.
//
// All G = Hq / Hkv query heads of a K/V group are handled by the CTA that
// streams that group's keys (GT at a time), so each K/V byte is read once per
// group ("Chapter 3 ...", section 3.3).
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "sm100_ptx.cuh"

namespace attn {

struct DecodeParams {
  const uint16_t* q;        // [B, Hq, D] bf16
  const uint16_t* k;        // [B, Lmax, Hkv, D] bf16
  const uint16_t* v;        // [B, Lmax, Hkv, D] bf16
  uint16_t* o;              // [B, Hq, D] bf16
  float* lse;               // [B, Hq] or null
  const int* seqlens;       // [B] or null
  float* ws_acc;            // [B, Hq, S, D] unnormalised partial outputs
  float* ws_ml;             // [B, Hq, S, 2] partial (max, sum), max in log2 units
  int B, Hq, Hkv, Lmax, S, chunk;
  int window_left;
  float scale_log2;         // scale * log2(e)
};

constexpr int kDecodeThreads = 128;   // 4 warps
constexpr int kDecodeUnroll = 4;      // passes per loaded block

__device__ __forceinline__ int decode_seqlen(const DecodeParams& p, int b) {
  if (p.seqlens == nullptr) return p.Lmax;
  int L = __ldg(p.seqlens + b);
  return L < 0 ? 0 : (L > p.Lmax ? p.Lmax : L);
}

// Split kernel. grid = (S, Hkv * (G / GT), B), block = 128.
// Lane layout: LPK = D / 8 lanes cover one key row (8 bf16 = 16 bytes each),
// so a warp handles KPP = 32 / LPK keys per pass and the CTA 4 * KPP.
template <int D, int GT>
__global__ void __launch_bounds__(kDecodeThreads)
decode_split_kernel(const DecodeParams p) {
  constexpr int LPK = D / 8;
  constexpr int KPP = 32 / LPK;
  constexpr int U = kDecodeUnroll;
  constexpr int NGRP = 4 * KPP;                 // lane-groups per CTA

  __shared__ float sm_m[GT][NGRP];
  __shared__ float sm_l[GT][NGRP];
  __shared__ __align__(16) float sm_acc[NGRP][GT][D];

  const int split = blockIdx.x;
  const int b = blockIdx.z;
  const int G = p.Hq / p.Hkv;
  const int tiles_per_kv = G / GT;
  const int hkv = blockIdx.y / tiles_per_kv;
  const int hq0 = hkv * G + (blockIdx.y % tiles_per_kv) * GT;

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int sub = lane / LPK;                   // key slot within the warp's pass
  const int c8 = (lane % LPK) * 8;              // first head-dim element of this lane
  const int grp = warp * KPP + sub;

  const int L = decode_seqlen(p, b);
  int lo = 0;
  if (p.window_left >= 0) lo = max(0, L - 1 - p.window_left);
  const int k_begin = max(lo, split * p.chunk);
  const int k_end = min(L, (split + 1) * p.chunk);
  const int n_keys = k_end - k_begin;
  const int n_pass = n_keys > 0 ? (n_keys + 4 * KPP - 1) / (4 * KPP) : 0;

  // query rows of this group tile, pre-scaled into log2 units
  float qf[GT][8];
#pragma unroll
  for (int g = 0; g < GT; ++g) {
    const uint4 raw = *reinterpret_cast<const uint4*>(p.q + (size_t(b) * p.Hq + hq0 + g) * D + c8);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      qf[g][2 * e] = bf16lo(w[e]) * p.scale_log2;
      qf[g][2 * e + 1] = bf16hi(w[e]) * p.scale_log2;
    }
  }

  float acc[GT][8];
  float m[GT], l[GT];
#pragma unroll
  for (int g = 0; g < GT; ++g) {
    m[g] = -CUDART_INF_F;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
  }

  const size_t key_stride = size_t(p.Hkv) * D;  // elements between consecutive keys
  const uint16_t* kb = p.k + (size_t(b) * p.Lmax * p.Hkv + hkv) * D + c8;
  const uint16_t* vb = p.v + (size_t(b) * p.Lmax * p.Hkv + hkv) * D + c8;

  uint4 kc[U], vc[U];
  auto load_block = [&](int t0, uint4 (&kr)[U], uint4 (&vr)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int key = k_begin + ((t0 + u) * 4 + warp) * KPP + sub;
      if (t0 + u < n_pass && key < k_end) {
        kr[u] = ld_nc_v4(kb + size_t(key) * key_stride);
        vr[u] = ld_nc_v4(vb + size_t(key) * key_stride);
      } else {
        kr[u] = make_uint4(0, 0, 0, 0);
        vr[u] = make_uint4(0, 0, 0, 0);
      }
    }
  };

  if (n_pass > 0) load_block(0, kc, vc);
  for (int t0 = 0; t0 < n_pass; t0 += U) {
    uint4 kn[U], vn[U];
    load_block(t0 + U, kn, vn);                 // prefetch the next block

    float s[U][GT];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t w[4] = {kc[u].x, kc[u].y, kc[u].z, kc[u].w};
      float kf[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        kf[2 * e] = bf16lo(w[e]);
        kf[2 * e + 1] = bf16hi(w[e]);
      }
#pragma unroll
      for (int g = 0; g < GT; ++g) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaf(qf[g][e], kf[e], a);
#pragma unroll
        for (int off = LPK / 2; off >= 1; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
        s[u][g] = a;
      }
      const int key = k_begin + ((t0 + u) * 4 + warp) * KPP + sub;
      if (!(t0 + u < n_pass && key < k_end)) {
#pragma unroll
        for (int g = 0; g < GT; ++g) s[u][g] = -CUDART_INF_F;
      }
    }

#pragma unroll
    for (int g = 0; g < GT; ++g) {
      float mb = s[0][g];
#pragma unroll
      for (int u = 1; u < U; ++u) mb = fmaxf(mb, s[u][g]);
      const float mn = fmaxf(m[g], mb);
      if (mn == -CUDART_INF_F) continue;        // nothing visible yet in this group
      const float alpha = ex2_approx(m[g] - mn);  // m = -inf gives 0
      float ps[U];
      float lsum = 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        ps[u] = ex2_approx(s[u][g] - mn);
        lsum += ps[u];
      }
      l[g] = fmaf(l[g], alpha, lsum);
      m[g] = mn;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[g][e] *= alpha;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t w[4] = {vc[u].x, vc[u].y, vc[u].z, vc[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[g][2 * e] = fmaf(ps[u], bf16lo(w[e]), acc[g][2 * e]);
          acc[g][2 * e + 1] = fmaf(ps[u], bf16hi(w[e]), acc[g][2 * e + 1]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      kc[u] = kn[u];
      vc[u] = vn[u];
    }
  }

  // ---- merge the lane-groups of this CTA ---------------------------------
  if ((lane % LPK) == 0) {
#pragma unroll
    for (int g = 0; g < GT; ++g) {
      sm_m[g][grp] = m[g];
      sm_l[g][grp] = l[g];
    }
  }
#pragma unroll
  for (int g = 0; g < GT; ++g) {
    float4* dst = reinterpret_cast<float4*>(&sm_acc[grp][g][c8]);
    dst[0] = make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
    dst[1] = make_float4(acc[g][4], acc[g][5], acc[g][6], acc[g][7]);
  }
  __syncthreads();

  // thread t covers (g, d) pairs t, t + 128, ...
  for (int idx = threadIdx.x; idx < GT * D; idx += kDecodeThreads) {
    const int g = idx / D;
    const int dd = idx % D;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int r = 0; r < NGRP; ++r) M = fmaxf(M, sm_m[g][r]);
    float Lsum = 0.f, a = 0.f;
    if (M != -CUDART_INF_F) {
#pragma unroll
      for (int r = 0; r < NGRP; ++r) {
        const float w = ex2_approx(sm_m[g][r] - M);
        Lsum = fmaf(sm_l[g][r], w, Lsum);
        a = fmaf(sm_acc[r][g][dd], w, a);
      }
    }
    const size_t row = (size_t(b) * p.Hq + hq0 + g) * p.S + split;
    p.ws_acc[row * D + dd] = a;
    if (dd == 0) {
      p.ws_ml[row * 2 + 0] = M;
      p.ws_ml[row * 2 + 1] = Lsum;
    }
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
