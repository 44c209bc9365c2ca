// merge_kernel.cuh — merge attention results computed over disjoint key sets.
//
// Each part r holds, for every query row, the normalised output O_r and the
// log-sum-exp LSE_r of the scores against its own keys. The combined result
// rescales every part to the common maximum before adding ("Chapter 3: MHA
// Limitations, MQA, GQA, and FlashAttention", section 3.5):
//   M = max_r LSE_r,  w_r = exp(LSE_r - M),  L = sum_r w_r,
//   O = sum_r w_r O_r / L,  LSE = M + ln L,
// and a row no part saw a key for gets O = 0, LSE = -inf. Used to assemble
// sequence-sharded (context-parallel) attention from per-shard results.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "sm100_ptx.cuh"

namespace attn {

// One warp per (b, head, 32 consecutive query rows); warps step the head
// fastest, so neighbouring warps read neighbouring rows of the [B, Nq, H, D]
// parts. Parts: o_parts [R][B, Nq, H, D] f32, lse_parts [R][B, H, Nq] f32;
// outputs o [B, Nq, H, D] bf16, lse [B, H, Nq] (or null).
//   1. lane i loads the parts' LSEs of query row q0 + i (coalesced 128-byte
//      reads), forms that row's weights w_r / L and writes its LSE
//      (coalesced);
//   2. the warp then walks its rows with the lanes over the head dim
//      (lane l owns elements [4l, 4l + 4) at D = 128, [2l, 2l + 2) at
//      D = 64); a row's weights come from its lane by shuffle. The rows'
//      loads do not depend on the LSEs, so they go out without waiting for
//      them.
// RMAX >= R bounds the parts at compile time (a part with LSE = -inf gets
// weight exp(-inf) = 0); parts are loaded RC at a time, U rows at a time.
template <int D, int RMAX>
__global__ void __launch_bounds__(256) attn_merge_kernel(const float* __restrict__ o_parts,
                                                         const float* __restrict__ lse_parts,
                                                         int R, uint16_t* __restrict__ o,
                                                         float* __restrict__ lse, int B, int Nq,
                                                         int H) {
  constexpr int EPL = D / 32;
  constexpr int RC = RMAX < 8 ? RMAX : 8;
  constexpr int U = RC <= 2 ? 4 : (RC <= 4 ? 2 : 1);
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int nqc = (Nq + 31) >> 5;
  const long long units = static_cast<long long>(B) * nqc * H;
  if (wid >= units) return;
  const int h = int(wid % H);
  const long long bc = wid / H;                               // b * nqc + q chunk
  const int q0 = int(bc % nqc) * 32, b = int(bc / nqc);
  const int nrows = min(32, Nq - q0);
  const size_t rows = static_cast<size_t>(B) * Nq * H;
  const size_t part_o = rows * D, part_l = rows;
  const size_t lrow = (size_t(b) * H + h) * Nq + q0 + lane;   // this lane's row in [B, H, Nq]

  // 1. weights of row q0 + lane
  float w[RMAX];
  float M = -CUDART_INF_F;
#pragma unroll
  for (int r = 0; r < RMAX; ++r) {
    w[r] = (r < R && lane < nrows) ? __ldg(lse_parts + r * part_l + lrow) : -CUDART_INF_F;
    M = fmaxf(M, w[r]);
  }
  float L = 0.f;
#pragma unroll
  for (int r = 0; r < RMAX; ++r) {
    w[r] = M > -CUDART_INF_F ? expf(w[r] - M) : 0.f;         // 0 for a part with no key
    L += w[r];
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int r = 0; r < RMAX; ++r) w[r] *= inv;
  if (lse != nullptr && lane < nrows && in_bounds(static_cast<long long>(lrow), static_cast<long long>(rows)))
    lse[lrow] = L > 0.f ? M + logf(L) : -CUDART_INF_F;

  // 2. the rows, U at a time
  const size_t row0 = (size_t(b) * Nq + q0) * H + h;         // row (b, q0, h) of [B, Nq, H]
  const float* src = o_parts + row0 * D + lane * EPL;
  uint16_t* dst = o + row0 * D + lane * EPL;
  const size_t rstride = size_t(H) * D;                       // one query row further
  for (int i = 0; i < nrows; i += U) {
    float acc[U][EPL];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[u][e] = 0.f;
#pragma unroll
    for (int r0 = 0; r0 < RMAX; r0 += RC) {
      if (r0 >= R) break;
      float v[U][RC][EPL];
#pragma unroll
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int rc = 0; rc < RC; ++rc) {
          const bool in = i + u < nrows && r0 + rc < R;
          const float* s = src + (r0 + rc) * part_o + (i + u) * rstride;
          if constexpr (EPL == 4) {
            const float4 x = in ? __ldg(reinterpret_cast<const float4*>(s)) : make_float4(0.f, 0.f, 0.f, 0.f);
            v[u][rc][0] = x.x; v[u][rc][1] = x.y; v[u][rc][2] = x.z; v[u][rc][3] = x.w;
          } else {
            const float2 x = in ? __ldg(reinterpret_cast<const float2*>(s)) : make_float2(0.f, 0.f);
            v[u][rc][0] = x.x; v[u][rc][1] = x.y;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int rc = 0; rc < RC; ++rc) {
          const float wr = __shfl_sync(0xffffffffu, w[r0 + rc], (i + u) & 31);
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[u][e] = fmaf(wr, v[u][rc][e], acc[u][e]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (i + u >= nrows) break;
      if (!in_bounds(static_cast<long long>(row0) + static_cast<long long>(i + u) * H,
                     static_cast<long long>(rows)))
        continue;
      uint16_t* d = dst + (i + u) * rstride;
      if constexpr (EPL == 4) {
        *reinterpret_cast<uint2*>(d) = make_uint2(pack_bf16x2(acc[u][0], acc[u][1]),
                                                  pack_bf16x2(acc[u][2], acc[u][3]));
      } else {
        *reinterpret_cast<uint32_t*>(d) = pack_bf16x2(acc[u][0], acc[u][1]);
      }
    }
  }
}

}  // namespace attn
